/*
 * sbl.h -- C ABI of the B200 (sm_100a) Sparse-BitLinear library (libsbl.so).
 *
 * The layer follows the Sparse-BitNet summary (paper-graph-ui, arXiv
 * 2603.05168), section 3.4, "The Full Sparse-BitLinear Layer: Forward and
 * Backward Pass": fp32 master weights are masked (N:M by magnitude) and
 * ternarised (absmean), activations are quantised to int8 per token, the
 * masked ternary weights multiply the int8 activations with int32
 * accumulation, one scalar per token restores the scale, and the backward is
 * the Dual straight-through estimator.
 *
 * Conventions for every entry point:
 *  - Every data pointer is a DEVICE pointer (cudaMalloc / PyTorch memory)
 *    owned by the caller; the library never allocates, frees or keeps them.
 *  - Row-major layouts.  O = out_features (d_out), K = in_features (d_in),
 *    T = tokens.  Weights are [O, K]; activations are [T, K]; outputs [T, O].
 *  - bf16 tensors are passed as uint16_t bit patterns.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *    only enqueues work on that stream and returns; none synchronises.
 *  - Arguments are validated on the host before anything is launched; an
 *    invalid call returns an error status and enqueues nothing.
 *  - Data pointers must be 16-byte aligned (SBL_ERR_ALIGNMENT otherwise).
 *  - Inputs must be finite; results for NaN/Inf inputs are unspecified.
 *  - The library needs an sm_100 device (B200); other devices get
 *    SBL_ERR_DEVICE.
 *  - A device-side wait that exceeds its time limit (it never should) makes
 *    the kernel record a code readable with sbl_device_error() and return.
 *  - Host calls are thread-safe: the per-device setup of the first call is
 *    done once under a lock.  Calls may run concurrently (several host
 *    threads, several streams) as long as they share no output buffer and
 *    no workspace; sbl_quantize_mask_pack_noalloc shares one scratch per
 *    device, so its calls must be ordered on one stream.
 *  - Results are deterministic: the same inputs give bit-identical outputs
 *    whatever the stream, the concurrency or the launch order.
 */
#ifndef SBL_H
#define SBL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SBL_OK = 0,
    SBL_ERR_INVALID_ARG = 1,  /* null pointer, unknown enum value          */
    SBL_ERR_SHAPE = 2,        /* sizes out of range or not divisible       */
    SBL_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned          */
    SBL_ERR_UNSUPPORTED = 4,  /* valid but not implemented (n:m, format)   */
    SBL_ERR_WORKSPACE = 5,    /* workspace missing or too small            */
    SBL_ERR_CUDA = 6,         /* a CUDA runtime call or launch failed      */
    SBL_ERR_DEVICE = 7        /* no sm_100 device current                  */
} sbl_status;

/* Packed weight formats (bit mask for sbl_quantize_mask_pack).
 *  PK2   2-bit codes of W_eff, code = w + 1 ({-1,0,+1} -> {0,1,2}, following
 *        the 2-bit packing of the BitNet b1.58 2B4T summary, "Inference
 *        Implementation: GPU"); weight k of a row sits at bits 2*(k%4) of
 *        byte k/4; rows are padded to a multiple of 16 bytes with 0x55
 *        (zero weights).  Layout [O, sbl_packed_row_bytes(PK2)] uint8.
 *  NM    compressed: per row, the 2-bit codes of the kept positions in
 *        ascending order, four per byte LSB-first, padded to 16 bytes with
 *        code 1 ([O, row_bytes(NM values)] uint8), plus a keep bitmap (bit
 *        k%8 of byte k/8 set when position k is kept, padded with 0 bits to
 *        16 bytes; [O, row_bytes(NM bitmap)] uint8).
 *  I8    W_eff as int8 [O, K] (the GEMM operand).
 *  BF16T W_eff transposed, bf16 [K, O] (the dX operand of the backward).
 *  SP24  W_eff as the operand of the 2:4 sparse tensor-core MMA, for masks
 *        with at most two kept weights in every group of four (n <= 2,
 *        m = 4 or 8; other n:m give SBL_ERR_UNSUPPORTED).  For group g of
 *        a row (positions 4g .. 4g+3) two positions i0 < i1 are stored: the
 *        kept ones, completed with the smallest positions not kept when
 *        fewer than two are kept.  Values: int8 W_eff at 4g+i0 and 4g+i1 in
 *        bytes 2g, 2g+1 ([O, row_bytes(SP24 main)] int8, row_bytes =
 *        K/2 rounded up to 16).  Metadata: nibble i0 | (i1 << 2) at bits
 *        4*(g%2) of byte g/2 ([O, row_bytes(SP24 meta)] uint8, K/8 rounded
 *        up to 16).  Padding bytes are 0.
 *  T24   W_eff in 6 bits per group of four, for the same masks as SP24 (a
 *        denser form of the 2-bit packing of the BitNet b1.58 2B4T summary,
 *        "Inference Implementation: GPU"): group g with nonzero positions
 *        p < q and sign bits s (1 for -1) has code 0 (none), 1 + 2p + s_p
 *        (one), or 9 + 4k + 2 s_p + s_q (two; k = index of (p, q) in
 *        (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)).  Low plane: code & 15 at bits
 *        4*(g%2) of byte g/2 ([O, row_bytes(T24 main)], K/8 rounded up to
 *        16); high plane: code >> 4 at bits 2*(g%4) of byte g/4 ([O,
 *        row_bytes(T24 high)], K/16 rounded up to 16).  Padding bytes 0. */
typedef enum {
    SBL_FMT_PK2 = 1,
    SBL_FMT_NM = 2,
    SBL_FMT_I8 = 4,
    SBL_FMT_BF16T = 8,
    SBL_FMT_SP24 = 16,
    SBL_FMT_T24 = 32
} sbl_format;

/* Which buffer of a format sbl_packed_row_bytes() describes. */
typedef enum {
    SBL_BUF_MAIN = 0,       /* PK2 / I8 / BF16T data, NM / SP24 values */
    SBL_BUF_NM_BITMAP = 1,  /* NM keep bitmap                          */
    SBL_BUF_SP24_META = 2,  /* SP24 position metadata                  */
    SBL_BUF_T24_HI = 3      /* T24 high plane (SBL_BUF_MAIN: low plane) */
} sbl_buffer;

/* Operations that take a workspace. */
typedef enum {
    SBL_OP_QUANTIZE_MASK_PACK = 0,
    SBL_OP_BACKWARD = 1
} sbl_op;

/* A Sparse-BitLinear layer: W is [out_features, in_features]; the N:M mask
 * keeps n of every m consecutive weights along in_features.
 * Requirements: 1 <= n <= m, m in {4, 8}; in_features >= 16 and a multiple
 * of 16 (and of m); out_features >= 16 and a multiple of 16. */
typedef struct {
    int32_t out_features;
    int32_t in_features;
    int32_t n;
    int32_t m;
} sbl_layer_desc;

/* Device buffers of a packed layer.  Only the members a call uses must be
 * non-null.  `gamma` is a device fp32 scalar written by
 * sbl_quantize_mask_pack and read by the forward and backward. */
typedef struct {
    uint8_t *pk2;       /* SBL_FMT_PK2                                  */
    uint8_t *nm_values; /* SBL_FMT_NM values                            */
    uint8_t *nm_bitmap; /* SBL_FMT_NM keep bitmap                       */
    int8_t *i8;         /* SBL_FMT_I8  [O, K]                           */
    uint16_t *bf16t;    /* SBL_FMT_BF16T [K, O] bf16 bits               */
    float *gamma;       /* device scalar                                */
    int8_t *sp24_values; /* SBL_FMT_SP24 values                         */
    uint8_t *sp24_meta;  /* SBL_FMT_SP24 position metadata              */
    uint8_t *t24_lo;     /* SBL_FMT_T24 low plane                       */
    uint8_t *t24_hi;     /* SBL_FMT_T24 high plane                      */
} sbl_packed;

/* Human-readable text for a status code (static storage). */
const char *sbl_status_string(sbl_status s);

/* Library version: major * 10000 + minor * 100 + patch. */
int32_t sbl_version(void);

/* Bytes per row of one buffer of a packed format (0 for an invalid
 * descriptor).  The buffer holds out_features rows, or in_features rows for
 * SBL_FMT_BF16T. */
size_t sbl_packed_row_bytes(const sbl_layer_desc *desc, sbl_format fmt, sbl_buffer which);

/* Workspace bytes an operation needs for `tokens` tokens (tokens is ignored
 * by SBL_OP_QUANTIZE_MASK_PACK).  0 for an invalid descriptor. */
size_t sbl_workspace_bytes(const sbl_layer_desc *desc, int32_t tokens, sbl_op op);

/* Steps 2-4 of the forward in "The Full Sparse-BitLinear Layer" (the
 * mask from the master weights, their ternary quantization, the mask
 * applied to the ternary weights):
 *   gamma = mean |W| over all O*K master weights (sum in fp64 over a
 *           pairwise tree in flat row-major order, then rounded to fp32);
 *   W_q   = clamp(round_half_even(fl32(W / gamma)), -1, 1)  (0 if gamma==0);
 *   M     = per group of m along K, keep the n largest |W| (lower index
 *           wins ties);
 *   W_eff = W_q * M, written in every format whose bit is set in `formats`.
 * W: [O, K] fp32 device.  out: the buffers of the requested formats plus
 * `gamma` (always written).  workspace: device memory of at least
 * sbl_workspace_bytes(desc, 0, SBL_OP_QUANTIZE_MASK_PACK) bytes, 256-byte
 * aligned; its contents are scratch.  Two launches. */
sbl_status sbl_quantize_mask_pack(const sbl_layer_desc *desc, const float *W,
                                  uint32_t formats, const sbl_packed *out,
                                  void *workspace, size_t workspace_bytes,
                                  void *stream);

/* By-products of the re-mask step, each optional (NULL to skip), computed
 * by the packing kernel from the values it already holds:
 *  keep            this step's keep mask M as a bitmap, bit k%8 of byte k/8 of
 *                  a row of round_up(K/8, 16) bytes ([O, that] uint8; the
 *                  same layout as the SBL_FMT_NM bitmap, padding bits 0);
 *  prev_keep       the previous step's bitmap in that layout (input; needed
 *                  by flips);
 *  flips           device uint64: the number of positions whose keep bit
 *                  differs from prev_keep -- the mask flip count; the flip
 *                  rate r_t of the Sparse-BitNet summary ("Dynamic Mask
 *                  Recomputation at Every Training Step") is flips / (O K);
 *  near_zero       device uint64: #{ w : fl32(|w| / gamma) < 0.5 } (all O K
 *                  when gamma == 0) -- the near-zero mass of "Polarization
 *                  analysis" times O K;
 *  block_threshold fp32 [O, K/m]: per group, the magnitude of the (n+1)-th
 *                  largest |w| (the largest |w| the mask drops; 0 when
 *                  n == m) -- the per-block pruning threshold t of
 *                  "Magnitude stratification".
 * Counters are overwritten (not accumulated).  Alignment: 16 bytes for the
 * arrays, 8 for the counters. */
typedef struct {
    const uint8_t *prev_keep;
    uint8_t *keep;
    unsigned long long *flips;
    unsigned long long *near_zero;
    float *block_threshold;
} sbl_mask_stats;

/* sbl_quantize_mask_pack plus the statistics requested in `stats` (NULL or
 * all-NULL members: exactly sbl_quantize_mask_pack).  flips without
 * prev_keep is SBL_ERR_INVALID_ARG.  formats may be 0 when only statistics
 * are wanted. */
sbl_status sbl_quantize_mask_pack_stats(const sbl_layer_desc *desc, const float *W,
                                        uint32_t formats, const sbl_packed *out,
                                        const sbl_mask_stats *stats, void *workspace,
                                        size_t workspace_bytes, void *stream);

/* Variants of the weight side, the ablation arms of the Sparse-BitNet
 * summary ("Composition Order", "Where the mask is computed"; the method
 * itself is all zeros):
 *  master_dtype  SBL_MASTER_FP32: W is fp32 [O, K]; SBL_MASTER_BF16: W is
 *                bf16 bits [O, K] (the pages' master precision), every step
 *                applied to its exact fp32 value;
 *  mask_source   SBL_MASK_FROM_MASTER ranks |W|; SBL_MASK_FROM_QUANTIZED
 *                ranks |W_q| in {0, 1} (ties, i.e. nearly all, to the
 *                lower index);
 *  order         SBL_QUANT_THEN_MASK: gamma over all O K weights;
 *                SBL_MASK_THEN_QUANT: W_eff = Q_t(W * M), gamma = the mean
 *                |W| over the kept weights only (same fp64 tree with zeros at
 *                dropped positions, divided by O K n / m).
 * SBL_MASK_FROM_QUANTIZED with SBL_MASK_THEN_QUANT is circular (the mask
 * needs gamma, gamma needs the mask): SBL_ERR_UNSUPPORTED. */
typedef enum { SBL_MASTER_FP32 = 0, SBL_MASTER_BF16 = 1 } sbl_master_dtype;
typedef enum { SBL_MASK_FROM_MASTER = 0, SBL_MASK_FROM_QUANTIZED = 1 } sbl_mask_source;
typedef enum { SBL_QUANT_THEN_MASK = 0, SBL_MASK_THEN_QUANT = 1 } sbl_compose_order;
typedef struct {
    int32_t master_dtype; /* sbl_master_dtype  */
    int32_t mask_source;  /* sbl_mask_source   */
    int32_t order;        /* sbl_compose_order */
} sbl_pack_variant;

/* sbl_quantize_mask_pack_stats with a variant (NULL = the method: fp32
 * master weights, mask from |W|, quant-then-mask).  W points to fp32 or bf16
 * data as the variant says. */
sbl_status sbl_quantize_mask_pack_ex(const sbl_layer_desc *desc, const void *W,
                                     const sbl_pack_variant *variant, uint32_t formats,
                                     const sbl_packed *out, const sbl_mask_stats *stats,
                                     void *workspace, size_t workspace_bytes, void *stream);

/* Same result as sbl_quantize_mask_pack, but the caller passes no workspace
 * and the library allocates nothing.  The paper has no counterpart; this
 * entry point exists for callers that cannot obtain device memory at the
 * call site: a plugin hosted by a framework that owns every device
 * allocation and exposes no allocator to it, a runtime that partitions a
 * fixed memory budget up front, or a latency-critical path that must not
 * risk the implicit device synchronisation cudaMalloc/cudaFree may perform.
 *
 * Scratch: one file-scope static device array of SBL_NOALLOC_SCRATCH_BYTES
 * (262400 bytes) per device that loads the library, held until the process
 * exits.  The first call on a device looks up that array's device address
 * (cudaGetSymbolAddress) with the device current; make that first call
 * before any stream capture.  Every call on a device shares the array and
 * the library resets the part that must start at zero on each call, so
 * calls whose kernels overlap on the GPU (different streams, no ordering)
 * race and may produce wrong results; order them on one stream.
 * Limit: O * K <= 2^28 weights (the array holds 32768 fp64 partial sums of
 * 8192 weights each), the same maximum as every entry point; larger layers
 * return SBL_ERR_SHAPE.  Other arguments, formats and errors as for
 * sbl_quantize_mask_pack. */
#define SBL_NOALLOC_SCRATCH_BYTES 262400
sbl_status sbl_quantize_mask_pack_noalloc(const sbl_layer_desc *desc, const float *W,
                                          uint32_t formats, const sbl_packed *out,
                                          void *stream);

/* ------------------------------------------- column-parallel sharding --
 * A layer split by rows (out_features) over ranks: every rank holds rows
 * [first_row, first_row + rows) of W, N:M groups stay inside a row, and only
 * gamma needs the whole matrix.  gamma's fp64 pairwise tree (flat row-major
 * order) has as its first level the sums of consecutive 8192-weight blocks;
 * when every shard starts at a multiple of 8192 weights (first_row * K %
 * 8192 == 0), each shard's blocks are blocks of the whole matrix, so
 *   1. sbl_gamma_partials on every rank (its blocks' sums, fp64),
 *   2. gather them in rank (= row) order (any collective; NCCL all-gather),
 *   3. sbl_gamma_combine on the gathered sums (the rest of the same tree),
 *   4. sbl_quantize_mask_pack_shard on every rank with that gamma
 * give every rank bit for bit the gamma and the packed rows of the unsharded
 * sbl_quantize_mask_pack.  The pages describe no distributed execution; this
 * is the library's own split of the same definitions. */

/* Number of first-level sums of a shard: ceil(rows * K / 8192). */
size_t sbl_gamma_node_count(const sbl_layer_desc *shard);

/* The shard's first-level sums: node_sums[j] = the fp64 tree sum of |W| over
 * the shard's flat weights [8192 j, min(8192 (j + 1), rows K)).
 * shard: (rows, K, n, m) as a layer descriptor; W: the shard's fp32 rows
 * [rows, K]; first_row: the shard's first row in the whole matrix, used only
 * to check the alignment (SBL_ERR_SHAPE unless first_row * K is a multiple of
 * 8192); node_sums: sbl_gamma_node_count(shard) doubles (device);
 * workspace: as for sbl_quantize_mask_pack.  Two launches (a memset, the
 * gamma kernel) and a device-to-device copy. */
sbl_status sbl_gamma_partials(const sbl_layer_desc *shard, const float *W, int64_t first_row, double *node_sums,
                              void *workspace, size_t workspace_bytes, void *stream);

/* gamma = fl32(S / total_weights), S = the pairwise tree over the gathered
 * first-level sums of the whole matrix (nodes = ceil(total_weights / 8192),
 * else SBL_ERR_SHAPE; total_weights <= 2^28).  node_sums and gamma: device.
 * One launch of one CTA. */
sbl_status sbl_gamma_combine(const double *node_sums, int64_t nodes, int64_t total_weights, float *gamma,
                             void *stream);

/* sbl_quantize_mask_pack of a shard's rows with the given gamma: out->gamma
 * is an INPUT here (from sbl_gamma_combine); no workspace.  One launch (plus
 * the BF16T transpose when asked for). */
sbl_status sbl_quantize_mask_pack_shard(const sbl_layer_desc *shard, const float *W, uint32_t formats,
                                        const sbl_packed *out, void *stream);

/* Step 1 of the forward, per-token absmax int8 quantisation (BitNet b1.58
 * 2B4T summary, "Activation Quantization: Per-Token Absmax"; Sparse-BitNet
 * summary, activation quantization equation):
 *   a_t = max_k |x[t,k]|;  a_t == 0 -> q[t,:] = 0, d[t] = 0;  otherwise
 *   q[t,k] = clamp(round_half_even(fl32(x[t,k] * fl32(127 / a_t))), -128, 127)
 *   d[t]   = fl32(a_t / 127).
 * X: [T, K] bf16 bits; Xq: [T, K] int8; d: [T] fp32.  K as for a layer
 * (multiple of 16); T >= 0 (T == 0 enqueues nothing).  One launch. */
sbl_status sbl_quantize_act(const uint16_t *X, int32_t T, int32_t K,
                            int8_t *Xq, float *d, void *stream);

/* RMSNorm fused with the activation quantiser (forward step 1 of the
 * Sparse-BitNet summary, x~ = Q_a(Norm(x)), Norm read as RMSNorm): per
 * token, S = the sum of x_k^2 in fp64 over the pairwise tree of the row
 * (flat order, as for gamma), r = fl32(1 / sqrt(S / K + eps)) computed in
 * fp64, u_k = fl32(fl32(x_k * r) * g_k) with g the bf16 gains [K] (NULL: 1),
 * then exactly the quantiser of sbl_quantize_act applied to the fp32 u (no
 * bf16 rounding in between).  eps: finite, >= 0 (a zero row needs eps > 0).
 * Shapes, outputs and errors as sbl_quantize_act.  One launch. */
sbl_status sbl_quantize_act_rmsnorm(const uint16_t *X, int32_t T, int32_t K, const uint16_t *g,
                                    float eps, int8_t *Xq, float *d, void *stream);

/* Step 5 of the forward: acc[t,o] = sum_k W_eff[o,k] * Xq[t,k] (int32), and
 *   Y[t,o] = fl32(fl32(acc) * fl32(gamma * d[t]))  (bf16 by RNE, or fp32).
 * fmt selects the weight operand: SBL_FMT_I8 runs the tcgen05 int8 tensor
 * core GEMM (any T); SBL_FMT_PK2 runs the decode kernel that streams the
 * 2-bit codes (T <= 16, K a multiple of 64); SBL_FMT_T24 the same kernel
 * streaming the 6-bit group codes (same limits; n <= 2, m = 4 or 8).  Y: [T, O] bf16 bits
 * (y_is_fp32 = 0) or fp32.  acc_out: optional [T, O] int32 copy of the
 * accumulators (NULL to skip).  One launch.
 * The SBL_FMT_PK2 kernel is launched with programmatic dependent launch: it
 * starts loading w->pk2 before it waits for the previous kernel on the
 * stream, so w->pk2 must not be written by a preceding kernel that triggers
 * its dependents early (sbl_quantize_mask_pack never does).  Xq, d, gamma
 * and Y are only touched after that wait.  It also lets the next kernel on
 * the stream launch as soon as it starts: a kernel launched after it with
 * programmatic stream serialization must wait for its grid dependencies
 * (griddepcontrol.wait) before it reads Y or acc_out; kernels launched
 * without that attribute see the usual stream order. */
sbl_status sbl_forward(const sbl_layer_desc *desc, const int8_t *Xq, const float *d,
                       int32_t T, const sbl_packed *w, sbl_format fmt,
                       void *Y, int32_t y_is_fp32, int32_t *acc_out, void *stream);

#define SBL_GROUP_MAX 4

/* Step 5 of the forward for `count` layers (1 <= count <= SBL_GROUP_MAX)
 * that read the same activations (for example the gate and up projections of
 * an MLP, or q, k and v): Y_i = the sbl_forward output of layer i with
 * SBL_FMT_I8, bit for bit, computed by ONE launch whose tiles cover every
 * layer's outputs (the launch's fixed cost is paid once, and the tile rounds
 * are filled across layers).
 * descs[i], w[i], Y[i]: layer i's descriptor, packed weights (w[i]->i8 and
 * w[i]->gamma required) and output [T, out_features_i] (bf16 bits, or fp32
 * when y_is_fp32); every layer has the same in_features K.  Xq [T, K], d [T]
 * as for sbl_forward.  The arrays are host arrays read during the call; the
 * buffers they point to are device memory owned by the caller.
 * Errors: SBL_ERR_INVALID_ARG for a NULL array, entry or buffer or count out
 * of range; SBL_ERR_SHAPE for a bad descriptor, T < 0 or differing
 * in_features; SBL_ERR_ALIGNMENT for a buffer not 16-byte aligned.  T == 0
 * enqueues nothing.  Launched like the SBL_FMT_I8 forward (programmatic
 * dependent launch). */
sbl_status sbl_forward_group(const sbl_layer_desc *const *descs, int32_t count, const int8_t *Xq,
                             const float *d, int32_t T, const sbl_packed *const *w, void *const *Y,
                             int32_t y_is_fp32, void *stream);

/* Output epilogue fused into the forward (all members optional):
 *  relu2     non-zero: v = max(v, 0)^2 on the fp32 output (Squared ReLU of the
 *            BitNet b1.58 2B4T summary, "Squared ReLU Activation in the
 *            Feed-Forward Network"), v = v > 0 ? fl32(v * v) : +0;
 *  residual  bf16 bits [T, O] (16-byte aligned): v = fl32(v + residual),
 *            applied after relu2;
 * then the bf16 (RNE) or fp32 store as in sbl_forward.  acc_out, when given,
 * still receives the raw int32 accumulators. */
typedef struct {
    int32_t relu2;
    const uint16_t *residual;
} sbl_epilogue;

/* sbl_forward with an output epilogue (NULL: exactly sbl_forward).  Every
 * forward format supports it. */
sbl_status sbl_forward_ex(const sbl_layer_desc *desc, const int8_t *Xq, const float *d,
                          int32_t T, const sbl_packed *w, sbl_format fmt, void *Y,
                          int32_t y_is_fp32, int32_t *acc_out, const sbl_epilogue *epi,
                          void *stream);

/* A layer's forward from its bf16 input: Xq, d = Q_a(X) exactly as
 * sbl_quantize_act, then Y exactly as sbl_forward_ex (forward steps 1-5 of
 * the Sparse-BitNet summary, "The Full Sparse-BitLinear Layer").  X: bf16
 * [T, K]; Xq int8 [T, K] and d fp32 [T] are outputs (the backward reuses
 * them); Y and epi as sbl_forward_ex (no accumulator output).  For
 * SBL_FMT_PK2 with T <= 16, K % 64 == 0 and T K <= 4096 this is ONE launch
 * (every CTA of the decode kernel quantises the small X in its prologue);
 * otherwise the activation kernel and the forward kernel, two launches.
 * Shapes, formats and errors as the two calls. */
sbl_status sbl_linear_forward(const sbl_layer_desc *desc, const uint16_t *X, int32_t T, const sbl_packed *w,
                              sbl_format fmt, int8_t *Xq, float *d, void *Y, int32_t y_is_fp32,
                              const sbl_epilogue *epi, void *stream);

/* One layer of a batched decode forward (sbl_forward_batch).  The layer's
 * forward steps 4-5 ("The Full Sparse-BitLinear Layer" of the Sparse-BitNet
 * summary) from its 2-bit PK2 weights, exactly as sbl_forward with
 * SBL_FMT_PK2:
 *   Y[t,o] = fl32(fl32(sum_k W_eff[o,k] Xq[t,k]) * fl32(gamma * d[t])).
 * desc       the layer (in_features a multiple of 64, at most 13824);
 * pk2, gamma its packed weights (sbl_packed.pk2 and .gamma);
 * xq, d      its int8 activations [T, K] and token scales [T] (inputs), or,
 *            when input_is_previous_output is nonzero, unused: the input is
 *            then the bf16 output Y of the batch's previous layer, quantised
 *            per token exactly as sbl_quantize_act (that layer must have
 *            out_features == this layer's in_features and y_is_fp32 == 0);
 * xq_out, d_out  with input_is_previous_output: where to store that
 *            quantised input and its scales (optional, NULL to skip);
 * y          [T, O] bf16 bits (y_is_fp32 == 0) or fp32. */
typedef struct {
    sbl_layer_desc desc;
    const uint8_t *pk2;
    const float *gamma;
    const int8_t *xq;
    const float *d;
    void *y;
    int32_t y_is_fp32;
    int32_t input_is_previous_output;
    int8_t *xq_out;
    float *d_out;
} sbl_batch_layer;

#define SBL_BATCH_MAX_LAYERS 256

/* Workspace bytes of sbl_forward_batch for these `count` layers at T tokens:
 * 128 per layer when some layer takes its input from the previous one, plus,
 * per distinct unchained input (the same xq pointer and in_features), T K
 * bytes rounded up to 256 and 256 more (the input as the MMA loop reads it:
 * every 16-byte group 4 x 4 transposed, and its per-token sums).  0 for
 * invalid arguments. */
size_t sbl_forward_batch_workspace_bytes(const sbl_batch_layer *layers, int32_t count, int32_t T);

/* The decode forward of `count` layers (1 <= count <= SBL_BATCH_MAX_LAYERS)
 * at T tokens (1 <= T <= 16) in ONE persistent launch: one CTA per SM
 * streams every layer's packed rows through a shared-memory ring by bulk
 * copies, ahead of the arithmetic and across layer boundaries, and computes
 * each layer as sbl_forward does (bit-identical results).  Independent
 * layers (no input_is_previous_output) run back to back with no
 * synchronisation between them.  A chained layer waits, inside the kernel,
 * until every output of the layer before it is written (a completion count
 * in the workspace; the wait is bounded and records SBL_DEVICE_ERROR bits on
 * expiry), then quantises that output in-kernel; chained batches are launched
 * cooperatively (every CTA resident) and do not let the next kernel start
 * early.  Each distinct unchained input is first rearranged once into the
 * workspace by a small kernel (its groups transposed, its token sums).
 * workspace: sbl_forward_batch_workspace_bytes bytes, 256-byte aligned; the
 * library zeroes the completion words (one memset) before the launch.
 * Unchained batches are launched with programmatic dependent launch like
 * sbl_forward (the weights are read before the wait on the previous kernel).
 * Two launches (one when every layer after the first is chained).
 * Errors: SBL_ERR_SHAPE for count, T or a descriptor out of range;
 * SBL_ERR_UNSUPPORTED for in_features not a multiple of 64 or above 13824;
 * SBL_ERR_INVALID_ARG for a null pointer a layer needs, a chained first
 * layer, or a chain whose shapes or output type do not match. */
sbl_status sbl_forward_batch(const sbl_batch_layer *layers, int32_t count, int32_t T, void *workspace,
                             size_t workspace_bytes, void *stream);

/* The forward operand format the library recommends for a layer and a
 * token count: SBL_FMT_SP24 (2:4 sparse tensor-core MMA on CTA pairs) when
 * the mask allows it (n <= 2) and the GEMM is large enough for the sparse
 * MMA to pay: in_features >= 1024 and tokens * out_features >= 8192 * 1024;
 * SBL_FMT_I8 (dense tensor-core MMA) otherwise.  On B200 the sparse kernel
 * measured 1.1-1.4x the dense one on such shapes and 0.8x on shorter ones
 * (short K or few output tiles), where the dense kernel's wider tiles and
 * cheaper epilogue win.  Either format gives identical results.  Returns
 * 0 for an invalid descriptor or tokens < 0. */
sbl_format sbl_forward_format(const sbl_layer_desc *desc, int32_t tokens);

/* Backward through the layer with the Dual straight-through estimator
 * (Sparse-BitNet summary, "The Dual Straight-Through Estimator": the
 * gradient passes through mask and quantiser as identity):
 *   dX[t,k] = gamma * sum_o dY[t,o] * W_eff[o,k]        (bf16 or fp32 out)
 *   dW[o,k] = sum_t dY[t,o] * d[t] * Xq[t,k]           (fp32, unmasked)
 * dY: [T, O] bf16 bits; Xq, d: the forward's quantised activations; w must
 * hold SBL_FMT_BF16T and gamma.  dX may be NULL (skips dX), dW may be NULL
 * (skips dW).  Arithmetic: tensor cores with fp32 accumulation; dY and W_eff
 * enter dX as bf16 (exact).  For dW, one power of two 2^s per call is chosen
 * from M = max |fl32(dY[t,o] * d[t])| so that M 2^s lies in [2^14, 2^15);
 * fl32(dY * d[t]) 2^s enters the MMA rounded to fp16 (relative error at most
 * 2^-11 per product), Xq as fp16 (exact), and the fp32 result is multiplied
 * by 2^-s (exact).  Any finite dY works, whatever its magnitude: only
 * products below 2^-29 M (fp16 subnormals) lose precision, and those below
 * 2^-40 M (or below 2^-126 in fp32) count as zero; s is clamped to
 * [-126, 126].  Five launches with dW (an absmax reduction over dY, two
 * transposes, the GEMM; the memset of the prescale word), one for dX.
 * workspace: at least sbl_workspace_bytes(desc, T, SBL_OP_BACKWARD) bytes,
 * 256-byte aligned. */
sbl_status sbl_backward_dual_ste(const sbl_layer_desc *desc, const uint16_t *dY,
                                 const int8_t *Xq, const float *d, int32_t T,
                                 const sbl_packed *w, void *dX, int32_t dx_is_fp32,
                                 float *dW, void *workspace, size_t workspace_bytes,
                                 void *stream);

/* sbl_backward_dual_ste with the mask-gated dW of the pages' ablation
 * ("Gradient flow through masked weights": gradients blocked at pruned
 * weights): dW[o, k] = 0 where bit k%8 of byte k/8 of row o of dw_keep is 0
 * (the keep bitmap of sbl_mask_stats or the SBL_FMT_NM bitmap, rows of
 * round_up(K/8, 16) bytes); dw_keep == NULL gives the method's ungated dW.
 * dX is never gated (identity through the mask either way). */
sbl_status sbl_backward_dual_ste_ex(const sbl_layer_desc *desc, const uint16_t *dY,
                                    const int8_t *Xq, const float *d, int32_t T,
                                    const sbl_packed *w, void *dX, int32_t dx_is_fp32,
                                    float *dW, const uint8_t *dw_keep, void *workspace,
                                    size_t workspace_bytes, void *stream);

/* Device error word of the current device: 0 when every kernel's bounded
 * waits completed; otherwise a bit per kernel family that gave up a wait.
 * Synchronises the device.  `clear` != 0 resets it to 0 afterwards. */
sbl_status sbl_device_error(uint32_t *code, int32_t clear);

/* Bit of the device error word set only by sbl_selftest_wait_expiry. */
#define SBL_DEVICE_ERROR_SELFTEST 0x80000000u

/* Self-test of failure detection: one launch of one CTA whose single thread
 * waits on a shared-memory mbarrier that nothing arrives at, through the
 * bounded wait every kernel of the library uses.  After the wait limit
 * (1 s) the wait gives up, sets SBL_DEVICE_ERROR_SELFTEST in the device
 * error word and the kernel returns, leaving the context usable.  Enqueued
 * on `stream`; read the result with sbl_device_error.  SBL_ERR_DEVICE
 * without an sm_100 device. */
sbl_status sbl_selftest_wait_expiry(void *stream);

/* ------------------------------------------------ packed-layer container --
 * A self-describing byte image of a packed layer, so that packed weights
 * (for decode: PK2 or T24 and gamma) can be stored and reloaded without
 * the master weights.  Host code only: these calls never touch a device.
 * The caller copies the device buffers to host memory before
 * sbl_container_write, and back to the device after sbl_container_read.
 *
 * Layout (integers little-endian):
 *   bytes  0-3   magic "SBLP"
 *          4-7   container version (SBL_CONTAINER_VERSION)
 *          8-23  out_features, in_features, n, m (int32 each)
 *         24-27  format mask (SBL_FMT_* bits)
 *         28-31  gamma (fp32 bits)
 *         32-39  payload bytes (everything after the 64-byte header)
 *         40-47  64-bit FNV-1a hash of every byte of the image except
 *                these eight (header and payload)
 *         48-51  sbl_version() of the writer
 *         52-63  zero (a reader refuses anything else)
 *   payload: for each format present, in the order PK2, NM values, NM
 *   bitmap, I8, BF16T, SP24 values, SP24 metadata, T24 low plane, T24 high
 *   plane, the buffer exactly as sbl_quantize_mask_pack writes it (rows x
 *   sbl_packed_row_bytes; K rows for BF16T), each starting at a multiple of
 *   64 bytes from the start of the image (zero bytes between; with rows a
 *   multiple of 16 and row bytes a multiple of 16, every buffer is a
 *   multiple of 256 bytes, so in practice none are needed).
 * The hash covers the header (gamma included) and every payload byte, so
 * any change to a stored value is detected on reading. */
#define SBL_CONTAINER_VERSION 1
#define SBL_CONTAINER_HEADER_BYTES 64

/* Host buffers of a packed layer, one per stored buffer (the layouts of
 * sbl_packed).  Only the members of the formats in use must be non-null;
 * they need no alignment. */
typedef struct {
    void *pk2;
    void *nm_values;
    void *nm_bitmap;
    void *i8;
    void *bf16t;
    void *sp24_values;
    void *sp24_meta;
    void *t24_lo;
    void *t24_hi;
} sbl_host_buffers;

/* Size of the image for a descriptor and format mask; 0 when the
 * descriptor or the mask is invalid (unknown bits; SBL_FMT_SP24 or
 * SBL_FMT_T24 with n > 2). */
size_t sbl_container_bytes(const sbl_layer_desc *desc, uint32_t formats);

/* Write the image of (desc, formats, gamma, src) into dst[0 .. dst_bytes).
 * SBL_ERR_INVALID_ARG: null desc/src/dst, a null buffer of a present format,
 * unknown format bits or a non-finite gamma; SBL_ERR_SHAPE: invalid
 * descriptor, or dst_bytes below sbl_container_bytes; SBL_ERR_UNSUPPORTED:
 * SP24 or T24 with n > 2. */
sbl_status sbl_container_write(const sbl_layer_desc *desc, uint32_t formats, float gamma,
                               const sbl_host_buffers *src, void *dst, size_t dst_bytes);

/* Check an image and report what it holds.  Any of desc, formats, gamma
 * may be NULL.  SBL_ERR_INVALID_ARG: null src, shorter than its header or
 * its payload, wrong magic, a payload size that does not match the
 * descriptor and formats, nonzero reserved bytes, or a hash mismatch;
 * SBL_ERR_UNSUPPORTED: a
 * container version this library does not read; SBL_ERR_SHAPE: an invalid
 * descriptor. */
sbl_status sbl_container_info(const void *src, size_t src_bytes, sbl_layer_desc *desc, uint32_t *formats,
                              float *gamma);

/* Check an image as sbl_container_info does, then copy every stored buffer
 * into dst (each member of a stored format must be non-null and hold the
 * buffer's rows x row bytes).  Nothing is written unless the image checks. */
sbl_status sbl_container_read(const void *src, size_t src_bytes, const sbl_host_buffers *dst);

#ifdef __cplusplus
}
#endif

#endif /* SBL_H */
