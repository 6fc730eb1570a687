// sbl_gemv.cuh -- persistent, streaming decode GEMV over a batch of packed
// Sparse-BitLinear layers (T <= 16 tokens), one launch for the whole batch.
//
// The arithmetic is the decode kernel's (sbl_decode.cuh): 2-bit PK2 codes
// c = w + 1 as the u8 operand of mma.sync m16n8k32 against the int8
// activations, the activation column sum subtracted to remove the +1 bias,
// y = fl32(fl32(acc) * fl32(gamma * d_t)) (forward steps 4-5 of "The Full
// Sparse-BitLinear Layer" of the Sparse-BitNet summary; the 2-bit storage of
// the BitNet b1.58 2B4T summary, "Inference Implementation: GPU").  What
// differs is how the weights reach the SMs:
//
//  * one CTA per SM runs for the whole batch; its work items are blocks of
//    64, 32 or 16 rows of a layer (as many 16-row tiles as one 54 KB stage
//    holds at that K), taken round-robin over the grid in batch order;
//  * a producer warp streams each item's packed rows -- contiguous, since a
//    PK2 row is exactly K / 4 bytes when K % 64 == 0 -- with ONE bulk copy
//    (cp.async.bulk, evict-first in L2) into a ring of four shared-memory stages,
//    as far ahead as the ring allows and across layer boundaries: the
//    weights never depend on the activations, so no launch gap or
//    dependency stalls the stream;
//  * sixteen consumer warps share an item: each owns one of its tiles and
//    takes that tile's 128-weight K slices round-robin with the other warps
//    of the tile (balanced for any K), frees the stage, and adds its exact
//    int32 partials into the item's sums in shared memory (shared atomics),
//    where the item's T x rows outputs are read, dequantised and stored;
//  * an unchained layer reads its int8 activations in a prepared layout
//    (every 16-byte group 4 x 4 transposed, written once per launch by a
//    small kernel together with the per-token sums that remove the +1 code
//    bias), so the inner loop is loads, masks and MMAs only;
//  * the 2-bit codes enter the MMA masked in place (one op per four weights)
//    rather than shifted down: code position j of every byte keeps its
//    factor 4^j, which a separate accumulator per j carries and an exact
//    shift removes at the end (four independent MMA chains per tile).
//
// Chained layers: a layer marked chained takes as input the bf16 output of
// the layer before it in the batch, quantised in-kernel exactly as the
// activation kernel does it (a_t = max |y|, q = sat8(rint(fl32(y fl32(127 /
// a_t)))), d_t = fl32(a_t / 127)).  The layer before it publishes, per token,
// max |y| of its bf16 outputs (an atomicMax on the bits) and, per item, a
// completion count; consumers of a chained layer wait (bounded) until every
// item of its input layer is counted, then read that output from L2.  The
// weight stream does not wait: the next layers' rows are already in shared
// memory when the dependency clears.
#pragma once

#include "sbl_decode.cuh"

namespace sbl {

constexpr int kGvMaxProblems = 256;
constexpr int kGvWarps = 16;                      // consumer warps
constexpr int kGvThreads = 32 * (kGvWarps + 1);   // + the producer warp
constexpr int kGvStageBytes = 54 * 1024;          // one item: 1, 2 or 4 tiles of 16 rows x K/4 bytes (2 at K = 6912)
constexpr int kGvStages = 4;
constexpr int kGvSlice = 128;                     // weights of a row in one K slice of a unit
constexpr int kGvItemMaxRows = 64;
constexpr int kGvPartStride = kGvItemMaxRows + 4;  // a token's row of item sums (padded: conflict-free adds)
constexpr int kGvSyncWords = 32;                  // per layer: [0] items done, [1 + t] max |y_t| bits
constexpr int kGvSmemBytes = kGvStages * kGvStageBytes + 2 * kDecMaxTokens * kGvPartStride * 4 +
                             2 * kGvWarps * kDecMaxTokens * 4 + 2 * kGvStages * 8;
static_assert(kGvSmemBytes + 256 <= 227 * 1024, "the ring, the sums and the barriers fit one SM's shared memory");

enum : int32_t {
    kGvOutFp32 = 1,   // Y is fp32 (else bf16)
    kGvChained = 2,   // the input is the previous layer's bf16 output
    kGvPublish = 4,   // the next layer is chained on this one: publish max |y| and item counts
    kGvTilesShift = 8,  // bits 8-10: log2 of the 16-row tiles per item (0, 1 or 2)
};

struct GvProblem {
    const uint8_t *pk2;  // PK2 codes [O, K / 4]
    const float *gamma;  // device scalar
    const int8_t *xt;    // unchained: the int8 activations [T, K], each 16-byte group 4 x 4 transposed
    const int32_t *colsum;  // unchained: sum_k Xq[t, k] per token [T]
    const float *d;      // [T] token scales (unchained layers)
    void *y;             // [T, O] bf16 bits or fp32
    int8_t *xq_out;      // chained: Q_a of the input, stored by the CTA of item 0 (optional)
    float *d_out;        // chained: its token scales (optional)
    int32_t O, K;
    int32_t item0;       // index of the layer's first item in the batch
    int32_t flags;
};

struct GvArgs {
    int32_t count, T, items, early_trigger;
    uint32_t *sync;  // [count][kGvSyncWords], zero before the launch (chained batches only)
    uint32_t *err;
    GvProblem p[kGvMaxProblems];
};

__device__ __forceinline__ void gv_consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kGvWarps * 32) : "memory"); }

__device__ __forceinline__ uint4 ld_global_cg16(const void *p)
{
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Lane (g, tg)'s 32 activations of token t at positions pos .. pos + 31 of a
// chained layer as two 16-byte int8 groups: the previous layer's bf16
// outputs, quantised with r = fl32(127 / a_t) (a_t == 0: zeros).
__device__ __forceinline__ void gv_load_x_chained(const GvProblem &prev, int K, int t, int pos, float r,
                                                  uint4 (&x)[2])
{
    const uint16_t *src = static_cast<const uint16_t *>(prev.y) + static_cast<int64_t>(t) * K + pos;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const uint4 a = ld_global_cg16(src + 16 * q), b = ld_global_cg16(src + 16 * q + 8);
        if (r == 0.0f) {
            x[q] = make_uint4(0u, 0u, 0u, 0u);
        } else {
            x[q].x = quant4(bf16_lo(a.x), bf16_hi(a.x), bf16_lo(a.y), bf16_hi(a.y), r);
            x[q].y = quant4(bf16_lo(a.z), bf16_hi(a.z), bf16_lo(a.w), bf16_hi(a.w), r);
            x[q].z = quant4(bf16_lo(b.x), bf16_hi(b.x), bf16_lo(b.y), bf16_hi(b.y), r);
            x[q].w = quant4(bf16_lo(b.z), bf16_hi(b.z), bf16_lo(b.w), bf16_hi(b.w), r);
        }
    }
}

// One K slice of one tile: four MMAs.  The lane's 8 weight bytes of a row are
// words 0 and 1, word wi holding positions pos + 16 wi .. + 15 with byte e
// the four positions pos + 16 wi + 4 e + j at bits 2 j.  Masking code position
// j in place (one op) leaves byte e = c(pos + 16 wi + 4 e + j) 4^j, which
// pairs with word j of the transposed activation group wi (byte e =
// x(pos + 16 wi + 4 e + j)); the 4^j stays in that j's accumulator.
template <int NT>
__device__ __forceinline__ void gv_mma_slice(int32_t (&acc)[4][NT][4], uint2 wa, uint2 wb,
                                             const uint4 (&xt)[NT][2])
{
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t mj = 0x03030303u << (2 * j);
        const uint32_t a0 = wa.x & mj, a1 = wb.x & mj, a2 = wa.y & mj, a3 = wb.y & mj;
#pragma unroll
        for (int b = 0; b < NT; ++b)
            mma_u8s8(acc[j][b], a0, a1, a2, a3, word_of(xt[b][0], j), word_of(xt[b][1], j));
    }
}

__device__ __forceinline__ uint2 ld_shared8(uint32_t addr)
{
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

// The activations of the unchained layers in the layout the MMA loop reads:
// one CTA per (distinct input, token) writes the token's row with every
// 16-byte group 4 x 4 transposed (word j = bytes j, 4 + j, 8 + j, 12 + j) and
// the row's sum.  Done once per input and launch instead of once per item.
struct GvPrepInput {
    const int8_t *xq;  // [T, K]
    int8_t *xt;        // [T, K]
    int32_t *colsum;   // [T]
    int32_t K;
};

struct GvPrepArgs {
    int32_t inputs, T;
    GvPrepInput in[kGvMaxProblems];
};

__global__ void __launch_bounds__(256) gemv_prep_kernel(const __grid_constant__ GvPrepArgs a)
{
    __shared__ int32_t red[8];
    const GvPrepInput &I = a.in[blockIdx.x / a.T];
    const int t = blockIdx.x % a.T;
    pdl_launch_dependents();
    pdl_wait_prior();  // Xq may come from the previous kernel
    const uint4 *src = reinterpret_cast<const uint4 *>(I.xq + static_cast<int64_t>(t) * I.K);
    uint4 *dst = reinterpret_cast<uint4 *>(I.xt + static_cast<int64_t>(t) * I.K);
    int s = 0;
    for (int i = threadIdx.x; i < I.K / 16; i += blockDim.x) {
        const uint4 v = ld_global16(src + i);
        s = __dp4a(static_cast<int>(v.x), 0x01010101, s);
        s = __dp4a(static_cast<int>(v.y), 0x01010101, s);
        s = __dp4a(static_cast<int>(v.z), 0x01010101, s);
        s = __dp4a(static_cast<int>(v.w), 0x01010101, s);
        dst[i] = transpose4x4(v);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        int total = 0;
        for (int w = 0; w < 8; ++w) total += red[w];
        I.colsum[t] = total;
    }
}

// NT: n8 token blocks (T <= 8: 1, T <= 16: 2).
template <int NT>
__global__ void __launch_bounds__(kGvThreads, 1) gemv_stream_kernel(const __grid_constant__ GvArgs args)
{
    extern __shared__ __align__(128) uint8_t gv_smem[];
    int32_t *part = reinterpret_cast<int32_t *>(gv_smem + kGvStages * kGvStageBytes);  // [2][t][row of item]
    int32_t *csum = part + 2 * kDecMaxTokens * kGvPartStride;                             // [2][warp][t]
    uint64_t *bars = reinterpret_cast<uint64_t *>(csum + 2 * kGvWarps * kDecMaxTokens);
    const uint32_t stage0 = smem_addr(gv_smem);
    auto full_bar = [&](int s) { return smem_addr(bars + s); };
    auto empty_bar = [&](int s) { return smem_addr(bars + kGvStages + s); };
    // failure flags by item parity: a flag is written before a consumer
    // barrier of its item and read after it; a faster warp already in the
    // next item writes the other one, so no warp can see a later failure
    // early and leave the others at a barrier
    __shared__ int s_fail[2];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kGvStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), kGvWarps);
        }
        s_fail[0] = s_fail[1] = 0;
        fence_barrier_init();
    }
    // the item sums start at zero; each finishing thread zeroes what it read
    for (int i = threadIdx.x; i < 2 * kDecMaxTokens * kGvPartStride; i += blockDim.x) part[i] = 0;
    __syncthreads();
    // unchained batches have no waits between CTAs: the next kernel may start
    // launching (and streaming its own read-only data) right away
    if (args.early_trigger) pdl_launch_dependents();

    if (warp == kGvWarps) {
        // ------------------------------------------------------ producer
        if (lane != 0) return;
        const uint64_t pol = l2_evict_first_policy();
        int stage = 0, p = 0;
        uint32_t phase = 0;
        uint32_t issued = 0, issued_phase[kGvStages] = {};
        bool ok = true;
        for (int item = blockIdx.x; item < args.items; item += gridDim.x) {
            while (p + 1 < args.count && item >= args.p[p + 1].item0) ++p;
            const GvProblem &P = args.p[p];
            const int item_rows = 16 << ((P.flags >> kGvTilesShift) & 7);
            const int r0 = (item - P.item0) * item_rows;
            const int rows = min(item_rows, P.O - r0);
            const uint32_t bytes = static_cast<uint32_t>(rows) * static_cast<uint32_t>(P.K / 4);
            if (!mbar_wait(empty_bar(stage), phase ^ 1u, args.err, kErrGemv)) {
                ok = false;
                break;
            }
            mbar_arrive_expect_tx(full_bar(stage), bytes);
            bulk_load_1d(stage0 + static_cast<uint32_t>(stage * kGvStageBytes),
                         P.pk2 + static_cast<int64_t>(r0) * (P.K / 4), bytes, full_bar(stage), pol);
            issued |= 1u << stage;
            issued_phase[stage] = phase;
            if (++stage == kGvStages) stage = 0, phase ^= 1u;
        }
        if (!ok) {
            // every copy in flight lands before the CTA may exit
            for (int s = 0; s < kGvStages; ++s)
                if (issued & (1u << s)) mbar_wait(full_bar(s), issued_phase[s], args.err, kErrGemv);
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    const int g = lane >> 2, tg = lane & 3;
    const int T = args.T;
    int stage = 0, p = 0, buf = 0;
    uint32_t phase = 0;
    int ready_p = -1;  // chained layer whose input is known complete
    pdl_wait_prior();  // activations, scales and gamma may come from the previous kernel
    for (int item = blockIdx.x; item < args.items; item += gridDim.x, buf ^= 1) {
        while (p + 1 < args.count && item >= args.p[p + 1].item0) ++p;
        const GvProblem &P = args.p[p];
        const bool chained = (P.flags & kGvChained) != 0;
        const GvProblem &prev = args.p[p > 0 ? p - 1 : 0];
        if (chained && ready_p != p) {
            if (threadIdx.x == 0) {
                const int prev_items = P.item0 - prev.item0;
                if (!wait_counter_geq(args.sync + (p - 1) * kGvSyncWords, static_cast<uint32_t>(prev_items), args.err,
                                      kErrGemv))
                    s_fail[buf] = 1;
            }
            gv_consumer_sync();
            if (s_fail[buf]) break;
            ready_p = p;
        }
        const int tl2 = (P.flags >> kGvTilesShift) & 7;  // log2 of the tiles per item (0, 1, 2)
        const int tiles = 1 << tl2;
        const int item_rows = 16 * tiles;
        const int r0 = (item - P.item0) * item_rows;
        const int rows = min(item_rows, P.O - r0);
        const int K = P.K, kb = K / 4;
        const int slices = (K + kGvSlice - 1) / kGvSlice;
        const int tile = warp & (tiles - 1);           // this warp's tile, fixed for the item
        const bool tile_in = 16 * tile < rows;         // warp-uniform
        const int rA = 16 * tile + g, rB = rA + 8;     // the lane's two rows in the item
        // the tile's warps take its K slices round-robin: slice (warp >> tl2) + i (16 >> tl2)
        const int sl0 = warp >> tl2, sl_step = kGvWarps >> tl2;
        // this lane's tokens 8 b + g: the quantisation factor of a chained input
        float rq[NT];
#pragma unroll
        for (int b = 0; b < NT; ++b) {
            rq[b] = 0.0f;
            const int t = 8 * b + g;
            if (chained && t < T) {
                const float a = __uint_as_float(ld_acquire_u32(args.sync + (p - 1) * kGvSyncWords + 1 + t));
                rq[b] = a > 0.0f ? __fdiv_rn(127.0f, a) : 0.0f;
            }
        }
        // a wait that gives up marks the CTA failed; the warps leave together
        // after the next consumer barrier (a warp leaving alone would strand
        // the others at it)
        if (!__all_sync(0xffffffffu, mbar_wait(full_bar(stage), phase, args.err, kErrGemv)) && lane == 0)
            s_fail[buf] = 1;
        const uint32_t st = stage0 + static_cast<uint32_t>(stage * kGvStageBytes);
        const uint32_t rowA = st + static_cast<uint32_t>(rA * kb), rowB = st + static_cast<uint32_t>(rB * kb);
        const bool inA = rA < rows, inB = rB < rows;
        // acc[j][b]: code position j (weights scaled by 4^j), token block b
        int32_t acc[4][NT][4];
        uint32_t cs[NT];
#pragma unroll
        for (int b = 0; b < NT; ++b) {
            cs[b] = 0u;
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[j][b][0] = acc[j][b][1] = acc[j][b][2] = acc[j][b][3] = 0;
        }
        if (tile_in) {
            const uint2 zero_codes = make_uint2(0x55555555u, 0x55555555u);
            if (!chained) {
                // the prepared activations: two 16-byte loads per slice and token
                // block, no arithmetic.  Lanes of tokens t >= T read token 0's
                // row (the same addresses, one request) and rows past the
                // layer's last read the stage's other bytes: both only reach
                // accumulator entries that are never stored, so the full
                // slices need no selects; the ragged last slice (K % 128 ==
                // 64) zeroes the lanes past K, whose products would land in
                // stored entries.
                const int8_t *xrow[NT];
#pragma unroll
                for (int b = 0; b < NT; ++b) {
                    const int t = 8 * b + g;
                    xrow[b] = P.xt + static_cast<int64_t>(t < T ? t : 0) * K + 32 * tg;
                }
                const int full = K / kGvSlice;
                int sl = sl0;
                for (; sl < full; sl += sl_step) {
                    const int off = sl * kGvSlice;  // this slice's first weight
                    const uint32_t bo = static_cast<uint32_t>(off / 4 + 8 * tg);
                    const uint2 wa = ld_shared8(rowA + bo);
                    const uint2 wb = ld_shared8(rowB + bo);
                    uint4 xt[NT][2];
#pragma unroll
                    for (int b = 0; b < NT; ++b) {
#pragma unroll
                        for (int q = 0; q < 2; ++q) xt[b][q] = ld_global16(xrow[b] + off + 16 * q);
                    }
                    gv_mma_slice<NT>(acc, wa, wb, xt);
                }
                if (sl < slices) {  // warp-uniform: this warp's share holds the ragged slice
                    const int off = sl * kGvSlice;
                    const bool kin = off + 32 * tg < K;
                    const uint32_t bo = static_cast<uint32_t>(off / 4 + 8 * tg);
                    const uint2 wa = kin ? ld_shared8(rowA + bo) : zero_codes;
                    const uint2 wb = kin ? ld_shared8(rowB + bo) : zero_codes;
                    uint4 xt[NT][2];
#pragma unroll
                    for (int b = 0; b < NT; ++b) {
#pragma unroll
                        for (int q = 0; q < 2; ++q)
                            xt[b][q] = kin ? ld_global16(xrow[b] + off + 16 * q) : make_uint4(0u, 0u, 0u, 0u);
                    }
                    gv_mma_slice<NT>(acc, wa, wb, xt);
                }
            } else {
                // the previous layer's bf16 output, quantised here; the warps of
                // tile 0 also sum the codes (the +1 bias) and, in the layer's
                // first item, store the quantised input
                const bool sums = tile == 0;
                const bool store_xq = sums && P.xq_out && item == P.item0;
                for (int sl = sl0; sl < slices; sl += sl_step) {
                    const int pos = sl * kGvSlice + 32 * tg;
                    const bool kin = pos < K;
                    const uint32_t bo = static_cast<uint32_t>(pos / 4);
                    const uint2 wa = (kin && inA) ? ld_shared8(rowA + bo) : zero_codes;
                    const uint2 wb = (kin && inB) ? ld_shared8(rowB + bo) : zero_codes;
                    uint4 xt[NT][2];
#pragma unroll
                    for (int b = 0; b < NT; ++b) {
                        const int t = 8 * b + g;
                        uint4 x[2];
                        if (kin && t < T) {
                            gv_load_x_chained(prev, K, t, pos, rq[b], x);
                            if (store_xq) {
                                uint4 *dst = reinterpret_cast<uint4 *>(P.xq_out + static_cast<int64_t>(t) * K + pos);
                                dst[0] = x[0];
                                dst[1] = x[1];
                            }
                        } else {
                            x[0] = x[1] = make_uint4(0u, 0u, 0u, 0u);
                        }
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            if (sums) {
                                int sum = static_cast<int>(cs[b]);
                                sum = __dp4a(static_cast<int>(x[q].x), 0x01010101, sum);
                                sum = __dp4a(static_cast<int>(x[q].y), 0x01010101, sum);
                                sum = __dp4a(static_cast<int>(x[q].z), 0x01010101, sum);
                                sum = __dp4a(static_cast<int>(x[q].w), 0x01010101, sum);
                                cs[b] = static_cast<uint32_t>(sum);
                            }
                            xt[b][q] = transpose4x4(x[q]);
                        }
                    }
                    gv_mma_slice<NT>(acc, wa, wb, xt);
                }
            }
        }
        // this warp is done with the stage: the producer may refill it
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(stage));
        if (++stage == kGvStages) stage = 0, phase ^= 1u;

        // partials added into the item's sums part[buf][token][row] (shared
        // atomics; integer addition in any order is exact); code sums
        // (chained layers) csum[buf][warp][token]
        int32_t *pb = part + buf * kDecMaxTokens * kGvPartStride + 16 * tile + g;
#pragma unroll
        for (int b = 0; b < NT; ++b) {
            const int tA = 8 * b + 2 * tg;
            // fold the code positions back: acc[j] is a multiple of 4^j
            // (every product is), so the arithmetic shifts are exact
            int32_t v[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                v[e] = acc[0][b][e] + (acc[1][b][e] >> 2) + (acc[2][b][e] >> 4) + (acc[3][b][e] >> 6);
            if (tile_in && tA < T) {
                atomicAdd(pb + tA * kGvPartStride, v[0]);
                atomicAdd(pb + tA * kGvPartStride + 8, v[2]);
            }
            if (tile_in && tA + 1 < T) {
                atomicAdd(pb + (tA + 1) * kGvPartStride, v[1]);
                atomicAdd(pb + (tA + 1) * kGvPartStride + 8, v[3]);
            }
            if (chained) {
                uint32_t s = cs[b];
                s += __shfl_xor_sync(0xffffffffu, s, 1);
                s += __shfl_xor_sync(0xffffffffu, s, 2);
                if (tg == 0) csum[(buf * kGvWarps + warp) * kDecMaxTokens + 8 * b + g] = static_cast<int32_t>(s);
            }
        }
        gv_consumer_sync();
        if (s_fail[buf]) break;

        // thread (t, r): the item's sum (wrapping int32 arithmetic is exact
        // when the result fits), the code sums removed, dequantised, stored;
        // the sum is zeroed for the item after next
        const float gam = ld_global_f32(P.gamma);
        const bool publish = (P.flags & kGvPublish) != 0;
        // the warps with the fewest K slices (the highest-numbered: their first
        // slice index is the largest) take the outputs first
        const int n_out = T * item_rows;
        for (int o0 = (kGvWarps - 1 - warp) * 32; o0 < n_out; o0 += kGvWarps * 32) {  // warp-uniform
            const int o = o0 + lane;
            const bool valid = o < n_out;
            const int t = valid ? o >> (4 + tl2) : 0, r = o - t * item_rows;
            uint32_t absbits = 0u;
            int32_t *ps = part + (buf * kDecMaxTokens + t) * kGvPartStride + r;
            const uint32_t sum = valid ? static_cast<uint32_t>(*ps) : 0u;
            if (valid) *ps = 0;
            if (valid && r < rows) {
                float d_t;
                uint32_t bias = 0u;
                if (chained) {
                    const float a = __uint_as_float(ld_acquire_u32(args.sync + (p - 1) * kGvSyncWords + 1 + t));
                    d_t = a > 0.0f ? __fdiv_rn(a, 127.0f) : 0.0f;
                    for (int w = 0; w < kGvWarps; w += tiles)  // the warps of tile 0
                        bias += static_cast<uint32_t>(csum[(buf * kGvWarps + w) * kDecMaxTokens + t]);
                } else {
                    d_t = ld_global_f32(P.d + t);
                    bias = static_cast<uint32_t>(__ldcg(P.colsum + t));
                }
                const uint32_t s = sum - bias;
                const float y = __fmul_rn(__int2float_rn(static_cast<int32_t>(s)), __fmul_rn(gam, d_t));
                const int64_t off = static_cast<int64_t>(t) * P.O + r0 + r;
                if (P.flags & kGvOutFp32) {
                    static_cast<float *>(P.y)[off] = y;
                } else {
                    const __nv_bfloat16 hb = __float2bfloat16_rn(y);
                    const uint16_t bits = *reinterpret_cast<const uint16_t *>(&hb);
                    static_cast<uint16_t *>(P.y)[off] = bits;
                    absbits = static_cast<uint32_t>(bits & 0x7fffu);
                }
            }
            if (publish) {
                // max |y_t| of the bf16 outputs (their fp32 bits order like the
                // values): the lanes of one token are the whole warp, or each
                // half of it when the item has 16 rows
                uint32_t m = absbits;
#pragma unroll
                for (int off = 1; off < 16; off <<= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
                if (item_rows >= 32) m = max(m, __shfl_xor_sync(0xffffffffu, m, 16));
                if (valid && (lane & (item_rows >= 32 ? 31 : 15)) == 0 && m)
                    atomicMax(args.sync + p * kGvSyncWords + 1 + t, m << 16);
            }
        }
        if (chained && item == P.item0 && P.d_out && threadIdx.x < T) {
            const float a = __uint_as_float(ld_acquire_u32(args.sync + (p - 1) * kGvSyncWords + 1 + threadIdx.x));
            P.d_out[threadIdx.x] = a > 0.0f ? __fdiv_rn(a, 127.0f) : 0.0f;
        }
        if (publish) {
            // every output and maximum of this item is written: count it
            gv_consumer_sync();
            if (threadIdx.x == 0) {
                __threadfence();
                atomicAdd(args.sync + p * kGvSyncWords, 1u);
            }
        }
    }
}

}  // namespace sbl
