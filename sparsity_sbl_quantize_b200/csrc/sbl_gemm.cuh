// sbl_gemm.cuh -- persistent, warp-specialised tcgen05 GEMM for sm_100a.
//
//   D[m, n] = sum_k A[m, k] * B[n, k]        (A, B K-major in global memory)
//
// Forward of the Sparse-BitLinear layer ("The Full Sparse-BitLinear Layer",
// forward step 5 of the Sparse-BitNet summary): A = int8 activations [T, K],
// B = int8 W_eff [O, K], int32 accumulators in tensor memory, then the
// epilogue y = fl32(fl32(acc) * fl32(gamma * d_t)).  The same kernel with
// 16-bit operands and fp32 accumulation runs the two GEMMs of the Dual-STE
// backward.
//
// Tiles are 128 x BN (BN = 256 or 128).  Roles (320 threads): warp 0 issues
// TMA loads into a shared-memory ring (4 stages of 48 KiB or 6 of 32 KiB);
// warp 1 owns the tensor memory (all 512 columns: 2 accumulators of 256
// columns or 4 of 128) and issues the MMAs from one lane; warps 2-9 drain
// the accumulators (tcgen05.ld; two warps per 32-lane quarter, each half of
// the columns), scale them and write the outputs through swizzled
// shared-memory staging and TMA bulk tensor stores, overlapping the next
// tiles' MMAs.  Every wait is time-bounded (see sbl_device.cuh).  The
// kernel is launched with programmatic dependent launch: its prologue
// overlaps the previous kernel, and it waits for that kernel before touching
// global memory.
//
// GEMMs with 256-wide tiles and more than 128 rows run the same roles on CTA
// pairs (cta_group::2, clusters of two): 256 x 256 per pair, each CTA
// loading its 128 A rows and 128 of the B rows, so a stage is 32 KiB and six
// are in flight.  The single-CTA form moves 48 KiB per 128-byte K step and,
// at the TMA latency measured on B200 (about 1.7 us per stage under load),
// four stages keep the int8 tensor core busy only about 65% of the time.
//
// gemm_group_kernel runs up to four int8 products that share A (the linears
// that read one input) in one launch, each with its own B and Y maps, width
// and gamma; its column tiles are the groups' tiles in order.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sbl_device.cuh"

namespace sbl {

enum GemmKind : int { kKindI8 = 0, kKindF16 = 1, kKindBF16 = 2 };

constexpr int kBM = 128;                 // tile rows (A rows, TMEM lanes)
constexpr int kBKBytes = 128;            // K bytes per stage (one 128-byte swizzle row)
constexpr int kABytes = kBM * kBKBytes;  // 16 KiB
constexpr int kTmemCols = 512;           // the whole tensor memory of the SM
constexpr int kEpiWarps = 8;
constexpr int kGemmThreads = 32 * (2 + kEpiWarps);
constexpr int kGroupM = 8;               // tile raster: groups of 8 row tiles
// Epilogue staging: per epilogue warp one 4 KiB buffer (32 rows x 128 bytes,
// 128-byte swizzle) feeding TMA bulk tensor stores.
constexpr int kEpiBufBytes = 32 * 128;
constexpr int kEpiBytes = kEpiWarps * kEpiBufBytes;

// PAIR: CTA pairs (cta_group::2) -- a tile is 256 A rows x BN, each CTA of
// the pair holding its 128 A rows and half of the BN B rows per stage.
template <int BN, bool PAIR = false>
struct GemmCfg {
    static_assert(BN == 128 || BN == 256, "tile width");
    static constexpr int kBRows = PAIR ? BN / 2 : BN;  // B rows per CTA and stage
    static constexpr int kBBytes = kBRows * kBKBytes;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStages = (192 * 1024) / kStageBytes;  // 4 (BN 256), 6 (BN 128 or a pair at 256)
    static constexpr int kNumAcc = kTmemCols / BN;              // 2 or 4 accumulators
    static constexpr int kSmemBytes = 1024 /*align slack*/ + kStages * kStageBytes + kEpiBytes + 256;
};

struct GemmArgs {
    int32_t M, N, K;        // K in elements
    int32_t tiles_m, tiles_n;
    int32_t k_blocks;       // ceil(K bytes / 128)
    void *out;              // [M, ldo] fp32 or bf16
    int64_t ldo;            // elements
    int32_t out_fp32;
    int32_t *acc_out;       // optional raw accumulators [M, ldo] (int32 / fp32 bits)
    const float *gamma;     // device scalar (nullptr: 1)
    const float *row_scale; // per-row d_t (nullptr: none)
    const uint8_t *col_keep;// fp32 output only: keep bitmap [M, keep_stride] (bit n%8 of byte n/8);
    int64_t keep_stride;    // columns whose bit is 0 are written as 0 (nullptr: none)
    int32_t relu2;          // output epilogue: v = max(v, 0)^2 ...
    const uint16_t *residual;  // ... then v = v + residual[m, n] (bf16 [M, ldo]; nullptr: none)
    uint32_t *err;
};

// The optional output epilogue of the forward (Squared ReLU, then a bf16
// residual), in fp32 with round-to-nearest operations.
__device__ __forceinline__ float epilogue_op(float v, int32_t relu2, uint32_t res_bits16, bool has_res)
{
    if (relu2) v = v > 0.0f ? __fmul_rn(v, v) : 0.0f;
    if (has_res) v = __fadd_rn(v, __uint_as_float(res_bits16 << 16));
    return v;
}

template <int KIND, int BN, int M = kBM>
__device__ __forceinline__ constexpr uint32_t gemm_idesc()
{
    // D format (bits 4-5), A/B formats (7-9, 10-12), K-major A and B (bits 15,
    // 16 = 0), N >> 3 (bits 17-22), M >> 4 (bits 24-28).
    uint32_t d = 0;
    if (KIND == kKindI8) d |= (2u << 4) | (1u << 7) | (1u << 10);       // s32 <- s8 x s8
    else if (KIND == kKindF16) d |= (1u << 4);                          // f32 <- f16 x f16
    else d |= (1u << 4) | (1u << 7) | (1u << 10);                       // f32 <- bf16 x bf16
    d |= static_cast<uint32_t>(BN >> 3) << 17;
    d |= static_cast<uint32_t>(M >> 4) << 24;
    return d;
}

__device__ __forceinline__ void tile_coords(int tile, int tiles_m, int tiles_n, int &tm, int &tn)
{
    const int per_group = kGroupM * tiles_n;
    const int group = tile / per_group;
    const int first_m = group * kGroupM;
    const int gm = min(tiles_m - first_m, kGroupM);
    const int r = tile - group * per_group;
    tm = first_m + r % gm;
    tn = r / gm;
}

// D(tmem) (+)= A * B^T over a CTA pair (M = 256: 128 A rows from each CTA's
// shared memory, B split the same way by rows), int8 -> int32 or 16-bit
// floats -> fp32; issued by the even CTA.
__device__ __forceinline__ void mma_i8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_f16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Grouped GEMMs: up to kGemmMaxGroups products that share A (the same
// activations, e.g. the gate and up projections) in one persistent grid.
// Group i's BN-column tiles are the column tiles tn0[i] .. tn0[i + 1] - 1 of
// the launch, with its own B and Y maps, width n[i] and gamma; the raster of
// tile_coords runs over all of them, so every A tile is reused across groups.
constexpr int kGemmMaxGroups = 4;
struct GemmGroups {
    int32_t count;
    int32_t tn0[kGemmMaxGroups + 1];
    int32_t n[kGemmMaxGroups];
    const float *gamma[kGemmMaxGroups];
};

// The group of column tile tn and the tile's index inside it.
__device__ __forceinline__ int group_of(const GemmGroups &grp, int tn, int &tn_local)
{
    int gi = 0;
    while (gi + 1 < grp.count && tn >= grp.tn0[gi + 1]) ++gi;
    tn_local = tn - grp.tn0[gi];
    return gi;
}

// The kernel body.  tmB and tmY point at G maps (kernel parameters); G == 1
// is the single product of `args` (grp unused), G > 1 the groups of grp
// (plain epilogue only: no EPI, raw accumulators or keep bits).
// EPI: the instantiation that applies the output epilogue (relu2 /
// residual); the others compile without it.  PAIR: the CTA-pair form: a
// cluster of two CTAs computes a 256 x BN tile with M = 256 MMAs issued by
// the even CTA; each CTA loads its own 128 A rows and BN / 2 B rows (so a
// stage is 32 KiB instead of 48 and six stages are in flight), the odd CTA's
// loads complete on the even CTA's full barriers, the even CTA's commits
// arrive on the barriers of both, each CTA drains its own 128 rows of the
// accumulator and its epilogue warps arrive on the even CTA's
// accumulator-free barriers.
template <int KIND, int BN, bool EPI, bool PAIR, int G>
__device__ __forceinline__ void gemm_body(const CUtensorMap *tmA, const CUtensorMap *tmB, const CUtensorMap *tmY,
                                          const GemmArgs &args, const GemmGroups &grp)
{
    static_assert(G == 1 || !EPI, "grouped products take the plain epilogue");
    using Cfg = GemmCfg<BN, PAIR>;
    constexpr int kStages = Cfg::kStages;
    constexpr int kNumAcc = Cfg::kNumAcc;
    constexpr int kTileM = PAIR ? 2 * kBM : kBM;  // A rows of a tile
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw);
    const uint32_t a_base = base;
    const uint32_t b_base = base + kStages * kABytes;
    const uint32_t epi_base = base + kStages * Cfg::kStageBytes;  // 1024-byte aligned
    const uint32_t bar_base = epi_base + kEpiBytes;
    // barrier addresses: full[s], empty[s], tfull[a], tempty[a], drain
    auto full_bar = [&](int s) { return bar_base + 8u * s; };
    auto empty_bar = [&](int s) { return bar_base + 8u * (kStages + s); };
    auto tfull_bar = [&](int a) { return bar_base + 8u * (2 * kStages + a); };
    auto tempty_bar = [&](int a) { return bar_base + 8u * (2 * kStages + kNumAcc + a); };
    const uint32_t drain_bar = bar_base + 8u * (2 * kStages + 2 * kNumAcc);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + (bar_base - base) + 224);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_tiles = args.tiles_m * args.tiles_n;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;  // CTA of the pair
    const bool leader = rank == 0;
    // tiles are dealt to CTAs, or to pairs: unit g takes tiles g, g + units, ...
    const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

    // ---------------------------------------------------------- prologue
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < kNumAcc; ++a) {
            mbar_init(tfull_bar(a), 1);
            // single CTA: every epilogue thread arrives; pair: one arrival per
            // epilogue warp of both CTAs, on the even CTA's barrier
            mbar_init(tempty_bar(a), PAIR ? 2 * kEpiWarps : kEpiWarps * 32);
        }
        mbar_init(drain_bar, 1);
        fence_barrier_init();
        tma_prefetch_map(tmA);
        for (int i = 0; i < (G > 1 ? grp.count : 1); ++i) {
            tma_prefetch_map(tmB + i);
            tma_prefetch_map(tmY + i);
        }
    }
    if (warp == 1) {
        if constexpr (PAIR) {
            tmem_alloc_pair(smem_addr(tmem_slot), kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_addr(tmem_slot), kTmemCols);
            tmem_relinquish();
        }
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    // both CTAs' barriers are initialised before either CTA signals the other
    if constexpr (PAIR) cluster_sync_all();
    const uint32_t tmem_base = *tmem_slot;
    // the previous kernel's outputs (our A operand, gamma, scales) are ready
    // after this; our own dependents may start their prologue now
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // Roles run as whole warps: every lane waits on the barriers (warp-uniform
    // outcome through __all_sync), lane 0 issues the TMA / MMA instructions.
    if (warp == 0) {
        // ---------------------------------------------------- TMA producer
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        uint32_t issued_mask = 0;
        uint32_t issued_phase[kStages];
        for (int s = 0; s < kStages; ++s) issued_phase[s] = 0;
        constexpr int kElemsPerBlock = (KIND == kKindI8) ? 128 : 64;
        for (int tile = unit; ok && tile < num_tiles; tile += units) {
            int tm, tn;
            tile_coords(tile, args.tiles_m, args.tiles_n, tm, tn);
            int tnl = tn;
            const int gi = G > 1 ? group_of(grp, tn, tnl) : 0;
            const CUtensorMap *mapB = tmB + gi;
            const int arow = tm * kTileM + static_cast<int>(rank) * kBM;
            const int brow = tnl * BN + static_cast<int>(rank) * Cfg::kBRows;
            for (int kb = 0; kb < args.k_blocks; ++kb) {
                const bool ready = mbar_wait(empty_bar(stage), phase ^ 1u, args.err, kErrGemmProducer);
                if (!__all_sync(0xffffffffu, ready)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    if constexpr (PAIR) {
                        const uint32_t fb = map_shared_rank(full_bar(stage), 0);  // the even CTA's barrier
                        if (leader) mbar_arrive_expect_tx(full_bar(stage), 2 * Cfg::kStageBytes);
                        tma_load_2d_pair(a_base + stage * kABytes, tmA, kb * kElemsPerBlock, arow, fb);
                        tma_load_2d_pair(b_base + stage * Cfg::kBBytes, mapB, kb * kElemsPerBlock, brow, fb);
                    } else {
                        mbar_arrive_expect_tx(full_bar(stage), Cfg::kStageBytes);
                        tma_load_2d(a_base + stage * kABytes, tmA, kb * kElemsPerBlock, arow, full_bar(stage));
                        tma_load_2d(b_base + stage * Cfg::kBBytes, mapB, kb * kElemsPerBlock, brow,
                                    full_bar(stage));
                    }
                }
                __syncwarp();
                issued_mask |= 1u << stage;
                issued_phase[stage] = phase;
                if (++stage == kStages) stage = 0, phase ^= 1u;
            }
        }
        if (!ok && leader) {
            // let any load still in flight land before the CTA can exit (a
            // pair's loads all complete on the even CTA's barriers; the odd
            // CTA stays alive through the closing cluster barrier)
            for (int s = 0; s < kStages; ++s)
                if (issued_mask & (1u << s)) mbar_wait(full_bar(s), issued_phase[s], args.err, kErrGemmProducer);
        }
    } else if (warp == 1 && leader) {
        // -------------------------------------------------------- MMA issuer
        constexpr uint32_t idesc = gemm_idesc<KIND, BN, kTileM>();
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        int local = 0;
        for (int tile = unit; ok && tile < num_tiles; tile += units, ++local) {
            const int acc = local % kNumAcc;
            const uint32_t acc_phase = (local / kNumAcc) & 1;
            const bool free_acc = mbar_wait(tempty_bar(acc), acc_phase ^ 1u, args.err, kErrGemmMma);
            if (!__all_sync(0xffffffffu, free_acc)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
            for (int kb = 0; kb < args.k_blocks; ++kb) {
                const bool ready = mbar_wait(full_bar(stage), phase, args.err, kErrGemmMma);
                if (!__all_sync(0xffffffffu, ready)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint64_t adesc = smem_desc_k128(a_base + stage * kABytes);
                    const uint64_t bdesc = smem_desc_k128(b_base + stage * Cfg::kBBytes);
#pragma unroll
                    for (int kk = 0; kk < kBKBytes / 32; ++kk) {
                        // +32 bytes along K = +2 in the 16-byte address field
                        const uint64_t step = static_cast<uint64_t>(2 * kk);
                        if constexpr (PAIR) {
                            if constexpr (KIND == kKindI8)
                                mma_i8_pair(d_tmem, adesc + step, bdesc + step, idesc, (kb | kk) != 0);
                            else
                                mma_f16_pair(d_tmem, adesc + step, bdesc + step, idesc, (kb | kk) != 0);
                        } else if (KIND == kKindI8)
                            mma_i8(d_tmem, adesc + step, bdesc + step, idesc, (kb | kk) != 0);
                        else
                            mma_f16(d_tmem, adesc + step, bdesc + step, idesc, (kb | kk) != 0);
                    }
                    // frees the stage (of both CTAs) once these MMAs finish
                    if constexpr (PAIR)
                        tc_commit_pair(empty_bar(stage), 0x3);
                    else
                        tc_commit(empty_bar(stage));
                }
                __syncwarp();
                if (++stage == kStages) stage = 0, phase ^= 1u;
            }
            if (!ok) break;
            if (lane == 0) {  // accumulator ready for the epilogue (of both CTAs)
                if constexpr (PAIR)
                    tc_commit_pair(tfull_bar(acc), 0x3);
                else
                    tc_commit(tfull_bar(acc));
            }
            __syncwarp();
        }
        // every MMA issued above has completed before TMEM is released
        if (lane == 0) {
            if constexpr (PAIR)
                tc_commit_pair(drain_bar, 0x1);
            else
                tc_commit(drain_bar);
        }
        __syncwarp();
        mbar_wait(drain_bar, 0, args.err, kErrGemmMma);
        __syncwarp();
    } else if (warp >= 2) {
        // ---------------------------------------------------- epilogue (warps 2-9)
        // this warp's share of accumulator a is in registers: hand it back
        // (pair: lane 0 for the warp, on the even CTA's barrier)
        auto release_accumulator = [&](int a) {
            if constexpr (PAIR) {
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(map_shared_rank(tempty_bar(a), 0));
            } else {
                mbar_arrive(tempty_bar(a));
            }
        };
        // Lane r of warp w drains TMEM row 32 (w % 4) + r over half of the
        // columns ((w - 2) / 4), scales it, and writes it as 128-byte rows
        // into a swizzled staging buffer that lane 0 stores with one TMA bulk
        // tensor store per 32 x 128-byte block.
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int half = (warp - 2) >> 2;
        const int r = quarter * 32 + lane;
        const float g1 = args.gamma ? *args.gamma : 1.0f;
        const uint32_t buf = epi_base + static_cast<uint32_t>(warp - 2) * kEpiBufBytes;
        constexpr int kColsPerChunk = 64;  // bf16: two 64-byte stores (one 128-byte with the epilogue); fp32: two
        constexpr int kChunks = BN / kColsPerChunk / 2;  // per warp
        uint32_t nstore = 0;  // bf16 blocks stored by this warp (staging half = nstore % 2)
        int local = 0;
        for (int tile = unit; tile < num_tiles; tile += units, ++local) {
            int tm, tn;
            tile_coords(tile, args.tiles_m, args.tiles_n, tm, tn);
            // grouped: this tile's product (its map, width and gamma); tn is
            // from here on the column tile inside it
            const int gi = G > 1 ? group_of(grp, tn, tn) : 0;
            const CUtensorMap *mapY = tmY + gi;
            const int N = G > 1 ? grp.n[gi] : args.N;
            const int acc = local % kNumAcc;
            const uint32_t acc_phase = (local / kNumAcc) & 1;
            const int m = tm * kTileM + static_cast<int>(rank) * kBM + r;
            const bool row_ok = m < args.M;
            const int row0 = m - lane;  // first row of this warp's block
            // the token scale (and a group's gamma) are loaded while the MMAs
            // of this tile still run
            const float d_m = (args.row_scale && row_ok) ? args.row_scale[m] : 0.0f;
            const float g = G > 1 ? *grp.gamma[gi] : g1;
            const bool ready = mbar_wait(tfull_bar(acc), acc_phase, args.err, kErrGemmEpilogue);
            if (!__all_sync(0xffffffffu, ready)) break;  // warp-uniform decision
            tc_fence_after();
            float scale = g;
            if (args.row_scale) scale = row_ok ? __fmul_rn(g, d_m) : 0.0f;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(acc * BN);
            if (!args.out_fp32 && !EPI) {
                // bf16: drain this warp's share of the accumulator, converting
                // each 64-column chunk to 32 packed words, hand TMEM back, and
                // only then store -- the MMAs of the tile after next need not
                // wait for the stores.
                uint32_t packed[kChunks][32];
#pragma unroll
                for (int jj = 0; jj < kChunks; ++jj) {
                    const int j = half * kChunks + jj;
                    uint32_t v0[32], v1[32];
                    __syncwarp();
                    tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(kColsPerChunk * j), v0);
                    tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(kColsPerChunk * j + 32), v1);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const uint32_t *v = (i < 16) ? v0 : v1;
                        const int k = 2 * (i & 15);
                        const float a0 = (KIND == kKindI8) ? __int2float_rn(static_cast<int32_t>(v[k]))
                                                           : __uint_as_float(v[k]);
                        const float a1 = (KIND == kKindI8) ? __int2float_rn(static_cast<int32_t>(v[k + 1]))
                                                           : __uint_as_float(v[k + 1]);
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(a0, scale), __fmul_rn(a1, scale));
                        packed[jj][i] = *reinterpret_cast<const uint32_t *>(&b2);
                    }
                    if (args.acc_out && row_ok) {
                        // raw accumulators for parity checks (direct stores)
                        const int n0 = tn * BN + kColsPerChunk * j;
                        for (int h = 0; h < 4; ++h) {
                            const int n = n0 + 16 * h;
                            if (n >= N) break;
                            uint4 *dst = reinterpret_cast<uint4 *>(args.acc_out + static_cast<int64_t>(m) * args.ldo + n);
                            const uint32_t *src = (h < 2) ? v0 + 16 * h : v1 + 16 * (h - 2);
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                dst[q] = make_uint4(src[4 * q], src[4 * q + 1], src[4 * q + 2], src[4 * q + 3]);
                        }
                    }
                }
                tc_fence_before();
                release_accumulator(acc);
                // 32-column blocks (64-byte rows) staged in turn in the two
                // halves of the warp's buffer: a block waits only for the store
                // before last, so staging overlaps the previous store's read
#pragma unroll
                for (int jj = 0; jj < kChunks; ++jj) {
                    const int j = half * kChunks + jj;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int col = tn * BN + kColsPerChunk * j + 32 * hh;
                        if (col >= N || row0 >= args.M) continue;  // warp-uniform: block outside Y
                        const uint32_t sbuf = buf + static_cast<uint32_t>((nstore & 1) * (kEpiBufBytes / 2));
                        if (lane == 0) bulk_wait_group_read<1>();
                        __syncwarp();
                        // row `lane`: 4 chunks of 16 bytes, chunk c at position
                        // c ^ ((lane / 2) % 4) (the 64-byte swizzle of the output map)
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const uint32_t addr = sbuf + static_cast<uint32_t>(lane * 64 + ((c ^ ((lane >> 1) & 3)) * 16));
                            const int w0 = 16 * hh + 4 * c;
                            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(packed[jj][w0]),
                                         "r"(packed[jj][w0 + 1]), "r"(packed[jj][w0 + 2]), "r"(packed[jj][w0 + 3])
                                         : "memory");
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(mapY, sbuf, col, row0);
                            bulk_commit_group();
                        }
                        ++nstore;
                    }
                }
                continue;
            }
            // fp32: chunk by chunk (the two 128-byte blocks of a chunk need all
            // of its 64 registers), TMEM handed back after the last load
#pragma unroll 1
            for (int jj = 0; jj < kChunks; ++jj) {
                const int j = half * kChunks + jj;
                const int n0 = tn * BN + kColsPerChunk * j;
                uint32_t v0[32], v1[32];
                __syncwarp();
                tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(kColsPerChunk * j), v0);
                tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(kColsPerChunk * j + 32), v1);
                tmem_wait_ld();
                if (jj == kChunks - 1) {
                    // all of this warp's share of the accumulator is in registers
                    tc_fence_before();
                    release_accumulator(acc);
                }
                if (n0 >= N || row0 >= args.M) continue;  // warp-uniform: block outside Y
                const int nparts = args.out_fp32 ? 2 : 1;  // 128-byte row blocks in this chunk
                for (int part = 0; part < nparts; ++part) {
                    const int col = args.out_fp32 ? n0 + 32 * part : n0;
                    if (col >= N) break;  // warp-uniform
                    uint32_t w[32];
                    const bool has_res = EPI && args.residual != nullptr && row_ok;
                    if (args.out_fp32) {
                        const uint32_t *v = part ? v1 : v0;
                        // mask-gated output: the 32 keep bits of these columns
                        const uint32_t keep_bits =
                            (args.col_keep && row_ok)
                                ? *reinterpret_cast<const uint32_t *>(args.col_keep + static_cast<int64_t>(m) * args.keep_stride +
                                                                      col / 8)
                                : 0xffffffffu;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const float a = (KIND == kKindI8) ? __int2float_rn(static_cast<int32_t>(v[i]))
                                                              : __uint_as_float(v[i]);
                            float y = __fmul_rn(a, scale);
                            if constexpr (EPI) {
                                // the residual of columns col + 8q .. + 7, one 16-byte load per 8
                                const int q = i >> 3;
                                const uint4 r4 = (has_res && col + 8 * q < N)
                                                     ? *reinterpret_cast<const uint4 *>(args.residual + static_cast<int64_t>(m) * args.ldo + col + 8 * q)
                                                     : make_uint4(0u, 0u, 0u, 0u);
                                const int e = i & 7;
                                const uint32_t word = e < 2 ? r4.x : e < 4 ? r4.y : e < 6 ? r4.z : r4.w;
                                y = epilogue_op(y, args.relu2, (word >> (16 * (e & 1))) & 0xffffu, has_res);
                            }
                            w[i] = ((keep_bits >> i) & 1u) ? __float_as_uint(y) : 0u;
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const uint32_t *v = (i < 16) ? v0 : v1;
                            const int k = 2 * (i & 15);
                            const float a0 = (KIND == kKindI8) ? __int2float_rn(static_cast<int32_t>(v[k]))
                                                               : __uint_as_float(v[k]);
                            const float a1 = (KIND == kKindI8) ? __int2float_rn(static_cast<int32_t>(v[k + 1]))
                                                               : __uint_as_float(v[k + 1]);
                            float y0 = __fmul_rn(a0, scale), y1 = __fmul_rn(a1, scale);
                            if constexpr (EPI) {
                                // word i of the residual row holds columns col + 2i, col + 2i + 1
                                const int q = i >> 2;
                                const uint4 r4 = (has_res && col + 8 * q < N)
                                                     ? *reinterpret_cast<const uint4 *>(args.residual + static_cast<int64_t>(m) * args.ldo + col + 8 * q)
                                                     : make_uint4(0u, 0u, 0u, 0u);
                                const int e = i & 3;
                                const uint32_t word = e == 0 ? r4.x : e == 1 ? r4.y : e == 2 ? r4.z : r4.w;
                                y0 = epilogue_op(y0, args.relu2, word & 0xffffu, has_res);
                                y1 = epilogue_op(y1, args.relu2, word >> 16, has_res);
                            }
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(y0, y1);
                            w[i] = *reinterpret_cast<const uint32_t *>(&b2);
                        }
                    }
                    // the previous store from this buffer has finished reading it
                    if (lane == 0) bulk_wait_group_read<0>();
                    __syncwarp();
                    // row `lane`: 8 chunks of 16 bytes, chunk c at position c ^ (lane % 8)
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t addr = buf + static_cast<uint32_t>(lane * 128 + ((c ^ (lane & 7)) * 16));
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[4 * c]),
                                     "r"(w[4 * c + 1]), "r"(w[4 * c + 2]), "r"(w[4 * c + 3])
                                     : "memory");
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(mapY, buf, col, row0);
                        bulk_commit_group();
                    }
                }
                if (args.acc_out && row_ok) {
                    // raw accumulators for parity checks (direct stores)
                    for (int h = 0; h < 4; ++h) {
                        const int n = n0 + 16 * h;
                        if (n >= N) break;
                        uint4 *dst = reinterpret_cast<uint4 *>(args.acc_out + static_cast<int64_t>(m) * args.ldo + n);
                        const uint32_t *src = (h < 2) ? v0 + 16 * h : v1 + 16 * (h - 2);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[q] = make_uint4(src[4 * q], src[4 * q + 1], src[4 * q + 2], src[4 * q + 3]);
                    }
                }
            }
        }
        if (lane == 0) bulk_wait_group<0>();  // every store has landed before the CTA exits
        __syncwarp();
    }

    __syncthreads();
    // neither CTA of a pair leaves while the other may still read its shared
    // memory or arrive on its barriers
    if constexpr (PAIR) cluster_sync_all();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        if constexpr (PAIR)
            tmem_dealloc_pair(tmem_base, kTmemCols);
        else
            tmem_dealloc(tmem_base, kTmemCols);
    }
}

template <int KIND, int BN, bool EPI = false, bool PAIR = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmY, GemmArgs args)
{
    gemm_body<KIND, BN, EPI, PAIR, 1>(&tmA, &tmB, &tmY, args, GemmGroups{});
}

// The products of one launch that share A (the int8 forward of several
// layers on the same activations), every map and group in the parameters.
struct GemmGroupParams {
    CUtensorMap a;
    CUtensorMap b[kGemmMaxGroups];
    CUtensorMap y[kGemmMaxGroups];
    GemmArgs args;
    GemmGroups grp;
};

template <int BN, bool PAIR>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_group_kernel(const __grid_constant__ GemmGroupParams p)
{
    gemm_body<kKindI8, BN, false, PAIR, kGemmMaxGroups>(&p.a, p.b, p.y, p.args, p.grp);
}

}  // namespace sbl
