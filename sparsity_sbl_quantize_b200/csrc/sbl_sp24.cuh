// sbl_sp24.cuh -- the forward GEMM of the Sparse-BitLinear layer on the 2:4
// sparse tensor cores of sm_100a (tcgen05.mma.sp, kind::i8), run by CTA pairs.
//
//   acc[t, o] = sum_k W_eff[o, k] * Xq[t, k]
//   Y[t, o]   = fl32(fl32(acc[t, o]) * fl32(gamma * d_t))
//
// ("The Full Sparse-BitLinear Layer", forward step 5 of the Sparse-BitNet
// summary.)  When every group of four weights along K keeps at most two
// (n <= 2 of m = 4 or 8), W_eff is stored as the sparse MMA operand (SP24:
// two int8 values per group of four plus a 4-bit nibble giving their two
// positions) and the tensor core skips the zero half, so each MMA covers 64
// logical K with the operand bytes of 32.
//
// The sparse operand is A, so the tile is weight rows (TMEM lanes) x tokens
// (TMEM columns), the transpose of the dense kernel's tile.  Per stage (256
// logical K) a CTA loads A = 128 rows x 128 compressed bytes (TMA, 128-byte
// swizzle), B = its share of the tokens x 256 bytes (two 128-byte swizzled
// boxes) and E = the metadata, 128 rows x 32 bytes, by TMA as a 3-D box into
// the no-swizzle canonical layout ([2][128][16] bytes) that tcgen05.cp copies
// into tensor memory (lane = weight row; the 64 metadata bits of one MMA fill
// two columns, nibble g at bits 4g).
#pragma once

#include <cuda_bf16.h>

#include "sbl_device.cuh"
#include "sbl_gemm.cuh"  // tile raster, role sizes

namespace sbl {

constexpr int kSpBM = 128;                       // weight rows per CTA
constexpr int kSpKLogical = 256;                 // logical K per stage
constexpr int kSpABytes = kSpBM * 128;           // 128 compressed bytes per row
constexpr int kSpEBytes = kSpBM * 32;            // 32 metadata bytes per row
constexpr int kSpEpiBufBytes = 32 * 32 * 4;      // one 32 x 32 block, fp32 at most
constexpr int kSpEpiBytes = kEpiWarps * kSpEpiBufBytes;

struct Sp24Args {
    int32_t O, T, K;
    int32_t tiles_m, tiles_n;  // weight-row tiles, token tiles
    int32_t k_blocks;          // ceil(K / 256)
    void *out;                 // [T, O] bf16 bits or fp32
    int32_t out_fp32;
    int32_t *acc_out;          // optional [T, O] int32
    const float *gamma;
    const float *d;            // [T]
    int32_t relu2;             // output epilogue: v = max(v, 0)^2 ...
    const uint16_t *residual;  // ... then v = v + residual[t, o] (bf16 [T, O]; nullptr: none)
    uint32_t *err;
};

// ------------------------------------------------------------ CTA pairs --
// The same GEMM on CTA pairs (cta_group::2): a cluster of two CTAs computes a
// 256-weight-row x BN-token tile with M = 256 MMAs issued by the even CTA.
// Each CTA loads its own 128 rows of A and E and half of the tile's tokens
// (BN / 2 rows of B), so a B byte fetched from L2 feeds 256 weight rows
// instead of 128; every CTA's tensor memory holds its 128 rows x BN columns.
// The odd CTA's loads complete on the even CTA's full barriers (which expect
// the bytes of both), the even CTA's commits arrive on the barriers of both,
// and both CTAs' epilogue warps arrive on the even CTA's accumulator-free
// barriers.  A final cluster barrier keeps each CTA alive until the other no
// longer touches its shared memory.
template <int BN>
struct Sp24PairCfg {
    static_assert(BN % 32 == 0 && BN >= 64 && BN <= 224, "pair tile width");
    static constexpr int kBHalf = BN / 2;                        // token rows per CTA
    static constexpr int kBBoxBytes = kBHalf * 128;
    static constexpr int kBBytes = 2 * kBBoxBytes;
    static constexpr int kStageBytes = kSpABytes + kBBytes + kSpEBytes;
    static constexpr int kStages = (192 * 1024) / kStageBytes < 6 ? (192 * 1024) / kStageBytes : 6;
    static constexpr int kNumAcc = 2;
    static constexpr int kMetaCol = kNumAcc * BN;
    static_assert(kMetaCol + 8 * kStages <= kTmemCols, "tensor memory");
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kSpEpiBytes + 256;
};

template <int BN>
__device__ __forceinline__ constexpr uint32_t sp24_pair_idesc()
{
    return (1u << 2) | (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
           (static_cast<uint32_t>(256 >> 4) << 24);
}

__device__ __forceinline__ void mma_sp_i8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t e_tmem,
                                               uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "tcgen05.mma.sp.cta_group::2.kind::i8 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tmem_cp_128x256b_pair(uint32_t taddr, uint32_t saddr)
{
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(2048u >> 4) << 16;
    d |= static_cast<uint64_t>(128u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    asm volatile("tcgen05.cp.cta_group::2.128x256b [%0], %1;" ::"r"(taddr), "l"(d) : "memory");
}

// EPI: the instantiation with the output epilogue (relu2 / residual).
template <int BN, bool EPI = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    sp24_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmY,
                     Sp24Args args)
{
    using Cfg = Sp24PairCfg<BN>;
    constexpr int kStages = Cfg::kStages;
    constexpr int kNumAcc = Cfg::kNumAcc;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw);
    const uint32_t a_base = base;
    const uint32_t b_base = a_base + kStages * kSpABytes;
    const uint32_t e_base = b_base + kStages * Cfg::kBBytes;
    const uint32_t epi_base = e_base + kStages * kSpEBytes;
    const uint32_t bar_base = epi_base + kSpEpiBytes;
    auto full_bar = [&](int s) { return bar_base + 8u * s; };
    auto empty_bar = [&](int s) { return bar_base + 8u * (kStages + s); };
    auto tfull_bar = [&](int a) { return bar_base + 8u * (2 * kStages + a); };
    auto tempty_bar = [&](int a) { return bar_base + 8u * (2 * kStages + kNumAcc + a); };
    const uint32_t drain_bar = bar_base + 8u * (2 * kStages + 2 * kNumAcc);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + (bar_base - base) + 224);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster_id = static_cast<int>(blockIdx.x >> 1);
    const int num_clusters = static_cast<int>(gridDim.x >> 1);
    const int num_tiles = args.tiles_m * args.tiles_n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < kNumAcc; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), 2 * kEpiWarps);  // one arrival per epilogue warp of both CTAs
        }
        mbar_init(drain_bar, 1);
        fence_barrier_init();
        tma_prefetch_map(&tmA);
        tma_prefetch_map(&tmB);
        tma_prefetch_map(&tmE);
        tma_prefetch_map(&tmY);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_addr(tmem_slot), kTmemCols);
        tmem_relinquish_pair();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    // both CTAs' barriers are initialised before either CTA signals the other
    cluster_sync_all();
    const uint32_t tmem_base = *tmem_slot;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer (both CTAs)
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        uint32_t issued_mask = 0;
        uint32_t issued_phase[kStages];
        for (int s = 0; s < kStages; ++s) issued_phase[s] = 0;
        for (int tile = cluster_id; ok && tile < num_tiles; tile += num_clusters) {
            int tm, tn;
            tile_coords(tile, args.tiles_m, args.tiles_n, tm, tn);
            const int row0 = tm * 256 + static_cast<int>(rank) * kSpBM;
            const int tok0 = tn * BN + static_cast<int>(rank) * Cfg::kBHalf;
            for (int kb = 0; kb < args.k_blocks; ++kb) {
                const bool ready = mbar_wait(empty_bar(stage), phase ^ 1u, args.err, kErrGemmProducer);
                if (!__all_sync(0xffffffffu, ready)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    const uint32_t fb = map_shared_rank(full_bar(stage), 0);  // the even CTA's barrier
                    if (leader) mbar_arrive_expect_tx(full_bar(stage), 2 * Cfg::kStageBytes);
                    tma_load_2d_pair(a_base + stage * kSpABytes, &tmA, kb * 128, row0, fb);
                    tma_load_2d_pair(b_base + stage * Cfg::kBBytes, &tmB, kb * kSpKLogical, tok0, fb);
                    tma_load_2d_pair(b_base + stage * Cfg::kBBytes + Cfg::kBBoxBytes, &tmB, kb * kSpKLogical + 128,
                                     tok0, fb);
                    tma_load_3d_pair(e_base + stage * kSpEBytes, &tmE, 0, row0, 2 * kb, fb);
                }
                __syncwarp();
                issued_mask |= 1u << stage;
                issued_phase[stage] = phase;
                if (++stage == kStages) stage = 0, phase ^= 1u;
            }
        }
        if (!ok && leader) {
            for (int s = 0; s < kStages; ++s)
                if (issued_mask & (1u << s)) mbar_wait(full_bar(s), issued_phase[s], args.err, kErrGemmProducer);
        }
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer (even CTA)
        if (leader) {
            constexpr uint32_t idesc = sp24_pair_idesc<BN>();
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int local = 0;
            for (int tile = cluster_id; ok && tile < num_tiles; tile += num_clusters, ++local) {
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
                        const uint32_t e_tmem = tmem_base + static_cast<uint32_t>(Cfg::kMetaCol + 8 * stage);
                        tmem_cp_128x256b_pair(e_tmem, e_base + stage * kSpEBytes);
                        const uint64_t adesc = smem_desc_k128(a_base + stage * kSpABytes);
                        const uint32_t b_stage = b_base + stage * Cfg::kBBytes;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint64_t bdesc = smem_desc_k128(b_stage + (j >> 1) * Cfg::kBBoxBytes) +
                                                   static_cast<uint64_t>(4 * (j & 1));
                            mma_sp_i8_pair(d_tmem, adesc + static_cast<uint64_t>(2 * j), bdesc, e_tmem + 2u * j,
                                           idesc, (kb | j) != 0);
                        }
                        tc_commit_pair(empty_bar(stage), 0x3);  // frees the stage in both CTAs
                    }
                    __syncwarp();
                    if (++stage == kStages) stage = 0, phase ^= 1u;
                }
                if (!ok) break;
                if (lane == 0) tc_commit_pair(tfull_bar(acc), 0x3);
                __syncwarp();
            }
            if (lane == 0) tc_commit_pair(drain_bar, 0x1);
            __syncwarp();
            mbar_wait(drain_bar, 0, args.err, kErrGemmMma);
            __syncwarp();
        }
    } else {
        // ---------------------------------------------------- epilogue (warps 2-9, both CTAs)
        const int quarter = warp & 3;
        const int half = (warp - 2) >> 2;
        const float g = *args.gamma;
        const uint32_t buf = epi_base + static_cast<uint32_t>(warp - 2) * kSpEpiBufBytes;
        uint32_t nstore = 0;  // bf16 stores issued by this warp (staging buffer = nstore % 2)
        int local = 0;
        for (int tile = cluster_id; tile < num_tiles; tile += num_clusters, ++local) {
            int tm, tn;
            tile_coords(tile, args.tiles_m, args.tiles_n, tm, tn);
            const int acc = local % kNumAcc;
            const uint32_t acc_phase = (local / kNumAcc) & 1;
            const int o0 = tm * 256 + static_cast<int>(rank) * kSpBM + quarter * 32;
            const int o = o0 + lane;
            constexpr int kChunks = BN / 32;
            constexpr int kMine = (kChunks + 1) / 2;  // chunks c = half, half + 2, ... (warp half 0 has the extra)
            // the token scales of this warp's chunks are loaded while the
            // tile's MMAs still run (one L2 round trip per tile, not per chunk)
            float d_pre[kMine];
#pragma unroll
            for (int i = 0; i < kMine; ++i) {
                const int t = tn * BN + 32 * (half + 2 * i) + lane;
                d_pre[i] = (half + 2 * i < kChunks && t < args.T) ? args.d[t] : 0.0f;
            }
            const bool ready = mbar_wait(tfull_bar(acc), acc_phase, args.err, kErrGemmEpilogue);
            if (!__all_sync(0xffffffffu, ready)) break;
            tc_fence_after();
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(acc * BN);
            if (!args.out_fp32 && !EPI) {
                // bf16: drain every chunk of this warp, converting it to 16
                // packed words of the transposed block (lanes 2i and 2i+1 swap
                // one value so each holds a word of two weight rows: the even
                // lane token j, the odd lane token j + 1), hand the
                // accumulator back, and only then stage and store
                uint32_t packed[kMine][16];
                const bool odd = lane & 1;
                // 16 tokens per step, step s = chunk s / 2, half s % 2; the
                // next step's TMEM load is in flight while this one converts
                // (registers va / vb in turn)
                uint32_t va[16], vb[16];
                tmem_ld_32x32b_x16(t_row + static_cast<uint32_t>(32 * half), va);
#pragma unroll
                for (int st = 0; st < 2 * kMine; ++st) {
                    const int i = st >> 1, hh = st & 1;
                    const int c = half + 2 * i;
                    if (c >= kChunks) break;  // warp-uniform
                    tmem_wait_ld();
                    const int cn = half + 2 * ((st + 1) >> 1);
                    if (st + 1 < 2 * kMine && cn < kChunks)
                        tmem_ld_32x32b_x16(t_row + static_cast<uint32_t>(32 * cn + 16 * ((st + 1) & 1)), hh ? va : vb);
                    const uint32_t(&v)[16] = hh ? vb : va;
                    const int t0 = tn * BN + 32 * c;
                    const int t = t0 + lane;
                    const float sc = t < args.T ? __fmul_rn(g, d_pre[i]) : 0.0f;
#pragma unroll
                    for (int jj = 0; jj < 16; jj += 2) {
                        const int j = 16 * hh + jj;
                        const float s0 = __shfl_sync(0xffffffffu, sc, j);
                        const float s1 = __shfl_sync(0xffffffffu, sc, j + 1);
                        const float y0 = __fmul_rn(__int2float_rn(static_cast<int32_t>(v[jj])), s0);
                        const float y1 = __fmul_rn(__int2float_rn(static_cast<int32_t>(v[jj + 1])), s1);
                        const float other = __shfl_xor_sync(0xffffffffu, odd ? y0 : y1, 1);
                        const __nv_bfloat162 b2 =
                            odd ? __floats2bfloat162_rn(other, y1) : __floats2bfloat162_rn(y0, other);
                        packed[i][j >> 1] = *reinterpret_cast<const uint32_t *>(&b2);
                    }
                    if (args.acc_out && o < args.O && t0 < args.T && o0 < args.O) {
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj)
                            if (t0 + 16 * hh + jj < args.T)
                                args.acc_out[static_cast<int64_t>(t0 + 16 * hh + jj) * args.O + o] =
                                    static_cast<int32_t>(v[jj]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(map_shared_rank(tempty_bar(acc), 0));
#pragma unroll
                for (int i = 0; i < kMine; ++i) {
                    const int c = half + 2 * i;
                    if (c >= kChunks) break;
                    const int t0 = tn * BN + 32 * c;
                    if (t0 >= args.T || o0 >= args.O) continue;  // warp-uniform: block outside Y
                    // two 2 KiB staging buffers used in turn: the previous
                    // store from this one has finished reading it
                    const uint32_t sbuf = buf + static_cast<uint32_t>((nstore & 1) * 2048);
                    if (lane == 0) bulk_wait_group_read<1>();
                    __syncwarp();
                    const int row_off = (lane & 1) ? 1 : 0;
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        const uint32_t addr = sbuf + static_cast<uint32_t>((j + row_off) * 64 + (lane & ~1) * 2);
                        asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(packed[i][j >> 1]) : "memory");
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmY, sbuf, o0, t0);
                        bulk_commit_group();
                    }
                    ++nstore;
                }
                continue;
            }
            // fp32, or any output with the epilogue: chunk by chunk, the
            // accumulator handed back after the last load
#pragma unroll 1
            for (int c = half; c < kChunks; c += 2) {
                const int t0 = tn * BN + 32 * c;
                const int t = t0 + lane;
                float dt = d_pre[0];
#pragma unroll
                for (int i = 1; i < kMine; ++i)
                    if (c == half + 2 * i) dt = d_pre[i];
                const float sc = t < args.T ? __fmul_rn(g, dt) : 0.0f;
                uint32_t v[32];
                tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(32 * c), v);
                tmem_wait_ld();
                if (c + 2 >= kChunks) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(map_shared_rank(tempty_bar(acc), 0));
                }
                if (t0 >= args.T || o0 >= args.O) continue;  // warp-uniform: block outside Y
                if (args.acc_out && o < args.O) {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (t0 + j < args.T)
                            args.acc_out[static_cast<int64_t>(t0 + j) * args.O + o] = static_cast<int32_t>(v[j]);
                }
                if (lane == 0) bulk_wait_group_read<0>();  // every earlier store has read its staging
                __syncwarp();
                const bool has_res = EPI && args.residual != nullptr && o < args.O;
                const bool odd = lane & 1;
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    float y[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float s = __shfl_sync(0xffffffffu, sc, j + h);
                        y[h] = __fmul_rn(__int2float_rn(static_cast<int32_t>(v[j + h])), s);
                        if constexpr (EPI) {
                            // the lanes of a warp read consecutive weight rows of one token
                            const uint32_t rb = (has_res && t0 + j + h < args.T)
                                                    ? args.residual[static_cast<int64_t>(t0 + j + h) * args.O + o]
                                                    : 0u;
                            y[h] = epilogue_op(y[h], args.relu2, rb, has_res);
                        }
                    }
                    if (args.out_fp32) {
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            asm volatile("st.shared.f32 [%0], %1;" ::"r"(buf + static_cast<uint32_t>((j + h) * 128 + lane * 4)),
                                         "f"(y[h])
                                         : "memory");
                    } else {
                        // lanes 2i and 2i+1 swap one value: the even lane writes
                        // token j of weight rows 2i, 2i+1, the odd lane token j+1
                        const float other = __shfl_xor_sync(0xffffffffu, odd ? y[0] : y[1], 1);
                        const __nv_bfloat162 b2 =
                            odd ? __floats2bfloat162_rn(other, y[1]) : __floats2bfloat162_rn(y[0], other);
                        const uint32_t addr = buf + static_cast<uint32_t>((j + (odd ? 1 : 0)) * 64 + (lane & ~1) * 2);
                        asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(*reinterpret_cast<const uint32_t *>(&b2))
                                     : "memory");
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmY, buf, o0, t0);
                    bulk_commit_group();
                }
            }
        }
        if (lane == 0) bulk_wait_group<0>();
        __syncwarp();
    }

    __syncthreads();
    // neither CTA leaves while the other may still read its shared memory or
    // arrive on its barriers
    cluster_sync_all();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

}  // namespace sbl
