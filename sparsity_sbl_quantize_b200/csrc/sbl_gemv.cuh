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
//  * one CTA per SM runs for the whole batch; its work items are 32-row
//    blocks of the layers (16 rows when K is large), taken round-robin over
//    the grid in batch order;
//  * a producer warp streams each item's packed rows -- contiguous, since a
//    PK2 row is exactly K / 4 bytes when K % 64 == 0 -- with ONE bulk copy
//    (cp.async.bulk, evict-first in L2) into a ring of shared-memory stages,
//    as far ahead as the ring allows and across layer boundaries: the
//    weights never depend on the activations, so no launch gap or
//    dependency stalls the stream;
//  * eight consumer warps split the item's 256-weight K chunks, each doing
//    both 16-row tiles per activation fragment, free the stage, and meet in
//    shared memory (exact int32 partials) where 32 T threads dequantise;
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
constexpr int kGvWarps = 8;                       // consumer warps
constexpr int kGvThreads = 32 * (kGvWarps + 1);   // + the producer warp
constexpr int kGvStageBytes = 56 * 1024;          // one item: 32 rows x K/4 for K <= 7168
constexpr int kGvStages = 3;
constexpr int kGvPartStride = 36;                 // padded row count of a token's partials
constexpr int kGvSyncWords = 32;                  // per layer: [0] items done, [1 + t] max |y_t| bits
constexpr int kGvSmemBytes = kGvStages * kGvStageBytes + 2 * kGvWarps * kDecMaxTokens * kGvPartStride * 4 +
                             2 * kGvWarps * kDecMaxTokens * 4 + 2 * kGvStages * 8;

enum : int32_t {
    kGvOutFp32 = 1,   // Y is fp32 (else bf16)
    kGvChained = 2,   // the input is the previous layer's bf16 output
    kGvPublish = 4,   // the next layer is chained on this one: publish max |y| and item counts
    kGvRows16 = 8,    // items of 16 rows (large K), else 32
};

struct GvProblem {
    const uint8_t *pk2;  // PK2 codes [O, K / 4]
    const float *gamma;  // device scalar
    const int8_t *xq;    // [T, K] int8 activations (unchained layers)
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

__device__ __forceinline__ void gv_consumer_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

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

// Lane (g, tg)'s 64 activations of token t at positions pos .. pos + 63 as
// four 16-byte int8 groups.  Unchained: the int8 input.  Chained: the previous
// layer's bf16 outputs, quantised with r = fl32(127 / a_t) (a_t == 0: zeros).
__device__ __forceinline__ void gv_load_x(const GvProblem &P, const GvProblem &prev, bool chained, int t, int pos,
                                          float r, uint4 (&x)[4])
{
    if (!chained) {
        const int8_t *src = P.xq + static_cast<int64_t>(t) * P.K + pos;
#pragma unroll
        for (int q = 0; q < 4; ++q) x[q] = ld_global16(src + 16 * q);
        return;
    }
    const uint16_t *src = static_cast<const uint16_t *>(prev.y) + static_cast<int64_t>(t) * P.K + pos;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
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

// NT: n8 token blocks (T <= 8: 1, T <= 16: 2).
template <int NT>
__global__ void __launch_bounds__(kGvThreads, 1) gemv_stream_kernel(const __grid_constant__ GvArgs args)
{
    extern __shared__ __align__(128) uint8_t gv_smem[];
    int32_t *part = reinterpret_cast<int32_t *>(gv_smem + kGvStages * kGvStageBytes);  // [2][warp][t][row]
    int32_t *csum = part + 2 * kGvWarps * kDecMaxTokens * kGvPartStride;                 // [2][warp][t]
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
            const int item_rows = (P.flags & kGvRows16) ? 16 : 32;
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
        const int item_rows = (P.flags & kGvRows16) ? 16 : 32;
        const int r0 = (item - P.item0) * item_rows;
        const int rows = min(item_rows, P.O - r0);
        const int K = P.K, kb = K / 4;
        const int chunks = (K + kDecChunk - 1) / kDecChunk;
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
        const bool tile1 = rows > 16;  // warp-uniform
        // acc[u][j][b]: tile u, code position j (weights scaled by 4^j), token block b
        int32_t acc[2][4][NT][4];
        uint32_t cs[NT];
#pragma unroll
        for (int b = 0; b < NT; ++b) {
            cs[b] = 0u;
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[u][j][b][0] = acc[u][j][b][1] = acc[u][j][b][2] = acc[u][j][b][3] = 0;
        }
        const bool store_xq = chained && P.xq_out && item == P.item0;
        for (int c = warp; c < chunks; c += kGvWarps) {
            const int pos = c * kDecChunk + 64 * tg;
            const bool kin = pos < K;
            // the lane's 16 bytes of rows g, g + 8, 16 + g, 24 + g (zeros past K or the item)
            uint4 w[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int row = g + 8 * r;
                w[r] = (kin && row < rows) ? ld_shared16(st + static_cast<uint32_t>(row * kb + pos / 4))
                                           : make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u);
            }
            uint4 xt[NT][4];
#pragma unroll
            for (int b = 0; b < NT; ++b) {
                const int t = 8 * b + g;
                uint4 x[4];
                if (kin && t < T) {
                    gv_load_x(P, prev, chained, t, pos, rq[b], x);
                    if (store_xq) {
                        uint4 *dst = reinterpret_cast<uint4 *>(P.xq_out + static_cast<int64_t>(t) * K + pos);
#pragma unroll
                        for (int q = 0; q < 4; ++q) dst[q] = x[q];
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 4; ++q) x[q] = make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    int s = static_cast<int>(cs[b]);
                    s = __dp4a(static_cast<int>(x[q].x), 0x01010101, s);
                    s = __dp4a(static_cast<int>(x[q].y), 0x01010101, s);
                    s = __dp4a(static_cast<int>(x[q].z), 0x01010101, s);
                    s = __dp4a(static_cast<int>(x[q].w), 0x01010101, s);
                    cs[b] = static_cast<uint32_t>(s);
                    xt[b][q] = transpose4x4(x[q]);
                }
            }
            // Weight word wi of a row holds positions 16 wi .. 16 wi + 15, byte
            // e the four positions 16 wi + 4 e + j at bits 2 j.  Masking code
            // position j in place (one op) leaves byte e = c(16 wi + 4 e + j) 4^j,
            // which pairs with word j of the transposed activation group wi
            // (byte e = x(16 wi + 4 e + j)).  One MMA takes words (0, 1) or
            // (2, 3) of a row at one j; the 4^j stays in that j's accumulator.
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t mj = 0x03030303u << (2 * j);
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        if (u == 1 && !tile1) break;
                        const uint32_t a0 = word_of(w[2 * u], 2 * h) & mj;
                        const uint32_t a1 = word_of(w[2 * u + 1], 2 * h) & mj;
                        const uint32_t a2 = word_of(w[2 * u], 2 * h + 1) & mj;
                        const uint32_t a3 = word_of(w[2 * u + 1], 2 * h + 1) & mj;
#pragma unroll
                        for (int b = 0; b < NT; ++b)
                            mma_u8s8(acc[u][j][b], a0, a1, a2, a3, word_of(xt[b][2 * h], j),
                                     word_of(xt[b][2 * h + 1], j));
                    }
                }
            }
        }
        // this warp is done with the stage: the producer may refill it
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(stage));
        if (++stage == kGvStages) stage = 0, phase ^= 1u;

        // partials: part[buf][warp][token][row], column sums csum[buf][warp][token]
        int32_t *pw = part + (buf * kGvWarps + warp) * kDecMaxTokens * kGvPartStride;
#pragma unroll
        for (int b = 0; b < NT; ++b) {
            const int tA = 8 * b + 2 * tg;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                // fold the code positions back: acc[j] is a multiple of 4^j
                // (every product is), so the arithmetic shifts are exact
                int32_t v[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    v[e] = acc[u][0][b][e] + (acc[u][1][b][e] >> 2) + (acc[u][2][b][e] >> 4) + (acc[u][3][b][e] >> 6);
                const int rA = 16 * u + g;
                pw[tA * kGvPartStride + rA] = v[0];
                pw[(tA + 1) * kGvPartStride + rA] = v[1];
                pw[tA * kGvPartStride + rA + 8] = v[2];
                pw[(tA + 1) * kGvPartStride + rA + 8] = v[3];
            }
            uint32_t s = cs[b];
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            if (tg == 0) csum[(buf * kGvWarps + warp) * kDecMaxTokens + 8 * b + g] = static_cast<int32_t>(s);
        }
        gv_consumer_sync();
        if (s_fail[buf]) break;

        // thread (t, r): sum the warps' partials (wrapping int32 arithmetic is
        // exact when the result fits), dequantise, store
        const float gam = ld_global_f32(P.gamma);
        const bool publish = (P.flags & kGvPublish) != 0;
        for (int o = threadIdx.x; o < T * 32; o += kGvWarps * 32) {
            const int t = o >> 5, r = o & 31;
            float d_t;
            if (chained) {
                const float a = __uint_as_float(ld_acquire_u32(args.sync + (p - 1) * kGvSyncWords + 1 + t));
                d_t = a > 0.0f ? __fdiv_rn(a, 127.0f) : 0.0f;
            } else {
                d_t = ld_global_f32(P.d + t);
            }
            uint32_t absbits = 0u;
            if (r < rows) {
                uint32_t s = 0u;
#pragma unroll
                for (int w = 0; w < kGvWarps; ++w)
                    s += static_cast<uint32_t>(part[((buf * kGvWarps + w) * kDecMaxTokens + t) * kGvPartStride + r]) -
                         static_cast<uint32_t>(csum[(buf * kGvWarps + w) * kDecMaxTokens + t]);
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
                // max |y_t| of the bf16 outputs (their fp32 bits order like the values)
                absbits = __reduce_max_sync(0xffffffffu, absbits);
                if (lane == 0 && absbits) atomicMax(args.sync + p * kGvSyncWords + 1 + t, absbits << 16);
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
