// sbl_pack.cuh -- weight side of the Sparse-BitLinear layer on sm_100a:
//   * gamma: mean |W| (Sparse-BitNet summary, section 3.4, "Step 1: Compute
//     the Rescaling Factor"), summed in fp64 over the pairwise tree of the
//     flat row-major order, so the result does not depend on the grid;
//   * the fused N:M mask ("N:M Mask Generation"), ternarisation ("Step 2:
//     Rescale and RoundClip") and mask application ("Composition Order"),
//     writing the packed formats in one pass over W.
#pragma once

#include <type_traits>

#include "sbl_device.cuh"

namespace sbl {

// Elements per first-level partial of the gamma tree (a tree node: the
// partial of block j covers [j * kGammaBlock, (j + 1) * kGammaBlock)).
constexpr int kGammaBlock = 8192;
// Leaves of the second-level tree: 256 threads x 128 partials each.
constexpr int kGammaMaxPartials = 32768;

struct GammaWorkspace {
    double partials[kGammaMaxPartials];
    uint32_t counter;       // blocks finished (zeroed by the host before each launch)
    uint32_t pad[3];
};

// Given gamma, the fp32 threshold T such that for every finite fp32 x
//   clamp(rint_half_even(fl32(|x| / gamma)), 0, 1) == 1  <=>  |x| >= T.
// fl32(q) > 0.5 exactly when q > 0.5 + 2^-25 (the midpoint to the next float
// above 0.5 rounds to the even 0.5), so T is the first float above the exact
// product gamma * (0.5 + 2^-25), which fp64 holds without rounding.  gamma == 0
// means every W_q is 0 (no float passes +inf).
__device__ __forceinline__ float ternary_threshold(float gamma)
{
    if (!(gamma > 0.0f)) return __int_as_float(0x7f800000);
    const double t = static_cast<double>(gamma) * (0.5 + 0x1p-25);
    float f = __double2float_ru(t);
    if (static_cast<double>(f) == t) f = __int_as_float(__float_as_int(f) + 1);
    return f;
}

// Packed output buffers of one pack launch.
struct PackOut {
    uint8_t *pk2;
    int64_t pk2_stride;
    int8_t *i8;
    uint8_t *nm_values;
    int64_t nm_values_stride;
    uint8_t *nm_bitmap;
    int64_t nm_bitmap_stride;
    int8_t *sp24_values;
    int64_t sp24_values_stride;
    uint8_t *sp24_meta;
    int64_t sp24_meta_stride;
    uint8_t *t24_lo;
    int64_t t24_lo_stride;
    uint8_t *t24_hi;
    int64_t t24_hi_stride;
};

// By-product statistics of the re-mask step (all optional; the counters are
// zeroed by the host before the launch).
struct PackStats {
    const uint8_t *prev_keep;        // keep bitmap of the previous step (bit k%8 of byte k/8)
    uint8_t *keep;                   // this step's keep bitmap, same layout
    int64_t keep_stride;             // bytes per bitmap row
    unsigned long long *flips;       // positions whose keep bit changed
    unsigned long long *near_zero;   // weights with fl32(|w| / gamma) < 0.5
    float *threshold;                // [rows, cols / M] largest dropped |w| per group
};

struct PackArgs {
    const void *W;         // fp32 or bf16 master weights
    int32_t rows, cols, n;
    int64_t count;         // rows * cols (a multiple of 16)
    uint64_t inv_cols;     // ceil(2^64 / cols): row = umul64hi(e, inv_cols) exactly for e < 2^28
    const float *gamma;    // written by gamma_kernel
    PackOut out;
    PackStats stats;
};

// fl32(|w| / gamma) < 0.5 exactly when |w| < gamma * (0.5 - 2^-26) (the
// quotients that round to a float below 0.5; the midpoint 0.5 - 2^-26 rounds
// to the even 0.5), and that product is exact in fp64: |w| is below it
// exactly when it is below the first fp32 at or above it.  Every weight
// counts when gamma == 0.
__device__ __forceinline__ uint32_t near_zero_bound_bits(float gamma)
{
    if (!(gamma > 0.0f)) return 0x7f800000u;  // +inf: every finite |w| is below
    return __float_as_uint(__double2float_ru(static_cast<double>(gamma) * (0.5 - 0x1p-26)));
}

template <int M>
__device__ __forceinline__ uint32_t keep_mask(const uint32_t (&key)[M], int n);

// Master weights are fp32 or bf16 (uint16_t bits); a bf16 weight is the fp32
// with the same upper 16 bits, so every step below sees exact fp32 values.
template <typename WT>
__device__ __forceinline__ float4 load4(const WT *W, int64_t e)
{
    if constexpr (sizeof(WT) == 4) {
        return __ldg(reinterpret_cast<const float4 *>(W + e));
    } else {
        const uint2 v = __ldg(reinterpret_cast<const uint2 *>(W + e));
        return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                           __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
    }
}

// Second level of the gamma tree, over the node partials parts[0 .. nparts)
// (nparts <= kGammaMaxPartials): chunks of 2048 partials (tree nodes); in each
// chunk thread t loads [8t, 8t + 8) (all threads, loads in flight together), a
// butterfly and a shared-memory tree combine the 256 thread sums, and the <= 16
// chunk sums finish pairwise (zeros past the end).  Called by all 256 threads
// of a CTA; the result is valid in thread 0.
__device__ __forceinline__ double gamma_tree_finish(const double *parts, int nparts, double *warp_sums,
                                                   double *chunk_sums)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nchunks = (nparts + 2047) / 2048;
    for (int c = 0; c < nchunks; ++c) {
        double v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int j = c * 2048 + threadIdx.x * 8 + i;
            v[i] = (j < nparts) ? __ldcg(&parts[j]) : 0.0;
        }
        double u = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) u = u + __shfl_xor_sync(0xffffffffu, u, off);
        if (lane == 0) warp_sums[warp] = u;
        __syncthreads();
        if (threadIdx.x == 0)
            chunk_sums[c] = ((warp_sums[0] + warp_sums[1]) + (warp_sums[2] + warp_sums[3])) +
                            ((warp_sums[4] + warp_sums[5]) + (warp_sums[6] + warp_sums[7]));
        __syncthreads();
    }
    double total = 0.0;
    if (threadIdx.x == 0) {
        constexpr int kChunks = kGammaMaxPartials / 2048;
        double cs[kChunks];
#pragma unroll
        for (int c = 0; c < kChunks; ++c) cs[c] = (c < nchunks) ? chunk_sums[c] : 0.0;
#pragma unroll
        for (int w = 1; w < kChunks; w *= 2)
#pragma unroll
            for (int i = 0; i < kChunks; i += 2 * w) cs[i] = cs[i] + cs[i + w];
        total = cs[0];
    }
    return total;
}

// gamma: one CTA per tree node of kGammaBlock weights.  Warp w owns the 1024
// consecutive weights [node*8192 + 1024w, +1024) as eight 128-weight chunks;
// for chunk q lane l loads the float4 at 128q + 4l (coalesced), sums its four
// leaves, and a butterfly over the lanes completes the chunk's tree; the eight
// chunk sums, the eight warp sums and finally (in the last CTA to finish) the
// node partials are combined over the same pairwise tree.  ws->counter must
// be zero at launch.  gamma_out and sum_out (the fp64 sum itself) are
// optional; with neither, the node partials in ws are the result.
// SURV_M = 0: gamma over all weights; SURV_M = m (4 or 8): mask-then-quant,
// the sum over the kept |w| only (the group's keep mask from |w| as in
// pack_kernel; zeros at dropped positions keep the same tree) divided by
// `divisor` (the number of kept weights).
template <typename WT, int SURV_M>
__global__ void __launch_bounds__(256) gamma_kernel(const WT *__restrict__ W, int64_t count,
                                                    GammaWorkspace *ws, float *gamma_out, int n, int64_t divisor,
                                                    double *sum_out = nullptr)
{
    __shared__ double warp_sums[8];
    __shared__ double chunk_sums[kGammaMaxPartials / 2048];
    __shared__ int is_last;
    // the pack kernel may launch now: it only streams W before waiting for us
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t wbase = static_cast<int64_t>(blockIdx.x) * kGammaBlock + warp * 1024;
    float4 f[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {  // count % 4 == 0: a float4 is all in or all out
        const int64_t e = wbase + 128 * q + 4 * lane;
        f[q] = (e < count) ? load4(W, e) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if constexpr (SURV_M != 0) {
        // zero the dropped weights: a group of 4 is one lane's float4, a
        // group of 8 the float4s of lanes 2i and 2i + 1
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            uint32_t own[4] = {__float_as_uint(f[q].x) & 0x7fffffffu, __float_as_uint(f[q].y) & 0x7fffffffu,
                               __float_as_uint(f[q].z) & 0x7fffffffu, __float_as_uint(f[q].w) & 0x7fffffffu};
            uint32_t keep4;
            if constexpr (SURV_M == 4) {
                keep4 = keep_mask<4>(own, n);
            } else {
                uint32_t other[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) other[i] = __shfl_xor_sync(0xffffffffu, own[i], 1);
                const bool odd = lane & 1;
                uint32_t key[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    key[i] = odd ? other[i] : own[i];
                    key[4 + i] = odd ? own[i] : other[i];
                }
                const uint32_t k8 = keep_mask<8>(key, n);
                keep4 = odd ? (k8 >> 4) : (k8 & 0xfu);
            }
            if (!(keep4 & 1u)) f[q].x = 0.f;
            if (!(keep4 & 2u)) f[q].y = 0.f;
            if (!(keep4 & 4u)) f[q].z = 0.f;
            if (!(keep4 & 8u)) f[q].w = 0.f;
        }
    }
    double c[8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
        c[q] = (fabs(static_cast<double>(f[q].x)) + fabs(static_cast<double>(f[q].y))) +
               (fabs(static_cast<double>(f[q].z)) + fabs(static_cast<double>(f[q].w)));
    // chunk q's tree over the lanes (adjacent lanes first; a + b == b + a
    // exactly) as a reduce-scatter: at xor 1, 2, 4 each lane keeps half, a
    // quarter, then one of the chunks; xor 8 and 16 finish it.  Lane L then
    // holds chunk 4 (L & 1) + 2 (L >> 1 & 1) + (L >> 2 & 1), so the chunks'
    // pairwise tree ((c0 + c1) + (c2 + c3)) + ((c4 + c5) + (c6 + c7)) is the
    // butterfly xor 4, 2, 1 over lanes 0..7.
    const bool b0 = lane & 1, b1 = (lane >> 1) & 1, b2 = (lane >> 2) & 1;
    double r1[4], r2[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const double keep = b0 ? c[4 + i] : c[i], give = b0 ? c[i] : c[4 + i];
        r1[i] = keep + __shfl_xor_sync(0xffffffffu, give, 1);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const double keep = b1 ? r1[2 + i] : r1[i], give = b1 ? r1[i] : r1[2 + i];
        r2[i] = keep + __shfl_xor_sync(0xffffffffu, give, 2);
    }
    double t;
    {
        const double keep = b2 ? r2[1] : r2[0], give = b2 ? r2[0] : r2[1];
        t = keep + __shfl_xor_sync(0xffffffffu, give, 4);
    }
    t = t + __shfl_xor_sync(0xffffffffu, t, 8);
    t = t + __shfl_xor_sync(0xffffffffu, t, 16);
    t = t + __shfl_xor_sync(0xffffffffu, t, 4);
    t = t + __shfl_xor_sync(0xffffffffu, t, 2);
    t = t + __shfl_xor_sync(0xffffffffu, t, 1);
    if (lane == 0) warp_sums[warp] = t;
    __syncthreads();
    if (threadIdx.x == 0) {
        ws->partials[blockIdx.x] = ((warp_sums[0] + warp_sums[1]) + (warp_sums[2] + warp_sums[3])) +
                                   ((warp_sums[4] + warp_sums[5]) + (warp_sums[6] + warp_sums[7]));
        __threadfence();
        const uint32_t prev = atomicAdd(&ws->counter, 1u);
        is_last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    if (!gamma_out && !sum_out) return;  // node partials only (a column shard's first level)
    const double total = gamma_tree_finish(ws->partials, static_cast<int>(gridDim.x), warp_sums, chunk_sums);
    if (threadIdx.x == 0) {
        if (sum_out) *sum_out = total;
        if (gamma_out) {
            const double mean = divisor > 0 ? __ddiv_rn(total, static_cast<double>(divisor)) : 0.0;
            *gamma_out = __double2float_rn(mean);
        }
    }
}

// Combine the first-level node sums of every column shard (gathered in row
// order) over the same tree: gamma = fl32(tree(nodes) / divisor).  One CTA
// of 256 threads.
__global__ void __launch_bounds__(256) gamma_combine_kernel(const double *__restrict__ nodes, int nparts,
                                                            int64_t divisor, float *gamma_out)
{
    __shared__ double warp_sums[8];
    __shared__ double chunk_sums[kGammaMaxPartials / 2048];
    asm volatile("griddepcontrol.wait;" ::: "memory");  // the node sums may come from the previous kernel
    const double total = gamma_tree_finish(nodes, nparts, warp_sums, chunk_sums);
    if (threadIdx.x == 0) {
        const double mean = divisor > 0 ? __ddiv_rn(total, static_cast<double>(divisor)) : 0.0;
        *gamma_out = __double2float_rn(mean);
    }
}

// Keep mask of the n largest |W| of a group (lower index wins ties; keys are
// |W| bit patterns, ordered like the magnitudes).  Rank counting is the
// general case; when at most two weights are dropped (or at most two kept) a
// scan for the extreme element is cheaper and gives the same set:
//  * the element dropped first is the minimum under (key ascending, index
//    descending) -- a scan from the highest index with a strict `<`;
//  * the element kept first is the maximum under (key descending, index
//    ascending) -- a scan from index 0 with a strict `>`.
template <int M>
__device__ __forceinline__ uint32_t keep_mask(const uint32_t (&key)[M], int n)
{
    constexpr uint32_t kAll = (1u << M) - 1u;
    const int drop = M - n;
    if (drop <= 2 || n <= 2) {
        const bool by_drop = drop <= 2;
        const int picks = by_drop ? drop : n;
        uint32_t chosen = 0;
        uint32_t k[M];
#pragma unroll
        for (int i = 0; i < M; ++i)  // both forms stay below 2^31, under the sentinel
            k[i] = by_drop ? key[i] : 0x7fffffffu - key[i];  // max of key = min of (2^31 - 1 - key)
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            if (p >= picks) break;
            // minimum of k with ties to the higher index (drop) or the lower
            // index (keep: the complement reverses the key order, not the index order)
            int best = by_drop ? M - 1 : 0;
            uint32_t kb = k[best];
#pragma unroll
            for (int t = 1; t < M; ++t) {
                const int i = by_drop ? M - 1 - t : t;
                if (k[i] < kb) { kb = k[i]; best = i; }
            }
            chosen |= 1u << best;
#pragma unroll
            for (int i = 0; i < M; ++i)
                if (i == best) k[i] = 0xffffffffu;  // above every k: never picked again
        }
        return by_drop ? (kAll & ~chosen) : chosen;
    }
    // rank_i = #{ j : key_j > key_i  or  (key_j == key_i and j < i) }
    int rank[M];
#pragma unroll
    for (int i = 0; i < M; ++i) rank[i] = 0;
#pragma unroll
    for (int i = 0; i < M; ++i)
#pragma unroll
        for (int j = i + 1; j < M; ++j) {
            if (key[j] > key[i]) ++rank[i];  // j beats i only if strictly larger
            else ++rank[j];
        }
    uint32_t keep = 0;
#pragma unroll
    for (int i = 0; i < M; ++i) keep |= (rank[i] < n ? 1u : 0u) << i;
    return keep;
}

// Mask + ternarise one group of M weights given as fp32 bit patterns.
// Returns W_eff as M bytes (int8, little-endian in w0/w1) and the keep mask.
// Ternarise one group of M weights (fp32 bit patterns) under its keep mask.
// Returns W_eff as M bytes (int8, little-endian in w0/w1).
template <int M>
__device__ __forceinline__ void ternarise_group(const uint32_t (&bits)[M], uint32_t keep_bits,
                                                uint32_t thr_bits, uint32_t &w0, uint32_t &w1)
{
    uint32_t b[M];
#pragma unroll
    for (int i = 0; i < M; ++i) {
        // |w| >= threshold (both non-negative) and kept -> 0x01 or 0xff by sign
        const bool on = ((bits[i] & 0x7fffffffu) >= thr_bits) && ((keep_bits >> i) & 1u);
        b[i] = on ? ((bits[i] >> 31) ? 0xffu : 0x01u) : 0u;
    }
    w0 = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
    w1 = 0;
    if constexpr (M == 8) w1 = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
}

// 2-bit codes (w + 1) of the M bytes of W_eff held in w0/w1, weight i at bits 2i.
template <int M>
__device__ __forceinline__ uint32_t codes_of(uint32_t w0, uint32_t w1)
{
    uint32_t c = 0;
#pragma unroll
    for (int i = 0; i < M; ++i) {
        const uint32_t byte = ((i < 4 ? w0 : w1) >> (8 * (i & 3))) & 0xffu;
        // 0x00 -> 1, 0x01 -> 2, 0xff -> 0
        c |= ((byte + 1u) & 3u) << (2 * i);
    }
    return c;
}

template <int M>
__device__ __forceinline__ void store_group(const PackArgs &a, int32_t row, int32_t gi, uint32_t w0,
                                            uint32_t w1, uint32_t keep_bits)
{
    const PackOut &out = a.out;
    const int32_t gpr = a.cols / M;
    const int64_t row64 = row;
    if (out.i8) {
        int8_t *dst = out.i8 + row64 * a.cols + static_cast<int64_t>(gi) * M;
        if constexpr (M == 8) *reinterpret_cast<uint2 *>(dst) = make_uint2(w0, w1);
        else *reinterpret_cast<uint32_t *>(dst) = w0;
    }
    if (out.pk2 || out.nm_values) {
        const uint32_t codes = codes_of<M>(w0, w1);
        if (out.pk2) {
            uint8_t *prow = out.pk2 + row64 * out.pk2_stride;
            if constexpr (M == 8)
                *reinterpret_cast<uint16_t *>(prow + gi * 2) = static_cast<uint16_t>(codes);
            else
                prow[gi] = static_cast<uint8_t>(codes);
            if (gi == gpr - 1)
                for (int64_t b = a.cols / 4; b < out.pk2_stride; ++b) prow[b] = 0x55;
        }
        if (out.nm_values) {
            // kept codes, ascending position, 2 bits each, at bit offset gi*2n
            uint32_t kc = 0;
            int s = 0;
#pragma unroll
            for (int i = 0; i < M; ++i)
                if (keep_bits & (1u << i)) {
                    kc |= ((codes >> (2 * i)) & 3u) << (2 * s);
                    ++s;
                }
            // the buffer was preset to 0x55 (code 1 everywhere): xor turns each
            // written slot's 01 into the code
            const uint32_t delta = kc ^ (0x55555555u & ((1u << (2 * a.n)) - 1u));
            const int64_t bit = static_cast<int64_t>(gi) * 2 * a.n;
            uint32_t *wrow = reinterpret_cast<uint32_t *>(out.nm_values + row64 * out.nm_values_stride);
            const int64_t wi = bit >> 5;
            const int sh = static_cast<int>(bit & 31);
            const uint64_t d64 = static_cast<uint64_t>(delta) << sh;
            if (static_cast<uint32_t>(d64)) atomicXor(wrow + wi, static_cast<uint32_t>(d64));
            if (static_cast<uint32_t>(d64 >> 32)) atomicXor(wrow + wi + 1, static_cast<uint32_t>(d64 >> 32));
            uint8_t *brow = out.nm_bitmap + row64 * out.nm_bitmap_stride;
            if constexpr (M == 8) {
                brow[gi] = static_cast<uint8_t>(keep_bits);
            } else {
                // two 4-bit groups per byte; the bitmap was preset to 0
                const int64_t bb = static_cast<int64_t>(gi) * 4;
                atomicOr(reinterpret_cast<uint32_t *>(brow) + (bb >> 5), keep_bits << (bb & 31));
            }
        }
    }
}

// The re-mask statistics of one thread's 16 weights, in two parts: the
// small per-thread results are computed from the weights first (so the
// weights' registers are freed by the format stores), then stored and the
// counts reduced over the warp, then the CTA, and added to the counters with
// one atomic each (every thread of the CTA takes part in that second part).
template <int M>
struct ThreadStats {
    uint32_t keep16, flips, nz;
    uint32_t drop_max[16 / M];  // largest dropped |w| (as bits) per group
};

template <int M>
__device__ __forceinline__ ThreadStats<M> stats_of(const PackArgs &a, const uint32_t (&bits)[16 / M][M],
                                                   const uint32_t (&keep)[16 / M], uint32_t prev16)
{
    constexpr int kBatch = 16 / M;
    ThreadStats<M> r;
    r.keep16 = 0;
#pragma unroll
    for (int b = 0; b < kBatch; ++b) r.keep16 |= keep[b] << (b * M);
    r.flips = a.stats.prev_keep ? static_cast<uint32_t>(__popc((r.keep16 ^ prev16) & 0xffffu)) : 0u;
    r.nz = 0;
    if (a.stats.near_zero) {
        const uint32_t bound = near_zero_bound_bits(*a.gamma);
#pragma unroll
        for (int b = 0; b < kBatch; ++b)
#pragma unroll
            for (int i = 0; i < M; ++i) r.nz += ((bits[b][i] & 0x7fffffffu) < bound) ? 1u : 0u;
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
        uint32_t dm = 0u;
#pragma unroll
        for (int i = 0; i < M; ++i) {
            const uint32_t key = bits[b][i] & 0x7fffffffu;
            if (!((keep[b] >> i) & 1u) && key > dm) dm = key;
        }
        r.drop_max[b] = dm;
    }
    return r;
}

template <int M>
__device__ __forceinline__ void stats_finish(const PackArgs &a, bool active, int64_t e0, const ThreadStats<M> &r)
{
    uint32_t flips = 0, nz = 0;
    if (active) {
        const int32_t row = static_cast<int32_t>(__umul64hi(static_cast<uint64_t>(e0), a.inv_cols));
        const int32_t col0 = static_cast<int32_t>(e0 - static_cast<int64_t>(row) * a.cols);
        if (a.stats.keep)
            *reinterpret_cast<uint16_t *>(a.stats.keep + static_cast<int64_t>(row) * a.stats.keep_stride + col0 / 8) =
                static_cast<uint16_t>(r.keep16);
        if (a.stats.threshold) {
            float *t = a.stats.threshold + static_cast<int64_t>(row) * (a.cols / M) + col0 / M;
            if constexpr (M == 8) {
                *reinterpret_cast<uint2 *>(t) = make_uint2(r.drop_max[0], r.drop_max[1]);
            } else {
                *reinterpret_cast<uint4 *>(t) = make_uint4(r.drop_max[0], r.drop_max[1], r.drop_max[2], r.drop_max[3]);
            }
        }
        flips = r.flips;
        nz = r.nz;
    }
    if (!a.stats.flips && !a.stats.near_zero) return;  // uniform over the grid
    __shared__ uint32_t red[2][8];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        flips += __shfl_xor_sync(0xffffffffu, flips, off);
        nz += __shfl_xor_sync(0xffffffffu, nz, off);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        red[0][warp] = flips;
        red[1][warp] = nz;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long f = 0, z = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            f += red[0][w];
            z += red[1][w];
        }
        if (a.stats.flips && f) atomicAdd(a.stats.flips, f);
        if (a.stats.near_zero && z) atomicAdd(a.stats.near_zero, z);
    }
}

// SP24 form of four-group q of a thread's 16 weights: the group's kept
// positions (at most two) completed with its smallest positions not kept,
// i0 < i1; values W_eff[i0], W_eff[i1] go to value bytes 2q, 2q+1 and the
// nibble i0 | i1 << 2 to bits 4q of the thread's 16 metadata bits.
__device__ __forceinline__ void sp24_group(uint32_t wbytes, uint32_t keep4, int q, uint32_t (&vals)[2],
                                           uint32_t &meta)
{
    uint32_t sel = keep4 & 0xfu;
    if (__popc(sel) < 2) sel |= ~sel & (sel + 1u);  // lowest position not yet chosen
    if (__popc(sel) < 2) sel |= ~sel & (sel + 1u);
    const uint32_t i0 = static_cast<uint32_t>(__ffs(sel) - 1), i1 = static_cast<uint32_t>(31 - __clz(sel));
    const uint32_t v = ((wbytes >> (8 * i0)) & 0xffu) | (((wbytes >> (8 * i1)) & 0xffu) << 8);
    vals[q >> 1] |= v << (16 * (q & 1));
    meta |= (i0 | (i1 << 2)) << (4 * q);
}

// T24 code of one group of four W_eff bytes (int8 -1 / 0 / +1): 0 (no
// nonzero), 1 + 2p + s_p (one at p), 9 + 4k + 2 s_p + s_q (two, p < q, k the
// index of (p, q) in (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)); s = 1 for -1.
__device__ __forceinline__ uint32_t t24_code(uint32_t wbytes)
{
    uint32_t nz = 0u, neg = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t b = (wbytes >> (8 * i)) & 0xffu;
        nz |= (b != 0u ? 1u : 0u) << i;
        neg |= (b >> 7) << i;
    }
    if (nz == 0u) return 0u;
    const uint32_t p = static_cast<uint32_t>(__ffs(nz) - 1);
    if (__popc(nz) == 1) return 1u + 2u * p + ((neg >> p) & 1u);
    const uint32_t q = static_cast<uint32_t>(31 - __clz(nz));
    const uint32_t k = p * (7u - p) / 2u + (q - p - 1u);
    return 9u + 4u * k + 2u * ((neg >> p) & 1u) + ((neg >> q) & 1u);
}

// Mask + ternarise + pack: thread t of CTA c owns the 16 consecutive weights
// (two groups of 8 or four of 4) starting at (256 c + t) * 16.  Launched with
// programmatic dependent launch right behind gamma_kernel: W is loaded and the
// N:M keep masks (which need only |W|) are computed before waiting for
// gamma_kernel (which does not write W); gamma is read after.
// SP24: also write the 2:4 formats that were asked for, the sparse-MMA
// operand and the 6-bit T24 codes (a separate instantiation, so the other
// formats' kernel carries none of their registers).
// Ternarise and store every requested format of one thread's 16 weights.
template <int M, bool SP24>
__device__ __forceinline__ void pack_formats(const PackArgs &a, int64_t e0, const uint32_t (&bits)[16 / M][M],
                                             const uint32_t (&keep)[16 / M])
{
    constexpr int kBatch = 16 / M;
    const uint32_t thr_bits = __float_as_uint(ternary_threshold(*a.gamma));
    const int32_t row = static_cast<int32_t>(__umul64hi(static_cast<uint64_t>(e0), a.inv_cols));
    const int32_t col0 = static_cast<int32_t>(e0 - static_cast<int64_t>(row) * a.cols);  // 16 | K: same row
    uint32_t sp_vals[2] = {0u, 0u}, sp_meta = 0u, t_lo = 0u, t_hi = 0u;
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
        uint32_t w0, w1;
        ternarise_group<M>(bits[b], keep[b], thr_bits, w0, w1);
        store_group<M>(a, row, col0 / M + b, w0, w1, keep[b]);
        if constexpr (SP24) {
            // the thread's four groups of four, j = 0..3
            const int j0 = M == 4 ? b : 2 * b;
            if constexpr (M == 4) {
                sp24_group(w0, keep[b], b, sp_vals, sp_meta);
            } else {
                sp24_group(w0, keep[b], 2 * b, sp_vals, sp_meta);
                sp24_group(w1, keep[b] >> 4, 2 * b + 1, sp_vals, sp_meta);
            }
            const uint32_t c0 = t24_code(w0);
            t_lo |= (c0 & 15u) << (4 * j0);
            t_hi |= (c0 >> 4) << (2 * j0);
            if constexpr (M == 8) {
                const uint32_t c1 = t24_code(w1);
                t_lo |= (c1 & 15u) << (4 * (j0 + 1));
                t_hi |= (c1 >> 4) << (2 * (j0 + 1));
            }
        }
    }
    if constexpr (SP24) {
        if (a.out.t24_lo) {
            // 2 low-plane bytes and 1 high-plane byte per thread
            uint8_t *lrow = a.out.t24_lo + static_cast<int64_t>(row) * a.out.t24_lo_stride;
            uint8_t *hrow = a.out.t24_hi + static_cast<int64_t>(row) * a.out.t24_hi_stride;
            *reinterpret_cast<uint16_t *>(lrow + col0 / 8) = static_cast<uint16_t>(t_lo);
            hrow[col0 / 16] = static_cast<uint8_t>(t_hi);
            if (col0 + 16 == a.cols) {
                for (int64_t b = a.cols / 8; b < a.out.t24_lo_stride; ++b) lrow[b] = 0;
                for (int64_t b = a.cols / 16; b < a.out.t24_hi_stride; ++b) hrow[b] = 0;
            }
        }
    }
    if (SP24 && a.out.sp24_values) {
        // 8 value bytes and 16 metadata bits per thread; the thread that ends
        // a row also zeroes the row padding
        uint8_t *vrow = reinterpret_cast<uint8_t *>(a.out.sp24_values) + static_cast<int64_t>(row) * a.out.sp24_values_stride;
        uint8_t *mrow = a.out.sp24_meta + static_cast<int64_t>(row) * a.out.sp24_meta_stride;
        *reinterpret_cast<uint2 *>(vrow + col0 / 2) = make_uint2(sp_vals[0], sp_vals[1]);
        *reinterpret_cast<uint16_t *>(mrow + col0 / 8) = static_cast<uint16_t>(sp_meta);
        if (col0 + 16 == a.cols) {
            for (int64_t b = a.cols / 2; b < a.out.sp24_values_stride; ++b) vrow[b] = 0;
            for (int64_t b = a.cols / 8; b < a.out.sp24_meta_stride; ++b) mrow[b] = 0;
        }
    }
}

// STATS: also the re-mask statistics of PackStats (flip count, near-zero
// count, per-group threshold, keep bitmap).
// Compile-time options of pack_kernel (a bit mask, so each combination is
// its own kernel and the common one carries nothing of the others).
enum : int { kPackSp24 = 1, kPackStats = 2, kPackMaskQ = 4, kPackBf16 = 8 };

template <int M, int OPT>
__global__ void __launch_bounds__(256) pack_kernel(PackArgs a)
{
    constexpr bool SP24 = (OPT & kPackSp24) != 0;
    constexpr bool STATS = (OPT & kPackStats) != 0;
    constexpr bool MASKQ = (OPT & kPackMaskQ) != 0;
    using WT = typename std::conditional<(OPT & kPackBf16) != 0, uint16_t, float>::type;
    constexpr int kBatch = 16 / M;  // groups per thread
    const int64_t e0 = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) * 16;
    const bool active = e0 < a.count;  // count % 16 == 0: the 16 weights are all in or all out
    uint32_t bits[kBatch][M];
    uint32_t keep[kBatch];
    uint32_t prev16 = 0;        // previous step's keep bits of these 16 weights
    if constexpr (STATS) {
        // the previous bitmap was written before gamma_kernel started (which
        // is not launched early), so it may be read before the wait
        if (active && a.stats.prev_keep) {
            const int32_t prow = static_cast<int32_t>(__umul64hi(static_cast<uint64_t>(e0), a.inv_cols));
            const int32_t pcol = static_cast<int32_t>(e0 - static_cast<int64_t>(prow) * a.cols);
            prev16 = *reinterpret_cast<const uint16_t *>(a.stats.prev_keep + static_cast<int64_t>(prow) * a.stats.keep_stride +
                                                         pcol / 8);
        }
    }
    if (active) {
        float4 f[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) f[j] = load4(static_cast<const WT *>(a.W), e0 + 4 * j);
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            uint32_t key[M];
#pragma unroll
            for (int i = 0; i < M; ++i) {
                const int e = b * M + i;
                const float4 &v = f[e >> 2];
                const float x = (e & 3) == 0 ? v.x : (e & 3) == 1 ? v.y : (e & 3) == 2 ? v.z : v.w;
                bits[b][i] = __float_as_uint(x);
                key[i] = bits[b][i] & 0x7fffffffu;  // |W| ordered as integers; -0 ties +0
            }
            keep[b] = MASKQ ? 0u : keep_mask<M>(key, a.n);
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (MASKQ && active) {
        // ablation: the mask ranks |W_q| in {0, 1} (ties to the lower index),
        // so it needs gamma first
        const uint32_t thr = __float_as_uint(ternary_threshold(*a.gamma));
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            uint32_t key01[M];
#pragma unroll
            for (int i = 0; i < M; ++i) key01[i] = ((bits[b][i] & 0x7fffffffu) >= thr) ? 1u : 0u;
            keep[b] = keep_mask<M>(key01, a.n);
        }
    }
    if constexpr (STATS) {
        // every thread takes part in the statistics' CTA-wide reduction
        ThreadStats<M> st{};
        if (active) st = stats_of<M>(a, bits, keep, prev16);
        stats_finish<M>(a, active, e0, st);
    }
    if (!active) return;
    pack_formats<M, SP24>(a, e0, bits, keep);
}


// W_eff^T as bf16 from the int8 W_eff: in [rows, cols] int8 -> out [cols,
// rows] bf16 bits, through 64 x 64 shared-memory tiles.  rows, cols % 16 == 0.
__global__ void __launch_bounds__(256) transpose_i8_to_bf16_kernel(const int8_t *__restrict__ in,
                                                                   int32_t rows, int32_t cols,
                                                                   uint16_t *__restrict__ out)
{
    __shared__ int8_t tile[64][64 + 16];
    const int r0 = blockIdx.y * 64, c0 = blockIdx.x * 64;
    {
        const int r = threadIdx.x >> 2, cq = (threadIdx.x & 3) * 16;
        if (r0 + r < rows && c0 + cq < cols) {
            const uint4 v = *reinterpret_cast<const uint4 *>(in + static_cast<int64_t>(r0 + r) * cols + c0 + cq);
            *reinterpret_cast<uint4 *>(&tile[r][cq]) = v;
        }
    }
    __syncthreads();
#pragma unroll
    for (int rep = 0; rep < 2; ++rep) {
        const int idx = threadIdx.x + rep * 256;  // 64 out rows x 8 chunks of 8
        const int c = idx >> 3, rq = (idx & 7) * 8;
        if (c0 + c < cols && r0 + rq < rows) {
            uint32_t w[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const int8_t a = tile[rq + 2 * p][c], b = tile[rq + 2 * p + 1][c];
                const uint32_t ha = a == 0 ? 0u : (a > 0 ? 0x3f80u : 0xbf80u);
                const uint32_t hb = b == 0 ? 0u : (b > 0 ? 0x3f80u : 0xbf80u);
                w[p] = ha | (hb << 16);
            }
            *reinterpret_cast<uint4 *>(out + static_cast<int64_t>(c0 + c) * rows + r0 + rq) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

}  // namespace sbl
