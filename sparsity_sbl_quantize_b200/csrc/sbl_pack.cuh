// sbl_pack.cuh -- weight side of the Sparse-BitLinear layer on sm_100a:
//   * gamma: mean |W| (Sparse-BitNet summary, section 3.4, "Step 1: Compute
//     the Rescaling Factor"), summed in fp64 over the pairwise tree of the
//     flat row-major order, so the result does not depend on the grid;
//   * the fused N:M mask ("N:M Mask Generation"), ternarisation ("Step 2:
//     Rescale and RoundClip") and mask application ("Composition Order"),
//     writing the packed formats in one pass over W.
#pragma once

#include "sbl_device.cuh"

namespace sbl {

// Elements per first-level partial of the gamma tree (a tree node: the
// partial of block j covers [j * kGammaBlock, (j + 1) * kGammaBlock)).
constexpr int kGammaBlock = 16384;
// Leaves of the second-level tree: 256 threads x 64 partials each.
constexpr int kGammaMaxPartials = 16384;

struct GammaWorkspace {
    double partials[kGammaMaxPartials];
    uint32_t counter;       // blocks finished (reset by the last block)
    float threshold;        // smallest fp32 t with |w| >= t  <=>  W_q != 0
    uint32_t pad[2];
};

// Pairwise sum of 16 consecutive leaves held by one thread.
__device__ __forceinline__ double tree16(double (&v)[16])
{
#pragma unroll
    for (int w = 1; w < 16; w *= 2)
#pragma unroll
        for (int i = 0; i < 16; i += 2 * w) v[i] = v[i] + v[i + w];
    return v[0];
}

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

// One block per kGammaBlock elements, 256 threads; the last block to finish
// combines the partials and writes gamma and the ternary threshold.
// Requires count % 16 == 0 and count <= kGammaBlock * kGammaMaxPartials.
__global__ void __launch_bounds__(256) gamma_kernel(const float *__restrict__ W, int64_t count,
                                                    GammaWorkspace *ws, float *gamma_out)
{
    __shared__ double warp_sums[8];
    __shared__ double thread_sums[256];
    __shared__ int is_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t base = static_cast<int64_t>(blockIdx.x) * kGammaBlock + warp * 2048;

    double sub[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const int64_t e = base + s * 512 + lane * 16;
        double v[16];
        if (e < count) {  // count % 16 == 0: the 16 leaves are all in range
            const float4 *p = reinterpret_cast<const float4 *>(W + e);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 f = __ldg(p + q);
                v[4 * q + 0] = fabs(static_cast<double>(f.x));
                v[4 * q + 1] = fabs(static_cast<double>(f.y));
                v[4 * q + 2] = fabs(static_cast<double>(f.z));
                v[4 * q + 3] = fabs(static_cast<double>(f.w));
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = 0.0;
        }
        double t = tree16(v);
        // butterfly: after the step with offset `off`, lane 0 holds the tree
        // over lanes [0, 2*off)
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) t = t + __shfl_xor_sync(0xffffffffu, t, off);
        sub[s] = t;
    }
    if (lane == 0) warp_sums[warp] = (sub[0] + sub[1]) + (sub[2] + sub[3]);
    __syncthreads();
    if (threadIdx.x == 0) {
        const double b = ((warp_sums[0] + warp_sums[1]) + (warp_sums[2] + warp_sums[3])) +
                         ((warp_sums[4] + warp_sums[5]) + (warp_sums[6] + warp_sums[7]));
        ws->partials[blockIdx.x] = b;
        __threadfence();
        const uint32_t prev = atomicAdd(&ws->counter, 1u);
        is_last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    // Second level: thread i combines partials [64 i, 64 i + 64) (a tree node),
    // then a shared-memory tree over the 256 thread sums.
    const int nparts = static_cast<int>(gridDim.x);
    double acc8[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        double v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int j = threadIdx.x * 64 + c * 8 + i;
            v[i] = (j < nparts) ? __ldcg(&ws->partials[j]) : 0.0;
        }
        acc8[c] = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
    }
    thread_sums[threadIdx.x] = ((acc8[0] + acc8[1]) + (acc8[2] + acc8[3])) +
                               ((acc8[4] + acc8[5]) + (acc8[6] + acc8[7]));
    __syncthreads();
    for (int stride = 1; stride < 256; stride *= 2) {
        const int i = threadIdx.x * 2 * stride;
        if (i < 256) thread_sums[i] = thread_sums[i] + thread_sums[i + stride];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const double mean = __ddiv_rn(thread_sums[0], static_cast<double>(count));
        const float g = __double2float_rn(mean);
        *gamma_out = g;
        ws->threshold = ternary_threshold(g);
        ws->counter = 0u;
    }
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
};

// One thread per group of M consecutive weights of a row.  Each CTA takes a
// contiguous range of groups, so row/column follow from one division per
// thread plus increments.
template <int M>
__global__ void __launch_bounds__(256) pack_kernel(const float *__restrict__ W, int32_t rows,
                                                   int32_t cols, int32_t n,
                                                   const GammaWorkspace *__restrict__ ws,
                                                   PackOut out, int64_t groups_per_cta)
{
    const float thr = ws->threshold;
    const uint32_t thr_bits = __float_as_uint(thr);
    const int32_t gpr = cols / M;  // groups per row
    const int64_t total = static_cast<int64_t>(rows) * gpr;
    const int64_t g_begin = static_cast<int64_t>(blockIdx.x) * groups_per_cta;
    const int64_t g_end = min(total, g_begin + groups_per_cta);
    int64_t g = g_begin + threadIdx.x;
    if (g >= g_end) return;
    int32_t row = static_cast<int32_t>(g / gpr);
    int32_t gi = static_cast<int32_t>(g - static_cast<int64_t>(row) * gpr);

    for (; g < g_end; g += blockDim.x) {
        const float *src = W + static_cast<int64_t>(row) * cols + static_cast<int64_t>(gi) * M;
        uint32_t bits[M];
#pragma unroll
        for (int q = 0; q < M / 4; ++q) {
            const float4 f = __ldg(reinterpret_cast<const float4 *>(src) + q);
            bits[4 * q + 0] = __float_as_uint(f.x);
            bits[4 * q + 1] = __float_as_uint(f.y);
            bits[4 * q + 2] = __float_as_uint(f.z);
            bits[4 * q + 3] = __float_as_uint(f.w);
        }
        // |W| as ordered integers (sign bit cleared; -0 and +0 tie).
        uint32_t key[M];
#pragma unroll
        for (int i = 0; i < M; ++i) key[i] = bits[i] & 0x7fffffffu;
        // rank_i = #{ j : key_j > key_i  or  (key_j == key_i and j < i) }
        int rank[M];
#pragma unroll
        for (int i = 0; i < M; ++i) rank[i] = 0;
#pragma unroll
        for (int i = 0; i < M; ++i)
#pragma unroll
            for (int j = i + 1; j < M; ++j) {
                const int jb = key[j] > key[i];  // j beats i only if strictly larger
                rank[i] += jb;
                rank[j] += 1 - jb;
            }
        int8_t weff[M];
        uint32_t keep_bits = 0;
#pragma unroll
        for (int i = 0; i < M; ++i) {
            const bool keep = rank[i] < n;
            const bool nz = key[i] >= thr_bits;  // |w| >= threshold (both non-negative)
            const int8_t t = nz ? ((bits[i] >> 31) ? int8_t(-1) : int8_t(1)) : int8_t(0);
            weff[i] = keep ? t : int8_t(0);
            keep_bits |= (keep ? 1u : 0u) << i;
        }
        const int64_t row64 = row;
        if (out.i8) {
            int8_t *dst = out.i8 + row64 * cols + static_cast<int64_t>(gi) * M;
            uint32_t w0 = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) w0 |= (static_cast<uint32_t>(weff[i]) & 0xffu) << (8 * i);
            if constexpr (M == 8) {
                uint32_t w1 = 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) w1 |= (static_cast<uint32_t>(weff[4 + i]) & 0xffu) << (8 * i);
                *reinterpret_cast<uint2 *>(dst) = make_uint2(w0, w1);
            } else {
                *reinterpret_cast<uint32_t *>(dst) = w0;
            }
        }
        uint32_t codes = 0;  // 2-bit code w + 1 of weight i at bits 2i
#pragma unroll
        for (int i = 0; i < M; ++i) codes |= static_cast<uint32_t>(weff[i] + 1) << (2 * i);
        if (out.pk2) {
            uint8_t *prow = out.pk2 + row64 * out.pk2_stride;
            if constexpr (M == 8)
                *reinterpret_cast<uint16_t *>(prow + gi * 2) = static_cast<uint16_t>(codes);
            else
                prow[gi] = static_cast<uint8_t>(codes);
            if (gi == gpr - 1)
                for (int64_t b = cols / 4; b < out.pk2_stride; ++b) prow[b] = 0x55;
        }
        if (out.nm_values) {
            // kept codes, ascending position, 2 bits each, at bit offset gi*2n
            uint32_t kc = 0;
            int s = 0;
#pragma unroll
            for (int i = 0; i < M; ++i)
                if (keep_bits & (1u << i)) {
                    kc |= static_cast<uint32_t>(weff[i] + 1) << (2 * s);
                    ++s;
                }
            // the buffer was preset to 0x55 (code 1 everywhere): xor turns each
            // written slot's 01 into the code
            const uint32_t delta = kc ^ (0x55555555u & ((1u << (2 * n)) - 1u));
            const int64_t bit = static_cast<int64_t>(gi) * 2 * n;
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
        gi += blockDim.x;
        while (gi >= gpr) {
            gi -= gpr;
            ++row;
        }
    }
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
