// sbl_act.cuh -- activation side of the Sparse-BitLinear layer on sm_100a.
//   * per-token absmax int8 quantisation (BitNet b1.58 2B4T summary, section
//     3.4, "Activation Quantization: Per-Token Absmax to 8-Bit Integers";
//     Sparse-BitNet summary, activation quantization equation): one row of X
//     is read once into registers, reduced to max|x|, then scaled, rounded
//     half-to-even and stored as int8 with d_t = max|x| / 127;
//   * the operand preparation of the Dual-STE backward: dY * d_t * 2^s as
//     fp16 transposed to [O, T] (2^s a power of two chosen per call from the
//     largest |dY * d_t|, so that fp16's narrow range holds the products of
//     gradients of any scale), and the int8 activations as fp16 transposed
//     to [K, T], so both dW operands are K-major for the tensor cores.
#pragma once

#include <cuda_fp16.h>

#include "sbl_device.cuh"

namespace sbl {

constexpr int kActMaxChunks = 8;  // 16-byte chunks (8 bf16) per thread

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Round-half-even of |v| < 2^22 by the fp32 adder: fl(v + 1.5 2^23) has ulp 1
// and lies in [2^23, 2^24), so its bits are 0x4B400000 + rint(v), and the low
// byte is rint(v) as an int8 bit pattern when rint(v) is in [-128, 127].  The
// quantiser's products satisfy |fl32(x fl32(127 / a))| <= 127 (1 + 2^-24) for
// |x| <= a, so rint lies in [-127, 127] and the clamp to [-128, 127] never
// binds; one FADD replaces the float-to-int conversion.
__device__ __forceinline__ uint32_t rne_byte(float v)
{
    return __float_as_uint(__fadd_rn(v, 12582912.0f));
}

// Four int8 codes sat8(rint(fl32(x r))) packed LSB first.
__device__ __forceinline__ uint32_t quant4(float a, float b, float c, float d, float r)
{
    const uint32_t q0 = rne_byte(__fmul_rn(a, r)), q1 = rne_byte(__fmul_rn(b, r));
    const uint32_t q2 = rne_byte(__fmul_rn(c, r)), q3 = rne_byte(__fmul_rn(d, r));
    uint32_t lo, hi, w;
    asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(lo) : "r"(q0), "r"(q1));
    asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(hi) : "r"(q2), "r"(q3));
    asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(w) : "r"(lo), "r"(hi));
    return w;
}

// RT threads per token row; 256 / RT rows per CTA (RT <= 256) or one row per
// CTA of RT threads (RT > 256).  Thread i of a row owns the 16-byte chunks
// i, i + RT, ... (at most kActMaxChunks), so loads and stores are coalesced.
template <int RT>
__global__ void __launch_bounds__(RT > 256 ? RT : 256)
    act_quant_kernel(const uint16_t *__restrict__ X, int32_t T, int32_t K, int8_t *__restrict__ Xq,
                     float *__restrict__ d)
{
    constexpr int kRowsPerCta = RT >= 256 ? 1 : 256 / RT;
    constexpr int kWarpsPerRow = RT / 32 > 0 ? RT / 32 : 1;
    __shared__ float red[kRowsPerCta][kWarpsPerRow];
    const int sub = threadIdx.x / RT, lt = threadIdx.x % RT;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + sub;
    // programmatic dependent launch: X may come from the previous kernel
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const bool active = row < T;
    const int chunks = K / 8;

    uint4 v[kActMaxChunks];
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < kActMaxChunks; ++c) {
        const int ci = lt + c * RT;
        if (active && ci < chunks) {
            v[c] = __ldg(reinterpret_cast<const uint4 *>(X + row * K) + ci);
            const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
                amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (kWarpsPerRow > 1) {
        if ((lt & 31) == 0) red[sub][lt >> 5] = amax;
        __syncthreads();
        amax = red[sub][0];
#pragma unroll
        for (int w = 1; w < kWarpsPerRow; ++w) amax = fmaxf(amax, red[sub][w]);
    }
    if (!active) return;
    const bool zero = !(amax > 0.0f);
    const float r = zero ? 0.0f : __fdiv_rn(127.0f, amax);
#pragma unroll
    for (int c = 0; c < kActMaxChunks; ++c) {
        const int ci = lt + c * RT;
        if (ci < chunks) {
            uint2 out = make_uint2(0u, 0u);
            if (!zero) {
                out.x = quant4(bf16_lo(v[c].x), bf16_hi(v[c].x), bf16_lo(v[c].y), bf16_hi(v[c].y), r);
                out.y = quant4(bf16_lo(v[c].z), bf16_hi(v[c].z), bf16_lo(v[c].w), bf16_hi(v[c].w), r);
            }
            reinterpret_cast<uint2 *>(Xq + row * K)[ci] = out;
        }
    }
    if (lt == 0) d[row] = zero ? 0.0f : __fdiv_rn(amax, 127.0f);
}

// u = fl32(fl32(x * r) * g) of one 8-element chunk (g: bf16 gains or none)
__device__ __forceinline__ void norm_chunk(const uint4 &v, const uint16_t *__restrict__ g, int ci, int chunks,
                                           float r, float (&u)[8])
{
    const uint4 gv = (g && ci < chunks) ? __ldg(reinterpret_cast<const uint4 *>(g) + ci) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        u[2 * i] = __fmul_rn(bf16_lo(w[i]), r);
        u[2 * i + 1] = __fmul_rn(bf16_hi(w[i]), r);
        if (g) {
            u[2 * i] = __fmul_rn(u[2 * i], bf16_lo(gw[i]));
            u[2 * i + 1] = __fmul_rn(u[2 * i + 1], bf16_hi(gw[i]));
        }
    }
}

// RMSNorm fused with the quantiser (the norm before Q_a in forward step 1 of
// the Sparse-BitNet summary): per row, S = sum of x_k^2 in fp64 over the
// pairwise tree of the row in flat order, r = fl32(1 / sqrt(S / K + eps)),
// u_k = fl32(fl32(x_k * r) * g_k) (g: bf16 gains, none = 1), then the
// absmax int8 quantisation of u.
//
// That tree equals the tree of the row padded with +0.0 to 64 RT elements (a
// sum with +0.0 is exact), so it is assembled from aligned subtrees of the
// layout of the plain quantiser: thread lt of a row holds the 8-element
// chunks lt + c RT (slot c < 8; coalesced loads).  Slot c of warp w is the
// aligned 256-element block of chunks c RT + 32 w .. + 31, and slot c of the
// row the aligned block c RT .. (c + 1) RT - 1.  Each chunk is an 8-leaf tree;
// a reduce-scatter over lanes (xor 1, 2, 4: adjacent lanes first, each lane
// keeping half, then a quarter, then one of its slot sums) and two
// butterflies (xor 8, 16) leave in lane L the warp's sum of slot
// 4 (L & 1) + 2 (L >> 1 & 1) + (L >> 2 & 1); the row's first warp then adds
// the warps of each slot pairwise and the slots pairwise.  Every addition
// joins two adjacent aligned subtrees (a + b == b + a exactly).
template <int RT>
__global__ void __launch_bounds__(RT > 256 ? RT : 256, RT > 256 ? 1 : 3)
    act_norm_quant_kernel(const uint16_t *__restrict__ X, int32_t T, int32_t K, const uint16_t *__restrict__ g,
                          float eps, int8_t *__restrict__ Xq, float *__restrict__ d)
{
    static_assert(RT >= 32 && (RT & (RT - 1)) == 0, "rows are whole warps, a power of two");
    constexpr int kRowsPerCta = RT >= 256 ? 1 : 256 / RT;
    constexpr int W = RT / 32;                        // warps per row
    constexpr int H = (8 * W + 31) / 32;              // (slot, warp) sums per lane of the combining warp
    __shared__ double wsum[kRowsPerCta][8 * W];       // [slot][warp]
    __shared__ float wmax[kRowsPerCta][W];
    __shared__ float rsh[kRowsPerCta];
    const int sub = threadIdx.x / RT, lt = threadIdx.x % RT;
    const int wr = lt >> 5, lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + sub;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const bool active = row < T;
    const int chunks = K / 8;

    uint4 v[kActMaxChunks];
#pragma unroll
    for (int c = 0; c < kActMaxChunks; ++c) {
        const int ci = lt + c * RT;
        v[c] = make_uint4(0u, 0u, 0u, 0u);
        if (active && ci < chunks) v[c] = __ldg(reinterpret_cast<const uint4 *>(X + row * K) + ci);
    }
    double cs[kActMaxChunks];
#pragma unroll
    for (int c = 0; c < kActMaxChunks; ++c) {
        const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
        double sq[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const double lo = static_cast<double>(bf16_lo(w[i])), hi = static_cast<double>(bf16_hi(w[i]));
            sq[2 * i] = lo * lo;  // exact: a bf16 square has at most 16 significant bits
            sq[2 * i + 1] = hi * hi;
        }
        cs[c] = ((sq[0] + sq[1]) + (sq[2] + sq[3])) + ((sq[4] + sq[5]) + (sq[6] + sq[7]));
    }
    // reduce-scatter over the lanes: keep slots 4 b0 .. 4 b0 + 3, then two of
    // them, then one
    const bool b0 = lane & 1, b1 = (lane >> 1) & 1, b2 = (lane >> 2) & 1;
    double r1[4], r2[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const double keep = b0 ? cs[4 + i] : cs[i], give = b0 ? cs[i] : cs[4 + i];
        r1[i] = keep + __shfl_xor_sync(0xffffffffu, give, 1);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const double keep = b1 ? r1[2 + i] : r1[i], give = b1 ? r1[i] : r1[2 + i];
        r2[i] = keep + __shfl_xor_sync(0xffffffffu, give, 2);
    }
    double r3;
    {
        const double keep = b2 ? r2[1] : r2[0], give = b2 ? r2[0] : r2[1];
        r3 = keep + __shfl_xor_sync(0xffffffffu, give, 4);
    }
    r3 = r3 + __shfl_xor_sync(0xffffffffu, r3, 8);
    r3 = r3 + __shfl_xor_sync(0xffffffffu, r3, 16);
    if (lane < 8) wsum[sub][(4 * b0 + 2 * b1 + b2) * W + wr] = r3;
    __syncthreads();
    if (wr == 0) {
        // value i = h 32 + lane is (slot i / W, warp i % W): warps pairwise
        // within each slot (xor < W), slots pairwise across the lane groups
        // (xor W .. 16; lanes past 8 W hold +0.0), then the H blocks pairwise
        double x[H];
#pragma unroll
        for (int h = 0; h < H; ++h) {
            const int i = h * 32 + lane;
            x[h] = i < 8 * W ? wsum[sub][i] : 0.0;
        }
#pragma unroll
        for (int off = 1; off < 32; off <<= 1)
#pragma unroll
            for (int h = 0; h < H; ++h) x[h] = x[h] + __shfl_xor_sync(0xffffffffu, x[h], off);
#pragma unroll
        for (int step = 1; step < H; step *= 2)
#pragma unroll
            for (int h = 0; h < H; h += 2 * step) x[h] = x[h] + x[h + step];
        if (lane == 0)
            rsh[sub] = __double2float_rn(__ddiv_rn(
                1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(x[0], static_cast<double>(K)), static_cast<double>(eps)))));
    }
    __syncthreads();
    const float r = rsh[sub];

    // u = fl32(fl32(x * r) * g), computed from the held x in both passes:
    // max|u| over the row, then the quantised stores
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < kActMaxChunks; ++c) {
        float u[8];
        norm_chunk(v[c], g, lt + c * RT, chunks, r, u);
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(u[i]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane == 0) wmax[sub][wr] = amax;
    __syncthreads();
    amax = wmax[sub][0];
#pragma unroll
    for (int w = 1; w < W; ++w) amax = fmaxf(amax, wmax[sub][w]);
    if (!active) return;
    const bool zero = !(amax > 0.0f);
    const float rq = zero ? 0.0f : __fdiv_rn(127.0f, amax);
#pragma unroll
    for (int c = 0; c < kActMaxChunks; ++c) {
        const int ci = lt + c * RT;
        if (ci >= chunks) continue;
        uint2 out = make_uint2(0u, 0u);
        if (!zero) {
            float u[8];
            norm_chunk(v[c], g, ci, chunks, r, u);
            out.x = quant4(u[0], u[1], u[2], u[3], rq);
            out.y = quant4(u[4], u[5], u[6], u[7], rq);
        }
        reinterpret_cast<uint2 *>(Xq + row * K)[ci] = out;
    }
    if (lt == 0) d[row] = zero ? 0.0f : __fdiv_rn(amax, 127.0f);
}

// The dW operand's power-of-two prescale.  grad_absmax_kernel leaves in *m the
// fp32 bits of M = max over (t, o) of |fl32(dY[t, o] * d_t)| (computed per row
// as fl32(max_o |dY[t, o]| * |d_t|), the same value since rounding is
// monotone); *m must be 0 before the launch.  From M, s is chosen so that
// M * 2^s lies in [2^14, 2^15): the largest product then sits in fp16's top
// binade with room for rounding (fp16 ends at 65504), and products down to
// 2^-29 M stay fp16 normals.  M == 0 gives s = 0; s is clamped to [-126, 126]
// so that 2^s and 2^-s are fp32 normals, which makes both scalings exact.
__device__ __forceinline__ int grad_prescale_exponent(uint32_t m_bits)
{
    if (m_bits == 0u) return 0;
    const int e = static_cast<int>(m_bits >> 23);  // biased exponent; 0 for fp32 subnormals
    const int s = 141 - (e > 0 ? e : 1);           // M in [2^(e-127), 2^(e-126)) -> M 2^s in [2^14, 2^15)
    return s < -126 ? -126 : (s > 126 ? 126 : s);
}

__device__ __forceinline__ float pow2f(int s) { return __uint_as_float(static_cast<uint32_t>(s + 127) << 23); }

// One warp per row of dY [T, O] (bf16 bits, O % 8 == 0): the row's largest
// |dY| as bf16 bits (|x| of a finite bf16 orders like its bits & 0x7fff),
// times |d_t|, reduced over the CTA, then one atomicMax on the fp32 bits of
// the non-negative result.
__global__ void __launch_bounds__(256, 4) grad_absmax_kernel(const uint16_t *__restrict__ dY,
                                                          const float *__restrict__ d, int32_t T, int32_t O,
                                                          uint32_t *__restrict__ m)
{
    __shared__ uint32_t red[8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int chunks = O / 8;
    uint32_t best = 0u;
    for (int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + warp; row < T; row += static_cast<int64_t>(gridDim.x) * 8) {
        const uint4 *p = reinterpret_cast<const uint4 *>(dY + row * O);
        uint32_t mx = 0u;  // two 16-bit maxima, one per half
        int c = lane;
        auto absmax8 = [](const uint4 &a) {
            return __vmaxu2(__vmaxu2(a.x & 0x7fff7fffu, a.y & 0x7fff7fffu),
                            __vmaxu2(a.z & 0x7fff7fffu, a.w & 0x7fff7fffu));
        };
        for (; c + 96 < chunks; c += 128) {
            const uint4 a = __ldg(p + c), b = __ldg(p + c + 32), e = __ldg(p + c + 64), f = __ldg(p + c + 96);
            mx = __vmaxu2(mx, __vmaxu2(__vmaxu2(absmax8(a), absmax8(b)), __vmaxu2(absmax8(e), absmax8(f))));
        }
        for (; c < chunks; c += 32) mx = __vmaxu2(mx, absmax8(__ldg(p + c)));
        // the sign bit of each half is cleared before every max, so the maxima
        // compare magnitudes only
        uint32_t h = max(mx & 0xffffu, mx >> 16);
        h = __reduce_max_sync(0xffffffffu, h);
        const float v = __fmul_rn(__uint_as_float(h << 16), fabsf(d[row]));
        best = max(best, __float_as_uint(v));
    }
    if (lane == 0) red[warp] = best;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = red[0];
#pragma unroll
        for (int w = 1; w < 8; ++w) b = max(b, red[w]);
        if (b) atomicMax(m, b);
    }
}

// out[c, r] = fp16(conv(in[r, c])) for r < rows, c < cols; out has row stride
// ld_out >= rows, and out[c, r] = 0 for rows <= r < ld_out (padding).
// Mode 0: in is bf16 bits, value = fl32(fl32(bf16 * scale[r]) * 2^s) rounded
//         to fp16, with s = grad_prescale_exponent(*pre) (the bits
//         grad_absmax_kernel left); block (0, 0) stores 2^-s to *inv_pre for
//         the GEMM epilogue that undoes the prescale.
// Mode 1: in is int8, value = fp16(in) (exact).
// 64 x 64 tiles through shared memory; cols % 16 == 0.
template <int MODE>
__global__ void __launch_bounds__(256) transpose_to_f16_kernel(const void *__restrict__ in,
                                                               int32_t rows, int32_t cols,
                                                               const float *__restrict__ scale,
                                                               const uint32_t *__restrict__ pre,
                                                               float *__restrict__ inv_pre,
                                                               __half *__restrict__ out,
                                                               int64_t ld_out)
{
    __shared__ float tile[64][65];
    const int r0 = blockIdx.y * 64, c0 = blockIdx.x * 64;
    float factor = 1.0f;
    if (MODE == 0) {
        const int s = grad_prescale_exponent(*pre);
        factor = pow2f(s);
        if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *inv_pre = pow2f(-s);
    }
    // load: 64 rows x 64 columns, 16 consecutive columns per thread-quarter
    for (int idx = threadIdx.x; idx < 64 * 4; idx += 256) {
        const int r = idx >> 2, cq = (idx & 3) * 16;
        const int gr = r0 + r, gc = c0 + cq;
        float vals[16];
        if (gr < rows && gc < cols) {
            if (MODE == 0) {
                const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(in) +
                                                                  static_cast<int64_t>(gr) * cols + gc);
                const float s = scale[gr];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint4 q = __ldg(p + h);
                    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        vals[8 * h + 2 * i] = __fmul_rn(__fmul_rn(bf16_lo(w[i]), s), factor);
                        vals[8 * h + 2 * i + 1] = __fmul_rn(__fmul_rn(bf16_hi(w[i]), s), factor);
                    }
                }
            } else {
                const uint4 q = __ldg(reinterpret_cast<const uint4 *>(static_cast<const int8_t *>(in) +
                                                                       static_cast<int64_t>(gr) * cols + gc));
                const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    vals[i] = static_cast<float>(static_cast<int8_t>((w[i >> 2] >> (8 * (i & 3))) & 0xffu));
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) vals[i] = 0.0f;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) tile[r][cq + i] = vals[i];
    }
    __syncthreads();
    // store: 64 output rows (columns of in) x 64 entries, 8 per thread-chunk
    for (int idx = threadIdx.x; idx < 64 * 8; idx += 256) {
        const int c = idx >> 3, rq = (idx & 7) * 8;
        const int gc = c0 + c, gr = r0 + rq;
        if (gc < cols && gr < ld_out) {
            uint32_t w[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const __half2 h2 = __floats2half2_rn(tile[rq + 2 * p][c], tile[rq + 2 * p + 1][c]);
                w[p] = *reinterpret_cast<const uint32_t *>(&h2);
            }
            *reinterpret_cast<uint4 *>(out + static_cast<int64_t>(gc) * ld_out + gr) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

}  // namespace sbl
