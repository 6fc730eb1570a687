// sbl_decode.cuh -- decode-time Sparse-BitLinear forward (T <= 16 tokens) that
// streams the 2-bit PK2 weight codes at HBM rate.
//
// The weights stay packed (four ternaries per byte, the storage of the BitNet
// b1.58 2B4T summary, "Inference Implementation: GPU") and go from HBM
// straight into registers, where the int8 tensor-core path of mma.sync
// consumes them:
//  * a 32-bit PK2 word holds codes c = w + 1 of 16 consecutive weights;
//    (word >> 2j) & 0x03030303 is the four codes of positions j, j+4, j+8,
//    j+12 as four u8 values - two ALU ops for four weights;
//  * every lane transposes its own 16-byte activation groups as 4 x 4 byte
//    matrices (prmt), so word j of a transposed group holds the activations
//    of the same four positions;
//  * sum_k c * x = sum_k w * x + sum_k x, so the kernel subtracts the
//    activation column sum to get the exact int32 accumulator.
// The order in which the MMA visits K is a permutation of 0..K-1 that both
// operands share; integer sums do not depend on it.
//
// Work split: a CTA owns 16 output rows (one m16 tile) per row group and the
// group's 8 warps take the 256-weight K chunks of those rows round-robin.
// Each warp issues the loads of all its chunks (up to CPW per round) before
// waiting on the previous kernel on the stream, so weights stream while that
// kernel finishes; there is no shared-memory staging of weights and no
// cluster.  The kernel also lets the next kernel launch as soon as it starts,
// so that kernel's weights stream during this one's arithmetic.  The warps'
// int32 partials meet in shared memory (exact) and one thread per (token,
// row) dequantises y = fl32(fl32(acc) * fl32(gamma * d_t)).
//
// Fused variant (FUSE): the input is the bf16 activation X itself (small:
// T K <= 8192).  After the wait every CTA loads X in one pass into registers,
// quantises it per token (absmax int8, the quantiser of the activation
// kernel) into shared memory, and CTA 0 also stores Xq and d; the MMA loop
// then reads the activations from shared memory.  One launch per layer
// instead of two.
#pragma once

#include <cuda_bf16.h>

#include "sbl_act.cuh"
#include "sbl_device.cuh"

namespace sbl {

constexpr int kDecRows = 16;        // output rows per CTA
constexpr int kDecMaxTokens = 16;
constexpr int kDecKUnit = 64;       // K must be a multiple of 64 (16 PK2 bytes)
constexpr int kDecChunk = 256;      // weights of one row in a warp's K chunk
constexpr int kDecPartStride = 20;  // padded token row of the partial sums

struct DecodeArgs {
    const uint8_t *pk2;   // PK2 codes (T24 variant: the low plane of the group codes)
    int64_t pk2_stride;   // bytes per packed row
    const int8_t *xq;     // [T, K]
    const float *d;       // [T]
    const float *gamma;   // device scalar
    void *out;            // [T, O] bf16 bits or fp32
    int32_t out_fp32;
    int32_t *acc_out;     // optional [T, O] int32
    int32_t relu2;        // output epilogue: v = max(v, 0)^2 ...
    const uint16_t *residual;  // ... then v = v + residual[t, o] (bf16 [T, O]; nullptr: none)
    int32_t T, K, O;
    int32_t chunks;       // ceil(K / 256)
    // fused variant only
    union {
        const uint16_t *x;       // bf16 activations [T, K]
        const uint8_t *t24_hi;   // T24 variant: the high plane (pk2 holds the low plane)
    };
    int8_t *xq_out;       // Q_a(x) [T, K], stored by CTA 0 (nullptr: not stored)
    float *d_out;         // d_t [T], stored by CTA 0 (nullptr: not stored)
    union {
        int32_t xs_stride;      // bytes per token row of the shared int8 copy (K + 16)
        int32_t t24_hi_stride;  // T24 variant: bytes per row of the high plane
    };
};

// dynamic shared memory of the fused variant: the int8 activations [T][K + 16]
constexpr int kDecXsPad = 16;
// 16-byte groups of X per thread of the fused prologue (T K <= 8 x 4 x 256)
constexpr int kDecFuseVec = 4;
constexpr int kDecFuseMaxElems = 8 * kDecFuseVec * 256;

// Programmatic dependent launch: let the next kernel on the stream start
// launching, and wait for the previous kernel's results.
__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait_prior()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// 16-byte load of data that stays constant while the kernel runs and is read
// once (the packed weights): no L1 allocation.
__device__ __forceinline__ uint4 ld_stream16(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// A lane's T24 weights of one row and chunk: 8 low-plane bytes and 4
// high-plane bytes (read once, no L1 allocation) as (lo, lo, hi, 0).
__device__ __forceinline__ uint4 ld_stream_t24(const void *lo, const void *hi)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(lo));
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v.z) : "l"(hi));
    v.w = 0u;
    return v;
}

// 16-byte coherent load of data written by the previous kernel (ordered
// after the grid-dependency wait by the memory clobbers, free to move past
// the MMAs).
__device__ __forceinline__ uint4 ld_global16(const void *p)
{
    uint4 v;
    asm("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

__device__ __forceinline__ float ld_global_f32(const float *p)
{
    float v;
    asm("ld.global.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint4 ld_shared16(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t absmax8_bits(const uint4 &v)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
    return __float_as_uint(m);  // |x| >= 0: the bit patterns order as the values
}

// Per-token absmax quantisation of the bf16 rows X[T][K] into the CTA's
// shared copy xs (row stride xs_stride), by all threads of the CTA in one
// pass: thread i holds the 16-byte groups i, i + 256, ... (at most
// kDecFuseVec, T K <= 8 kDecFuseVec blockDim) in registers; per-token maxima
// meet in shared memory; CTA 0 also stores Xq and d.  The same arithmetic as
// the activation kernel: a = max|x|, r = fl32(127 / a),
// q = sat8(rint(fl32(x r))), d = fl32(a / 127); a == 0 gives q = 0, d = 0.
// s_amax was zeroed, and a barrier passed, before the grid-dependency wait.
__device__ __forceinline__ void decode_quantize_x(const DecodeArgs &a, uint32_t xs, uint32_t *s_amax)
{
    const int tid = threadIdx.x, nth = blockDim.x;
    const int k8 = a.K >> 3, n = a.T * k8;
    const uint4 *x4 = reinterpret_cast<const uint4 *>(a.x);
    uint4 v[kDecFuseVec];
#pragma unroll
    for (int u = 0; u < kDecFuseVec; ++u) {
        const int i = tid + u * nth;
        v[u] = i < n ? ld_global16(x4 + i) : make_uint4(0u, 0u, 0u, 0u);
    }
    int tcur = -1;
    uint32_t mcur = 0u;
#pragma unroll
    for (int u = 0; u < kDecFuseVec; ++u) {
        const int i = tid + u * nth;
        if (i >= n) break;
        const int t = i / k8;
        const uint32_t m = absmax8_bits(v[u]);
        if (t != tcur) {
            if (tcur >= 0) atomicMax(&s_amax[tcur], mcur);
            tcur = t;
            mcur = m;
        } else {
            mcur = max(mcur, m);
        }
    }
    if (tcur >= 0) atomicMax(&s_amax[tcur], mcur);
    __syncthreads();
    const bool store = blockIdx.x == 0 && a.xq_out != nullptr;
#pragma unroll
    for (int u = 0; u < kDecFuseVec; ++u) {
        const int i = tid + u * nth;
        if (i >= n) break;
        const int t = i / k8, kk = i - t * k8;
        const float amax = __uint_as_float(s_amax[t]);
        uint2 q = make_uint2(0u, 0u);
        if (amax > 0.0f) {
            const float r = __fdiv_rn(127.0f, amax);
            q.x = quant4(bf16_lo(v[u].x), bf16_hi(v[u].x), bf16_lo(v[u].y), bf16_hi(v[u].y), r);
            q.y = quant4(bf16_lo(v[u].z), bf16_hi(v[u].z), bf16_lo(v[u].w), bf16_hi(v[u].w), r);
        }
        asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(xs + t * a.xs_stride + 8 * kk), "r"(q.x), "r"(q.y)
                     : "memory");
        if (store) reinterpret_cast<uint2 *>(a.xq_out + static_cast<int64_t>(t) * a.K)[kk] = q;
    }
    if (blockIdx.x == 0 && a.d_out && tid < a.T) {
        const float amax = __uint_as_float(s_amax[tid]);
        a.d_out[tid] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
    }
    __syncthreads();
}

// T24 decoding: the PK2 byte (2-bit codes w + 1 of four weights) of a 6-bit
// group code (0: none; 1 + 2p + s_p: one; 9 + 4k + 2 s_p + s_q: two at pair
// k of (0,1) (0,2) (0,3) (1,2) (1,3) (2,3); s = 1 for -1).  Codes above 32
// are never written; they decode as zeros.
__device__ __forceinline__ uint32_t t24_pk2_byte(uint32_t c)
{
    uint32_t b = 0x55u;  // four zero weights
    if (c >= 1u && c <= 8u) {
        const uint32_t p = (c - 1u) >> 1, neg = (c - 1u) & 1u;
        b = (b & ~(3u << (2 * p))) | ((neg ? 0u : 2u) << (2 * p));
    } else if (c >= 9u && c <= 32u) {
        const uint32_t k = (c - 9u) >> 2, r = (c - 9u) & 3u;
        const uint32_t pq = (0x323121302010ull >> (8 * k)) & 0xffu;  // q << 4 | p
        const uint32_t p = pq & 15u, q = pq >> 4;
        b = (b & ~(3u << (2 * p)) & ~(3u << (2 * q))) | (((r & 2u) ? 0u : 2u) << (2 * p)) |
            (((r & 1u) ? 0u : 2u) << (2 * q));
    }
    return b;
}

// Two PK2 bytes of a pair of groups from its 12-bit index: the low-plane byte
// (two nibbles) | the pair's 4 high-plane bits << 8.
__device__ __forceinline__ uint32_t t24_pair_pk2(uint32_t idx)
{
    const uint32_t lo = idx & 0xffu, hi = idx >> 8;
    return t24_pk2_byte((lo & 15u) | ((hi & 3u) << 4)) | (t24_pk2_byte((lo >> 4) | ((hi >> 2) << 4)) << 8);
}

// The four PK2 words of a lane's 64 weights of one row from its 8 low-plane
// bytes (v.x, v.y) and 32 high-plane bits (v.z): word j is pairs 2j and
// 2j + 1 through the shared table.
__device__ __forceinline__ void t24_decode(const uint4 &v, const uint16_t *lut, uint32_t (&w)[4])
{
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t lo = j < 2 ? v.x : v.y;
        const uint32_t i0 = ((lo >> (16 * (j & 1))) & 0xffu) | (((v.z >> (8 * j)) & 15u) << 8);
        const uint32_t i1 = ((lo >> (16 * (j & 1) + 8)) & 0xffu) | (((v.z >> (8 * j + 4)) & 15u) << 8);
        w[j] = static_cast<uint32_t>(lut[i0]) | (static_cast<uint32_t>(lut[i1]) << 16);
    }
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s)
{
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(s));
    return r;
}

__device__ __forceinline__ void mma_u8s8(int32_t (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 4 x 4 byte transpose of a 16-byte group: word j of the result holds input
// bytes j, 4 + j, 8 + j, 12 + j.
__device__ __forceinline__ uint4 transpose4x4(uint4 q)
{
    const uint32_t t0 = prmt(q.x, q.y, 0x5140), t1 = prmt(q.z, q.w, 0x5140);
    const uint32_t t2 = prmt(q.x, q.y, 0x7362), t3 = prmt(q.z, q.w, 0x7362);
    return make_uint4(prmt(t0, t1, 0x5410), prmt(t0, t1, 0x7632), prmt(t2, t3, 0x5410),
                      prmt(t2, t3, 0x7632));
}

__device__ __forceinline__ uint32_t word_of(const uint4 &v, int i)
{
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// NT: n8 token blocks (T <= 8 or T <= 16); CPW: chunks per warp per round;
// RG: groups of 16 rows per CTA, each worked by 8 warps that split the K
// chunks of its rows (the groups read the same activations: L1 hits).
// T24: the weights come as 6-bit group codes (two planes), expanded to PK2
// words through a 4096-entry table in dynamic shared memory (8 KiB) built
// before the wait.
template <int NT, int CPW, int RG, bool FUSE = false, bool T24 = false>
__global__ void __launch_bounds__(256 * RG) decode_kernel(DecodeArgs args)
{
    extern __shared__ __align__(16) uint8_t dec_xs[];
    __shared__ uint32_t s_amax[FUSE ? kDecMaxTokens : 1];
    static_assert(!(T24 && FUSE), "T24 and the fused prologue share the dynamic shared memory");
    uint16_t *t24_lut = reinterpret_cast<uint16_t *>(dec_xs);  // T24: 4096 entries of dynamic shared memory
    if constexpr (FUSE) {
        if (threadIdx.x < kDecMaxTokens) s_amax[threadIdx.x] = 0u;
        __syncthreads();
    }
    if constexpr (T24) {
        for (int i = threadIdx.x; i < 4096; i += blockDim.x) t24_lut[i] = static_cast<uint16_t>(t24_pair_pk2(i));
        __syncthreads();
    }
    constexpr int kWarps = 8;                          // warps per row group
    constexpr int NA = CPW < 4 ? CPW : 4;              // independent MMA chains
    constexpr int G = NT == 1 ? (CPW < 4 ? CPW : 4) : 1;  // chunks loaded together
    __shared__ int32_t part[RG * kWarps][kDecMaxTokens * kDecPartStride];  // [w][t][row]
    __shared__ int32_t csum[RG * kWarps][kDecMaxTokens];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wig = warp % kWarps;                     // warp in its row group
    const int g = lane >> 2, tg = lane & 3;
    const int row0 = (blockIdx.x * RG + warp / kWarps) * kDecRows;
    const bool okA = row0 + g < args.O, okB = row0 + g + 8 < args.O;
    // lane (g, tg) reads rows g and g + 8, bytes 16 tg .. 16 tg + 15 of every
    // 64-byte chunk (weights pos = 256 c + 64 tg .. pos + 63, bytes pos / 4 ..)
    const uint8_t *wA = args.pk2 + static_cast<int64_t>(okA ? row0 + g : 0) * args.pk2_stride;
    const uint8_t *wB = args.pk2 + static_cast<int64_t>(okB ? row0 + g + 8 : 0) * args.pk2_stride;
    // output (t, r) of the row group belongs to thread 16 t + r of the group
    // (the group of thread i is i / 256, the same as its warp's)
    const int t_out = (threadIdx.x & 255) >> 4, r_out = threadIdx.x & 15;
    const bool has_out = t_out < args.T && row0 + r_out < args.O;

    // this kernel only reads what earlier kernels wrote: the next kernel on
    // the stream may launch (and stream its own weights) right away
    pdl_launch_dependents();

    int32_t acc[NA][NT][4];
    uint32_t cs[NT];
#pragma unroll
    for (int b = 0; b < NT; ++b) {
#pragma unroll
        for (int u = 0; u < NA; ++u) acc[u][b][0] = acc[u][b][1] = acc[u][b][2] = acc[u][b][3] = 0;
        cs[b] = 0u;
    }
    float scale = 0.0f;  // gamma * d_t of this thread's output
    for (int round0 = 0; round0 < args.chunks; round0 += kWarps * CPW) {
        // 1. weights of this round's chunks; the first round's loads are in
        //    flight before the wait on the previous kernel
        uint4 wa[CPW], wb[CPW];
#pragma unroll
        for (int i = 0; i < CPW; ++i) {
            const int c = round0 + wig + kWarps * i;
            const int pos = c * kDecChunk + 64 * tg;
            const bool ok = c < args.chunks && pos < args.K;
            if constexpr (T24) {
                // the same rows of the two planes (8 + 4 bytes per lane and chunk)
                const int64_t ra = okA ? row0 + g : 0, rb = okB ? row0 + g + 8 : 0;
                wa[i] = (ok && okA) ? ld_stream_t24(wA + pos / 8, args.t24_hi + ra * args.t24_hi_stride + pos / 16)
                                    : make_uint4(0u, 0u, 0u, 0u);
                wb[i] = (ok && okB) ? ld_stream_t24(wB + pos / 8, args.t24_hi + rb * args.t24_hi_stride + pos / 16)
                                    : make_uint4(0u, 0u, 0u, 0u);
            } else {
                wa[i] = (ok && okA) ? ld_stream16(wA + pos / 4) : make_uint4(0u, 0u, 0u, 0u);
                wb[i] = (ok && okB) ? ld_stream16(wB + pos / 4) : make_uint4(0u, 0u, 0u, 0u);
            }
        }
        if (round0 == 0) {
            pdl_wait_prior();  // activations, scales and gamma
            if constexpr (FUSE) {
                decode_quantize_x(args, smem_addr(dec_xs), s_amax);
                if (has_out) {
                    const float amax = __uint_as_float(s_amax[t_out]);
                    const float d_t = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
                    scale = __fmul_rn(ld_global_f32(args.gamma), d_t);
                }
            } else {
                if (has_out) scale = __fmul_rn(ld_global_f32(args.gamma), ld_global_f32(args.d + t_out));
            }
        }

        // 2. groups of G chunks: the lane's 64 activations of each chunk and
        //    token block (the group's loads first), transposed in registers,
        //    then 8 MMA steps of K = 32 per chunk
#pragma unroll
        for (int i0 = 0; i0 < CPW; i0 += G) {
            if (round0 + wig + kWarps * i0 >= args.chunks) break;  // warp-uniform
            uint4 xr[G][NT][4];
#pragma unroll
            for (int j = 0; j < G; ++j) {
                const int c = round0 + wig + kWarps * (i0 + j);
                const int pos = c * kDecChunk + 64 * tg;
#pragma unroll
                for (int b = 0; b < NT; ++b) {
                    const int t = 8 * b + g;
                    const bool ok = c < args.chunks && pos < args.K && t < args.T;
                    if constexpr (FUSE) {
                        const uint32_t src = smem_addr(dec_xs) + (ok ? t * args.xs_stride + pos : 0);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            xr[j][b][q] = ok ? ld_shared16(src + 16 * q) : make_uint4(0u, 0u, 0u, 0u);
                    } else {
                        const int8_t *src =
                            args.xq + static_cast<int64_t>(ok ? t : 0) * args.K + (ok ? pos : 0);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            xr[j][b][q] = ok ? ld_global16(src + 16 * q) : make_uint4(0u, 0u, 0u, 0u);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < G; ++j) {
                const int i = i0 + j;
                uint4 xt[NT][4];
#pragma unroll
                for (int b = 0; b < NT; ++b) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 v = xr[j][b][q];
                        int c = static_cast<int>(cs[b]);
                        c = __dp4a(static_cast<int>(v.x), 0x01010101, c);
                        c = __dp4a(static_cast<int>(v.y), 0x01010101, c);
                        c = __dp4a(static_cast<int>(v.z), 0x01010101, c);
                        c = __dp4a(static_cast<int>(v.w), 0x01010101, c);
                        cs[b] = static_cast<uint32_t>(c);
                        xt[b][q] = transpose4x4(v);
                    }
                }
                if constexpr (T24) {
                    // the chunk's codes become its PK2 words, in place
                    uint32_t t[4];
                    t24_decode(wa[i], t24_lut, t);
                    wa[i] = make_uint4(t[0], t[1], t[2], t[3]);
                    t24_decode(wb[i], t24_lut, t);
                    wb[i] = make_uint4(t[0], t[1], t[2], t[3]);
                }
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    // step s takes word s/2 of the lane's 16 bytes and the
                    // code shifts ja (K slots 0..15) and ja + 1 (K slots 16..31)
                    const int wi = s >> 1, ja = 2 * (s & 1);
                    const uint32_t ra = word_of(wa[i], wi), rb = word_of(wb[i], wi);
                    const uint32_t a0 = (ra >> (2 * ja)) & 0x03030303u;
                    const uint32_t a1 = (rb >> (2 * ja)) & 0x03030303u;
                    const uint32_t a2 = (ra >> (2 * ja + 2)) & 0x03030303u;
                    const uint32_t a3 = (rb >> (2 * ja + 2)) & 0x03030303u;
#pragma unroll
                    for (int b = 0; b < NT; ++b)
                        mma_u8s8(acc[i % NA][b], a0, a1, a2, a3, word_of(xt[b][wi], ja),
                                 word_of(xt[b][wi], ja + 1));
                }
            }
        }
    }

    // 3. the warps' partials: part[w][token][row]; column sums per token
#pragma unroll
    for (int b = 0; b < NT; ++b) {
        int32_t v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            uint32_t sum = 0u;
#pragma unroll
            for (int u = 0; u < NA; ++u) sum += static_cast<uint32_t>(acc[u][b][e]);
            v[e] = static_cast<int32_t>(sum);
        }
        const int tA = 8 * b + 2 * tg;
        part[warp][tA * kDecPartStride + g] = v[0];
        part[warp][(tA + 1) * kDecPartStride + g] = v[1];
        part[warp][tA * kDecPartStride + g + 8] = v[2];
        part[warp][(tA + 1) * kDecPartStride + g + 8] = v[3];
        uint32_t s = cs[b];
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        if (tg == 0) csum[warp][8 * b + g] = static_cast<int32_t>(s);
    }
    __syncthreads();

    // 4. thread (t, r) of each row group adds its group's 8 partials
    //    (integers: order-free, wrapping arithmetic is exact when the result
    //    fits) and dequantises y = fl32(fl32(acc) * fl32(gamma * d_t))
    if (has_out) {
        const int w0 = (threadIdx.x >> 8) * kWarps;
        uint32_t s = 0u;
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
            s += static_cast<uint32_t>(part[w0 + w][t_out * kDecPartStride + r_out]) -
                 static_cast<uint32_t>(csum[w0 + w][t_out]);
        const int32_t acc_v = static_cast<int32_t>(s);
        const int64_t off = static_cast<int64_t>(t_out) * args.O + row0 + r_out;
        float y = __fmul_rn(__int2float_rn(acc_v), scale);
        if (args.relu2) y = y > 0.0f ? __fmul_rn(y, y) : 0.0f;
        if (args.residual) y = __fadd_rn(y, __uint_as_float(static_cast<uint32_t>(args.residual[off]) << 16));
        if (args.out_fp32) static_cast<float *>(args.out)[off] = y;
        else {
            const __nv_bfloat16 hb = __float2bfloat16_rn(y);
            static_cast<uint16_t *>(args.out)[off] = *reinterpret_cast<const uint16_t *>(&hb);
        }
        if (args.acc_out) args.acc_out[off] = acc_v;
    }
}

}  // namespace sbl
