// sbl_decode.cuh -- decode-time Sparse-BitLinear forward (T <= 16 tokens) that
// streams the 2-bit PK2 weight codes at HBM rate.
//
// The weights stay packed (four ternaries per byte, the storage of the BitNet
// b1.58 2B4T summary, "Inference Implementation: GPU"); the int8 tensor-core
// path of mma.sync consumes them straight from registers:
//  * a 32-bit PK2 word holds codes c = w + 1 of 16 consecutive weights; lane j
//    of a quad extracts (word >> 2j) & 0x03030303, i.e. the four codes of
//    positions j, j+4, j+8, j+12, as four u8 values - two ALU ops for four
//    weights;
//  * the activations are staged in shared memory with every 16-byte group
//    transposed as a 4 x 4 byte matrix, so the B fragment of lane j holds the
//    same positions;
//  * sum_k c * x = sum_k w * x + sum_k x, so the kernel subtracts the
//    activation column sum to get the exact int32 accumulator.
// A CTA owns 128 output rows (8 warps x 16) of one K slice; the CTAs of a
// cluster split K and rank 0 adds their int32 partials (exact) through
// distributed shared memory before the dequantisation
// y = fl32(fl32(acc) * fl32(gamma * d_t)).
#pragma once

#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "sbl_device.cuh"

namespace sbl {

constexpr int kDecRows = 128;      // output rows per CTA
constexpr int kDecThreads = 256;   // 8 warps x 16 rows
constexpr int kDecMaxTokens = 16;
constexpr int kDecKUnit = 64;      // K slices are multiples of 64 (16 PK2 bytes)

struct DecodeArgs {
    const uint8_t *pk2;
    int64_t pk2_stride;   // bytes per packed row
    const int8_t *xq;     // [T, K]
    const float *d;       // [T]
    const float *gamma;   // device scalar
    void *out;            // [T, O] bf16 bits or fp32
    int32_t out_fp32;
    int32_t *acc_out;     // optional [T, O] int32
    int32_t T, K, O;
    int32_t units;        // K / 64
    int32_t cluster;      // CTAs per cluster (K split)
    int32_t w_stride;     // shared-memory bytes per weight row (odd multiple of 16)
    int32_t a_stride;     // shared-memory bytes per activation row
    int32_t max_slice;    // largest K slice of any rank
    uint32_t *err;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

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

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s)
{
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(s));
    return r;
}

__device__ __forceinline__ void mma_u8s8(int32_t (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void slice_of(int rank, int nranks, int units, int &u0, int &u1)
{
    const int base = units / nranks, extra = units % nranks;
    u0 = rank * base + min(rank, extra);
    u1 = u0 + base + (rank < extra ? 1 : 0);
}

template <int NT>  // 1 or 2 n8 token blocks (T <= 8 or T <= 16)
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(DecodeArgs args)
{
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    extern __shared__ __align__(128) uint8_t smem[];
    const int rank = static_cast<int>(cluster.block_rank());
    const int nranks = args.cluster;
    const int row_block = blockIdx.x / nranks;
    const int row0 = row_block * kDecRows;
    const int rows_here = min(kDecRows, args.O - row0);
    int u0, u1;
    slice_of(rank, nranks, args.units, u0, u1);
    const int k0 = u0 * kDecKUnit;
    const int klen = (u1 - u0) * kDecKUnit;

    uint8_t *w_sm = smem;                                             // [128][w_stride]
    uint8_t *a_sm = w_sm + kDecRows * args.w_stride;                  // [16][a_stride]
    int32_t *part = reinterpret_cast<int32_t *>(a_sm + kDecMaxTokens * args.a_stride);  // [128][16]
    int32_t *colsum = part + kDecRows * kDecMaxTokens;                // [16]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // 1. the packed weights of this slice (read-only for the whole decode
    //    chain): 16-byte asynchronous copies from every thread, issued before
    //    waiting on the previous kernel so the stream overlaps its tail
    {
        const int cpr = klen / 64;  // 16-byte chunks per packed row slice
        const int total = rows_here * cpr;
        for (int c = threadIdx.x; c < total; c += kDecThreads) {
            const int r = c / cpr, q = c - r * cpr;
            cp_async16(smem_addr(w_sm + r * args.w_stride + 16 * q),
                       args.pk2 + static_cast<int64_t>(row0 + r) * args.pk2_stride + k0 / 4 + 16 * q);
        }
    }
    pdl_wait_prior();  // activations, scales and gamma come from earlier kernels

    // 2. activations of this K slice: 4x4 byte transpose per 16-byte group
    //    (tokens >= T are zero), plus the per-token column sums.  Each thread
    //    issues all of its loads before transposing.
    const int tokens = NT * 8;
    const int groups = klen / 16;
    {
        constexpr int kMaxPer = (kDecMaxTokens * 1024 / 16 + kDecThreads - 1) / kDecThreads;  // slice <= 1024
        const int total = tokens * groups;
        uint4 q[kMaxPer];
#pragma unroll
        for (int i = 0; i < kMaxPer; ++i) {
            const int idx = threadIdx.x + i * kDecThreads;
            q[i] = make_uint4(0u, 0u, 0u, 0u);
            if (idx < total) {
                const int t = idx / groups, gq = idx - t * groups;
                if (t < args.T)
                    q[i] = __ldg(reinterpret_cast<const uint4 *>(args.xq + static_cast<int64_t>(t) * args.K + k0) + gq);
            }
        }
#pragma unroll
        for (int i = 0; i < kMaxPer; ++i) {
            const int idx = threadIdx.x + i * kDecThreads;
            if (idx < total) {
                const int t = idx / groups, gq = idx - t * groups;
                const uint32_t t0 = prmt(q[i].x, q[i].y, 0x5140), t1 = prmt(q[i].z, q[i].w, 0x5140);
                const uint32_t t2 = prmt(q[i].x, q[i].y, 0x7362), t3 = prmt(q[i].z, q[i].w, 0x7362);
                *reinterpret_cast<uint4 *>(a_sm + t * args.a_stride + gq * 16) =
                    make_uint4(prmt(t0, t1, 0x5410), prmt(t0, t1, 0x7632), prmt(t2, t3, 0x5410),
                               prmt(t2, t3, 0x7632));
            }
        }
    }
    __syncthreads();
    for (int t = warp; t < tokens; t += kDecThreads / 32) {
        int s = 0;
        for (int wi = lane; wi < klen / 4; wi += 32)
            s = __dp4a(*reinterpret_cast<const int32_t *>(a_sm + t * args.a_stride + 4 * wi),
                       0x01010101, s);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) colsum[t] = s;
    }
    cp_async_wait_all();
    __syncthreads();
    // the weights are in shared memory: let the next kernel start streaming its own
    pdl_launch_dependents();

    // 3. MMAs: warp w owns rows 16w .. 16w+15 of the block
    const int g = lane >> 2, tg = lane & 3;
    int32_t acc[NT][4];
#pragma unroll
    for (int b = 0; b < NT; ++b) acc[b][0] = acc[b][1] = acc[b][2] = acc[b][3] = 0;
    {
        const uint8_t *wr0 = w_sm + (16 * warp + g) * args.w_stride;
        const uint8_t *wr1 = wr0 + 8 * args.w_stride;
        const int sh = 2 * tg;
#pragma unroll 4
        for (int kk = 0; kk < klen; kk += 32) {
            const uint32_t w00 = *reinterpret_cast<const uint32_t *>(wr0 + kk / 4);
            const uint32_t w01 = *reinterpret_cast<const uint32_t *>(wr0 + kk / 4 + 4);
            const uint32_t w10 = *reinterpret_cast<const uint32_t *>(wr1 + kk / 4);
            const uint32_t w11 = *reinterpret_cast<const uint32_t *>(wr1 + kk / 4 + 4);
            const uint32_t a0 = (w00 >> sh) & 0x03030303u, a2 = (w01 >> sh) & 0x03030303u;
            const uint32_t a1 = (w10 >> sh) & 0x03030303u, a3 = (w11 >> sh) & 0x03030303u;
#pragma unroll
            for (int b = 0; b < NT; ++b) {
                const uint8_t *ar = a_sm + (8 * b + g) * args.a_stride + kk + 4 * tg;
                const uint32_t b0 = *reinterpret_cast<const uint32_t *>(ar);
                const uint32_t b1 = *reinterpret_cast<const uint32_t *>(ar + 16);
                mma_u8s8(acc[b], a0, a1, a2, a3, b0, b1);
            }
        }
    }
    // 4. partial (with the code bias removed) to shared memory: part[row][token]
#pragma unroll
    for (int b = 0; b < NT; ++b) {
        const int tA = 8 * b + 2 * tg, tB = tA + 1;
        const int rA = 16 * warp + g, rB = rA + 8;
        part[rA * kDecMaxTokens + tA] = acc[b][0] - colsum[tA];
        part[rA * kDecMaxTokens + tB] = acc[b][1] - colsum[tB];
        part[rB * kDecMaxTokens + tA] = acc[b][2] - colsum[tA];
        part[rB * kDecMaxTokens + tB] = acc[b][3] - colsum[tB];
    }
    cluster.sync();

    // 5. every rank finishes a share of the (row, token) outputs: it adds the
    //    partials of all ranks (integers: order-free) and dequantises
    {
        const float gam = *args.gamma;
        const int items = kDecRows * args.T;
        const int per = (items + nranks - 1) / nranks;
        const int i0 = rank * per, i1 = min(items, i0 + per);
        for (int idx = i0 + threadIdx.x; idx < i1; idx += kDecThreads) {
            const int t = idx / kDecRows, r = idx - t * kDecRows;
            if (r >= rows_here) continue;
            int32_t v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)  // all remote loads in flight together
                v[q] = (q < nranks) ? cluster.map_shared_rank(part, q)[r * kDecMaxTokens + t] : 0;
            const int32_t s = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
            const int o = row0 + r;
            const int64_t off = static_cast<int64_t>(t) * args.O + o;
            const float c = __fmul_rn(gam, args.d[t]);
            const float y = __fmul_rn(__int2float_rn(s), c);
            if (args.out_fp32) static_cast<float *>(args.out)[off] = y;
            else {
                const __nv_bfloat16 hb = __float2bfloat16_rn(y);
                static_cast<uint16_t *>(args.out)[off] = *reinterpret_cast<const uint16_t *>(&hb);
            }
            if (args.acc_out) args.acc_out[off] = s;
        }
    }
    cluster.sync();  // keep every rank's shared memory alive until all reads are done
}

}  // namespace sbl
