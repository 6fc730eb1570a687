// sbl_api.cu -- host side of libsbl.so: argument validation, tensor-map
// encoding and kernel launches behind the C ABI declared in include/sbl.h.
// The library allocates no device memory; every call only enqueues work on
// the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "sbl.h"
#include "sbl_act.cuh"
#include "sbl_decode.cuh"
#include "sbl_gemv.cuh"
#include "sbl_sp24.cuh"
#include "sbl_gemm.cuh"
#include "sbl_pack.cuh"

namespace sbl {

__device__ uint32_t g_device_error;

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxDim = 65536;

struct DeviceInfo {
    bool probed = false;
    bool ok = false;
    int num_sms = 0;
    uint32_t *err = nullptr;
};

static std::mutex g_mutex;
static DeviceInfo g_devices[kMaxDevices];

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
static EncodeTiledFn g_encode = nullptr;

// Probe the current device once: sm_100, SM count, error word address,
// kernel attributes.
static sbl_status current_device(DeviceInfo **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SBL_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo &di = g_devices[dev];
    if (!di.probed) {
        di.probed = true;
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&di.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            return SBL_ERR_DEVICE;
        }
        if (major != 10 || minor != 0) return SBL_ERR_DEVICE;
        if (cudaGetSymbolAddress(reinterpret_cast<void **>(&di.err), g_device_error) != cudaSuccess)
            return SBL_ERR_CUDA;
        if (cudaFuncSetAttribute(gemm_kernel<kKindI8, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmCfg<256>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_kernel<kKindF16, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmCfg<256>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_kernel<kKindBF16, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmCfg<256>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_kernel<kKindI8, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmCfg<128>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_kernel<kKindF16, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmCfg<128>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_kernel<kKindBF16, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmCfg<128>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_kernel<kKindI8, 256, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmCfg<256>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_kernel<kKindI8, 128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmCfg<128>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_kernel<kKindI8, 256, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmCfg<256, true>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_kernel<kKindI8, 256, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmCfg<256, true>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_kernel<kKindF16, 256, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmCfg<256, true>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_group_kernel<256, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmCfg<256, true>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_group_kernel<256, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmCfg<256>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_group_kernel<128, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmCfg<128>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_kernel<kKindBF16, 256, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmCfg<256, true>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(sp24_pair_kernel<224>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Sp24PairCfg<224>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(sp24_pair_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Sp24PairCfg<128>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(sp24_pair_kernel<224, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Sp24PairCfg<224>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(sp24_pair_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Sp24PairCfg<128>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(gemv_stream_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kGvSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(gemv_stream_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kGvSmemBytes) != cudaSuccess)
            return SBL_ERR_CUDA;
        if (!g_encode) {
            void *fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                                 &q) != cudaSuccess ||
                q != cudaDriverEntryPointSuccess || !fn)
                return SBL_ERR_CUDA;
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
        di.ok = true;
    }
    if (!di.ok) return SBL_ERR_DEVICE;
    *out = &di;
    return SBL_OK;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

static sbl_status check_desc(const sbl_layer_desc *d)
{
    if (!d) return SBL_ERR_INVALID_ARG;
    if (d->m != 4 && d->m != 8) return SBL_ERR_UNSUPPORTED;
    if (d->n < 1 || d->n > d->m) return SBL_ERR_SHAPE;
    if (d->in_features < 16 || d->in_features % 16 != 0 || d->in_features % d->m != 0 ||
        d->in_features > kMaxDim)
        return SBL_ERR_SHAPE;
    if (d->out_features < 16 || d->out_features % 16 != 0 || d->out_features > kMaxDim)
        return SBL_ERR_SHAPE;
    const int64_t count = static_cast<int64_t>(d->out_features) * d->in_features;
    if (count > static_cast<int64_t>(kGammaBlock) * kGammaMaxPartials) return SBL_ERR_SHAPE;
    return SBL_OK;
}

// The SP24 operand needs at most two kept weights in every group of four:
// n <= 2 with m = 4, or n <= 2 with m = 8 (each half of a group of eight then
// keeps at most two).
static bool sp24_fits(const sbl_layer_desc *d) { return d->n <= 2; }

static sbl_status launch_status()
{
    return cudaGetLastError() == cudaSuccess ? SBL_OK : SBL_ERR_CUDA;
}

// 2-D K-major tensor map with the 128-byte swizzle: rows x inner elements,
// box = 128 bytes of K x box_rows rows.
static bool encode_kmajor(CUtensorMap *map, const void *base, CUtensorMapDataType dt, int elem_bytes,
                          int64_t inner, int64_t rows, int64_t row_stride_bytes, int box_rows)
{
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_stride_bytes)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kBKBytes / elem_bytes), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Output tensor map for the epilogue's TMA stores: rows x cols of bf16 or
// fp32 with row stride ld elements; box = 32 rows x 128 bytes, 128-byte swizzle.
static bool encode_output(CUtensorMap *map, void *base, bool fp32, int64_t rows, int64_t cols, int64_t ld,
                          bool rows64 = false)
{
    // box: 32 rows of 128 bytes, 128-byte swizzle; rows64: 32 rows of 64
    // bytes, 64-byte swizzle (the bf16 output without the epilogue)
    const int eb = fp32 ? 4 : 2;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * eb)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>((rows64 ? 64 : 128) / eb), 32};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(map, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                                base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                rows64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Tile width per shape: the persistent grid runs ceil(tiles / grid) rounds of
// tiles whose MMA time is proportional to BN.  128-wide tiles move 30% more
// operand bytes per MMA and ran slower at equal rounds on B200, so they are
// taken only when they cut the column-rounds by at least 20%.
static int choose_bn(int32_t M, int32_t N, int num_sms)
{
    auto rounds = [&](int bn) {
        const int64_t tiles = static_cast<int64_t>((M + kBM - 1) / kBM) * ((N + bn - 1) / bn);
        const int64_t grid = tiles < num_sms ? tiles : num_sms;
        return ((tiles + grid - 1) / grid) * bn;
    };
    return 5 * rounds(128) <= 4 * rounds(256) ? 128 : 256;
}

template <int KIND, int BN, bool EPI, bool PAIR = false>
static sbl_status launch_gemm_bn(const DeviceInfo *di, const CUtensorMap &ta, const CUtensorMap &tb,
                                 const CUtensorMap &ty, GemmArgs args, cudaStream_t stream)
{
    constexpr int tile_m = PAIR ? 2 * kBM : kBM;
    args.tiles_m = static_cast<int32_t>((args.M + tile_m - 1) / tile_m);
    args.tiles_n = static_cast<int32_t>((args.N + BN - 1) / BN);
    const int tiles = args.tiles_m * args.tiles_n;
    const int units = PAIR ? di->num_sms / 2 : di->num_sms;  // CTAs, or CTA pairs
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>((PAIR ? 2 : 1) * (tiles < units ? tiles : units)));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = GemmCfg<BN, PAIR>::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = PAIR ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, gemm_kernel<KIND, BN, EPI, PAIR>, ta, tb, ty, args) != cudaSuccess)
        return SBL_ERR_CUDA;
    return launch_status();
}

template <int KIND>
static sbl_status launch_gemm(const DeviceInfo *di, const void *A, int64_t lda_bytes, const void *B,
                              int64_t ldb_bytes, int32_t M, int32_t N, int32_t K, GemmArgs args,
                              cudaStream_t stream)
{
    const int eb = (KIND == kKindI8) ? 1 : 2;
    const CUtensorMapDataType dt = (KIND == kKindI8)    ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                   : (KIND == kKindF16) ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                        : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const int bn = choose_bn(M, N, di->num_sms);
    // 256-wide tiles run on CTA pairs (256 x 256 per pair, each CTA loading
    // 128 rows of B): a third fewer operand bytes per MMA, so more of them are
    // in flight
    const bool pair = bn == 256 && M > kBM;
    CUtensorMap ta, tb, ty;
    if (!encode_kmajor(&ta, A, dt, eb, K, M, lda_bytes, kBM)) return SBL_ERR_CUDA;
    if (!encode_kmajor(&tb, B, dt, eb, K, N, ldb_bytes, pair ? bn / 2 : bn)) return SBL_ERR_CUDA;
    const bool with_epi = KIND == kKindI8 && (args.relu2 || args.residual);
    if (!encode_output(&ty, args.out, args.out_fp32 != 0, M, N, args.ldo, !args.out_fp32 && !with_epi))
        return SBL_ERR_CUDA;
    args.M = M;
    args.N = N;
    args.K = K;
    args.k_blocks = static_cast<int32_t>((static_cast<int64_t>(K) * eb + kBKBytes - 1) / kBKBytes);
    args.err = di->err;
    if constexpr (KIND == kKindI8) {
        if (pair)
            return with_epi ? launch_gemm_bn<KIND, 256, true, true>(di, ta, tb, ty, args, stream)
                            : launch_gemm_bn<KIND, 256, false, true>(di, ta, tb, ty, args, stream);
        if (with_epi)
            return bn == 128 ? launch_gemm_bn<KIND, 128, true>(di, ta, tb, ty, args, stream)
                             : launch_gemm_bn<KIND, 256, true>(di, ta, tb, ty, args, stream);
    }
    if (pair) return launch_gemm_bn<KIND, 256, false, true>(di, ta, tb, ty, args, stream);
    return bn == 128 ? launch_gemm_bn<KIND, 128, false>(di, ta, tb, ty, args, stream)
                     : launch_gemm_bn<KIND, 256, false>(di, ta, tb, ty, args, stream);
}

// One launch of grouped int8 products (p.grp and every map filled in).
template <int BN, bool PAIR>
static sbl_status launch_gemm_group(const DeviceInfo *di, GemmGroupParams &p, cudaStream_t stream)
{
    constexpr int tile_m = PAIR ? 2 * kBM : kBM;
    p.args.tiles_m = static_cast<int32_t>((p.args.M + tile_m - 1) / tile_m);
    p.args.tiles_n = p.grp.tn0[p.grp.count];
    const int tiles = p.args.tiles_m * p.args.tiles_n;
    const int units = PAIR ? di->num_sms / 2 : di->num_sms;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>((PAIR ? 2 : 1) * (tiles < units ? tiles : units)));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = GemmCfg<BN, PAIR>::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = PAIR ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, gemm_group_kernel<BN, PAIR>, p) != cudaSuccess) return SBL_ERR_CUDA;
    return launch_status();
}

// 3-D view of the SP24 metadata [O, row_bytes] for the sparse GEMM: dims
// (16 bytes, O rows, row_bytes / 16 chunks) with strides (row_bytes, 16), box
// (16, 128, 2), so one load writes the [2][128][16] no-swizzle layout that
// tcgen05.cp reads.
static bool encode_sp24_meta(CUtensorMap *map, const void *base, int64_t rows, int64_t row_bytes)
{
    cuuint64_t dims[3] = {16, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(row_bytes / 16)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_bytes), 16};
    cuuint32_t box[3] = {16, static_cast<cuuint32_t>(kSpBM), 2};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Output map of the sparse GEMM's stores: [rows, cols] bf16 or fp32, box 32
// rows x 32 columns, no swizzle.
static bool encode_output_32x32(CUtensorMap *map, void *base, bool fp32, int64_t rows, int64_t cols)
{
    const int eb = fp32 ? 4 : 2;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * eb)};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(map, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                                base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Token-tile width of the CTA-pair sparse GEMM: the persistent grid of
// num_sms / 2 pairs runs ceil(tiles / pairs) rounds, each costing about the
// tile width plus a fixed part (pipeline fill, epilogue tail) worth 64
// columns; the narrower tile wins only when it saves whole rounds.
static int choose_pair_bn(int32_t O, int32_t T, int num_sms)
{
    const int pairs = num_sms / 2;
    auto cost = [&](int bn) {
        const int64_t tiles = static_cast<int64_t>((O + 255) / 256) * ((T + bn - 1) / bn);
        const int64_t p = tiles < pairs ? tiles : pairs;
        return ((tiles + p - 1) / p) * (bn + 64);
    };
    return cost(128) < cost(224) ? 128 : 224;
}

// The same GEMM on CTA pairs: 256 weight rows x BN tokens per cluster of two.
template <int BN>
static sbl_status launch_sp24_pair(const DeviceInfo *di, int32_t O, int32_t K, int32_t T, const int8_t *Xq,
                                   const float *d, const sbl_packed *w, void *Y, bool y_fp32, int32_t *acc_out,
                                   const sbl_epilogue *epi, cudaStream_t stream)
{
    const int64_t vstride = round_up(K / 2, 16), mstride = round_up(K / 8, 16);
    CUtensorMap ta, tb, te, ty;
    if (!encode_kmajor(&ta, w->sp24_values, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, O, vstride, kSpBM) ||
        !encode_kmajor(&tb, Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, T, K, BN / 2) ||
        !encode_sp24_meta(&te, w->sp24_meta, O, mstride) || !encode_output_32x32(&ty, Y, y_fp32, T, O))
        return SBL_ERR_CUDA;
    Sp24Args a;
    memset(&a, 0, sizeof(a));
    a.O = O;
    a.T = T;
    a.K = K;
    a.tiles_m = (O + 255) / 256;
    a.tiles_n = (T + BN - 1) / BN;
    a.k_blocks = (K + kSpKLogical - 1) / kSpKLogical;
    a.out = Y;
    a.out_fp32 = y_fp32 ? 1 : 0;
    a.acc_out = acc_out;
    a.gamma = w->gamma;
    a.d = d;
    a.err = di->err;
    const bool with_epi = epi && (epi->relu2 || epi->residual);
    if (with_epi) {
        a.relu2 = epi->relu2 ? 1 : 0;
        a.residual = epi->residual;
    }
    const int tiles = a.tiles_m * a.tiles_n;
    const int pairs = tiles < di->num_sms / 2 ? tiles : di->num_sms / 2;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = Sp24PairCfg<BN>::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const cudaError_t e = with_epi ? cudaLaunchKernelEx(&cfg, sp24_pair_kernel<BN, true>, ta, tb, te, ty, a)
                                   : cudaLaunchKernelEx(&cfg, sp24_pair_kernel<BN, false>, ta, tb, te, ty, a);
    if (e != cudaSuccess) return SBL_ERR_CUDA;
    return launch_status();
}

}  // namespace sbl

using namespace sbl;

namespace {

// Row groups (16 rows, 8 warps each) per decode CTA: the kernel supports
// more than one, but one measured fastest for every T (two groups halve the
// activation re-reads from L2 but lose more to fewer, larger CTAs).
constexpr int kDecRowGroups = 1;

// opt: the kPack* bits of the kernel to run.
template <int M>
cudaError_t launch_pack(const cudaLaunchConfig_t &cfg, const PackArgs &pa, int opt)
{
    switch (opt) {
    case 0: return cudaLaunchKernelEx(&cfg, pack_kernel<M, 0>, pa);
    case 1: return cudaLaunchKernelEx(&cfg, pack_kernel<M, 1>, pa);
    case 2: return cudaLaunchKernelEx(&cfg, pack_kernel<M, 2>, pa);
    case 3: return cudaLaunchKernelEx(&cfg, pack_kernel<M, 3>, pa);
    case 4: return cudaLaunchKernelEx(&cfg, pack_kernel<M, 4>, pa);
    case 5: return cudaLaunchKernelEx(&cfg, pack_kernel<M, 5>, pa);
    case 6: return cudaLaunchKernelEx(&cfg, pack_kernel<M, 6>, pa);
    case 7: return cudaLaunchKernelEx(&cfg, pack_kernel<M, 7>, pa);
    case 8: return cudaLaunchKernelEx(&cfg, pack_kernel<M, 8>, pa);
    case 9: return cudaLaunchKernelEx(&cfg, pack_kernel<M, 9>, pa);
    case 10: return cudaLaunchKernelEx(&cfg, pack_kernel<M, 10>, pa);
    case 11: return cudaLaunchKernelEx(&cfg, pack_kernel<M, 11>, pa);
    case 12: return cudaLaunchKernelEx(&cfg, pack_kernel<M, 12>, pa);
    case 13: return cudaLaunchKernelEx(&cfg, pack_kernel<M, 13>, pa);
    case 14: return cudaLaunchKernelEx(&cfg, pack_kernel<M, 14>, pa);
    case 15: return cudaLaunchKernelEx(&cfg, pack_kernel<M, 15>, pa);
    }
    return cudaErrorInvalidValue;
}

// cpw: chunks per warp per round, 1, 2, 4 or 8.
template <int NT>
cudaError_t launch_decode_nt(const cudaLaunchConfig_t &cfg, const DecodeArgs &a, int cpw)
{
    switch (cpw) {
    case 1: return cudaLaunchKernelEx(&cfg, decode_kernel<NT, 1, kDecRowGroups>, a);
    case 2: return cudaLaunchKernelEx(&cfg, decode_kernel<NT, 2, kDecRowGroups>, a);
    case 4: return cudaLaunchKernelEx(&cfg, decode_kernel<NT, 4, kDecRowGroups>, a);
    default: return cudaLaunchKernelEx(&cfg, decode_kernel<NT, 8, kDecRowGroups>, a);
    }
}

template <int NT>
cudaError_t launch_decode_fused(const cudaLaunchConfig_t &cfg, const DecodeArgs &a, int cpw)
{
    switch (cpw) {
    case 1: return cudaLaunchKernelEx(&cfg, decode_kernel<NT, 1, 1, true>, a);
    case 2: return cudaLaunchKernelEx(&cfg, decode_kernel<NT, 2, 1, true>, a);
    case 4: return cudaLaunchKernelEx(&cfg, decode_kernel<NT, 4, 1, true>, a);
    default: return cudaLaunchKernelEx(&cfg, decode_kernel<NT, 8, 1, true>, a);
    }
}

template <int NT>
cudaError_t launch_decode_t24(const cudaLaunchConfig_t &cfg, const DecodeArgs &a, int cpw)
{
    switch (cpw) {
    case 1: return cudaLaunchKernelEx(&cfg, decode_kernel<NT, 1, 1, false, true>, a);
    case 2: return cudaLaunchKernelEx(&cfg, decode_kernel<NT, 2, 1, false, true>, a);
    case 4: return cudaLaunchKernelEx(&cfg, decode_kernel<NT, 4, 1, false, true>, a);
    default: return cudaLaunchKernelEx(&cfg, decode_kernel<NT, 8, 1, false, true>, a);
    }
}

}  // namespace

extern "C" {

const char *sbl_status_string(sbl_status s)
{
    switch (s) {
    case SBL_OK: return "ok";
    case SBL_ERR_INVALID_ARG: return "invalid argument (null pointer or unknown enum)";
    case SBL_ERR_SHAPE: return "unsupported or inconsistent sizes";
    case SBL_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case SBL_ERR_UNSUPPORTED: return "valid but unsupported configuration";
    case SBL_ERR_WORKSPACE: return "workspace missing or too small";
    case SBL_ERR_CUDA: return "CUDA runtime error";
    case SBL_ERR_DEVICE: return "no sm_100 (B200) device current";
    }
    return "unknown status";
}

int32_t sbl_version(void) { return 100; }

size_t sbl_packed_row_bytes(const sbl_layer_desc *desc, sbl_format fmt, sbl_buffer which)
{
    if (check_desc(desc) != SBL_OK) return 0;
    const int64_t K = desc->in_features, O = desc->out_features;
    switch (fmt) {
    case SBL_FMT_PK2: return which == SBL_BUF_MAIN ? static_cast<size_t>(round_up(K / 4, 16)) : 0;
    case SBL_FMT_NM:
        if (which == SBL_BUF_MAIN) return static_cast<size_t>(round_up((K / desc->m * desc->n + 3) / 4, 16));
        return static_cast<size_t>(round_up(K / 8, 16));
    case SBL_FMT_I8: return which == SBL_BUF_MAIN ? static_cast<size_t>(K) : 0;
    case SBL_FMT_BF16T: return which == SBL_BUF_MAIN ? static_cast<size_t>(2 * O) : 0;
    case SBL_FMT_SP24:
        if (which == SBL_BUF_MAIN) return static_cast<size_t>(round_up(K / 2, 16));
        if (which == SBL_BUF_SP24_META) return static_cast<size_t>(round_up(K / 8, 16));
        return 0;
    case SBL_FMT_T24:
        if (which == SBL_BUF_MAIN) return static_cast<size_t>(round_up(K / 8, 16));
        if (which == SBL_BUF_T24_HI) return static_cast<size_t>(round_up(K / 16, 16));
        return 0;
    }
    return 0;
}

size_t sbl_workspace_bytes(const sbl_layer_desc *desc, int32_t tokens, sbl_op op)
{
    if (check_desc(desc) != SBL_OK) return 0;
    if (op == SBL_OP_QUANTIZE_MASK_PACK) return static_cast<size_t>(round_up(sizeof(GammaWorkspace), 256));
    if (op == SBL_OP_BACKWARD) {
        if (tokens < 0) return 0;
        const int64_t tp = round_up(tokens > 0 ? tokens : 1, 64);
        // the two transposed fp16 operands, then 256 bytes for the prescale
        // (the bits of max |dY d_t| and 2^-s)
        return static_cast<size_t>(round_up(static_cast<int64_t>(desc->out_features) * tp * 2, 256) +
                                   round_up(static_cast<int64_t>(desc->in_features) * tp * 2, 256) + 256);
    }
    return 0;
}

}  // extern "C"

// sbl_quantize_mask_pack with optional re-mask statistics (stats may be null).
// gamma_given: out->gamma already holds gamma (a column shard's, from
// sbl_gamma_combine): no workspace, no gamma kernel, and the packing kernel in
// plain stream order.
static sbl_status quantize_mask_pack_impl(const sbl_layer_desc *desc, const void *W, uint32_t formats,
                                          const sbl_packed *out, const sbl_mask_stats *stats,
                                          const sbl_pack_variant *variant, void *workspace,
                                          size_t workspace_bytes, void *stream_p, bool gamma_given = false)
{
    sbl_status st = check_desc(desc);
    const sbl_pack_variant def = {SBL_MASTER_FP32, SBL_MASK_FROM_MASTER, SBL_QUANT_THEN_MASK};
    const sbl_pack_variant v = variant ? *variant : def;
    if ((v.master_dtype != SBL_MASTER_FP32 && v.master_dtype != SBL_MASTER_BF16) ||
        (v.mask_source != SBL_MASK_FROM_MASTER && v.mask_source != SBL_MASK_FROM_QUANTIZED) ||
        (v.order != SBL_QUANT_THEN_MASK && v.order != SBL_MASK_THEN_QUANT))
        return SBL_ERR_INVALID_ARG;
    if (v.mask_source == SBL_MASK_FROM_QUANTIZED && v.order == SBL_MASK_THEN_QUANT) return SBL_ERR_UNSUPPORTED;
    const bool bf16 = v.master_dtype == SBL_MASTER_BF16;
    if (st != SBL_OK) return st;
    if (!W || !out || !out->gamma) return SBL_ERR_INVALID_ARG;
    const uint32_t known = SBL_FMT_PK2 | SBL_FMT_NM | SBL_FMT_I8 | SBL_FMT_BF16T | SBL_FMT_SP24 | SBL_FMT_T24;
    if (formats & ~known) return SBL_ERR_INVALID_ARG;
    if (formats & SBL_FMT_SP24) {
        if (!out->sp24_values || !out->sp24_meta) return SBL_ERR_INVALID_ARG;
        if (!sp24_fits(desc)) return SBL_ERR_UNSUPPORTED;
        if (!aligned16(out->sp24_values) || !aligned16(out->sp24_meta)) return SBL_ERR_ALIGNMENT;
    }
    if (formats & SBL_FMT_T24) {
        if (!out->t24_lo || !out->t24_hi) return SBL_ERR_INVALID_ARG;
        if (!sp24_fits(desc)) return SBL_ERR_UNSUPPORTED;
        if (!aligned16(out->t24_lo) || !aligned16(out->t24_hi)) return SBL_ERR_ALIGNMENT;
    }
    if ((formats & SBL_FMT_PK2) && !out->pk2) return SBL_ERR_INVALID_ARG;
    if ((formats & SBL_FMT_NM) && (!out->nm_values || !out->nm_bitmap)) return SBL_ERR_INVALID_ARG;
    if ((formats & SBL_FMT_I8) && !out->i8) return SBL_ERR_INVALID_ARG;
    if (formats & SBL_FMT_BF16T) {
        if (!out->bf16t) return SBL_ERR_INVALID_ARG;
        if (!(formats & SBL_FMT_I8)) return SBL_ERR_UNSUPPORTED;  // transposed from the int8 copy
    }
    if (!aligned16(W) || !aligned16(out->gamma) || ((formats & SBL_FMT_PK2) && !aligned16(out->pk2)) ||
        ((formats & SBL_FMT_NM) && (!aligned16(out->nm_values) || !aligned16(out->nm_bitmap))) ||
        ((formats & SBL_FMT_I8) && !aligned16(out->i8)) ||
        ((formats & SBL_FMT_BF16T) && !aligned16(out->bf16t)))
        return SBL_ERR_ALIGNMENT;
    if (stats) {
        if (stats->flips && !stats->prev_keep) return SBL_ERR_INVALID_ARG;  // nothing to compare with
        if ((stats->prev_keep && !aligned16(stats->prev_keep)) || (stats->keep && !aligned16(stats->keep)) ||
            (stats->flips && (reinterpret_cast<uintptr_t>(stats->flips) & 7u)) ||
            (stats->near_zero && (reinterpret_cast<uintptr_t>(stats->near_zero) & 7u)) ||
            (stats->block_threshold && !aligned16(stats->block_threshold)))
            return SBL_ERR_ALIGNMENT;
    }
    if (!gamma_given) {
        if (!workspace || workspace_bytes < sbl_workspace_bytes(desc, 0, SBL_OP_QUANTIZE_MASK_PACK))
            return SBL_ERR_WORKSPACE;
        if (reinterpret_cast<uintptr_t>(workspace) & 255u) return SBL_ERR_ALIGNMENT;
    }
    DeviceInfo *di = nullptr;
    if ((st = current_device(&di)) != SBL_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_p);

    const int32_t O = desc->out_features, K = desc->in_features;
    const int64_t count = static_cast<int64_t>(O) * K;
    GammaWorkspace *ws = static_cast<GammaWorkspace *>(workspace);
    if (!gamma_given && cudaMemsetAsync(&ws->counter, 0, sizeof(uint32_t), stream) != cudaSuccess)
        return SBL_ERR_CUDA;
    if (formats & SBL_FMT_NM) {
        // presets the packing kernel edits in place (set before gamma_kernel,
        // so the packing kernel follows gamma_kernel directly: a memset in
        // between would break its programmatic dependent launch)
        if (cudaMemsetAsync(out->nm_values, 0x55,
                            static_cast<size_t>(O) * sbl_packed_row_bytes(desc, SBL_FMT_NM, SBL_BUF_MAIN),
                            stream) != cudaSuccess ||
            cudaMemsetAsync(out->nm_bitmap, 0,
                            static_cast<size_t>(O) * sbl_packed_row_bytes(desc, SBL_FMT_NM, SBL_BUF_NM_BITMAP),
                            stream) != cudaSuccess)
            return SBL_ERR_CUDA;
    }
    if (stats) {
        // before gamma_kernel, for the same reason
        if ((stats->flips && cudaMemsetAsync(stats->flips, 0, sizeof(unsigned long long), stream) != cudaSuccess) ||
            (stats->near_zero &&
             cudaMemsetAsync(stats->near_zero, 0, sizeof(unsigned long long), stream) != cudaSuccess))
            return SBL_ERR_CUDA;
        if (stats->keep && round_up(K / 8, 16) > K / 8 &&
            cudaMemsetAsync(stats->keep, 0, static_cast<size_t>(O) * round_up(K / 8, 16), stream) != cudaSuccess)
            return SBL_ERR_CUDA;  // row padding of the bitmap reads 0
    }

    const int gblocks = static_cast<int>((count + kGammaBlock - 1) / kGammaBlock);
    const bool surv = v.order == SBL_MASK_THEN_QUANT;
    const int64_t divisor = surv ? count / desc->m * desc->n : count;
    const int gm = surv ? desc->m : 0;
    if (gamma_given) {
        // gamma is in out->gamma already
    } else if (bf16) {
        const uint16_t *Wb = static_cast<const uint16_t *>(W);
        if (gm == 0) gamma_kernel<uint16_t, 0><<<gblocks, 256, 0, stream>>>(Wb, count, ws, out->gamma, desc->n, divisor);
        else if (gm == 4) gamma_kernel<uint16_t, 4><<<gblocks, 256, 0, stream>>>(Wb, count, ws, out->gamma, desc->n, divisor);
        else gamma_kernel<uint16_t, 8><<<gblocks, 256, 0, stream>>>(Wb, count, ws, out->gamma, desc->n, divisor);
    } else {
        const float *Wf = static_cast<const float *>(W);
        if (gm == 0) gamma_kernel<float, 0><<<gblocks, 256, 0, stream>>>(Wf, count, ws, out->gamma, desc->n, divisor);
        else if (gm == 4) gamma_kernel<float, 4><<<gblocks, 256, 0, stream>>>(Wf, count, ws, out->gamma, desc->n, divisor);
        else gamma_kernel<float, 8><<<gblocks, 256, 0, stream>>>(Wf, count, ws, out->gamma, desc->n, divisor);
    }
    if ((st = launch_status()) != SBL_OK) return st;

    PackArgs pa;
    memset(&pa, 0, sizeof(pa));
    pa.W = W;
    pa.rows = O;
    pa.cols = K;
    pa.n = desc->n;
    pa.count = count;
    pa.inv_cols = ~0ull / static_cast<uint64_t>(K) + 1ull;  // ceil(2^64 / K)
    pa.gamma = out->gamma;
    if (formats & SBL_FMT_PK2) {
        pa.out.pk2 = out->pk2;
        pa.out.pk2_stride = static_cast<int64_t>(sbl_packed_row_bytes(desc, SBL_FMT_PK2, SBL_BUF_MAIN));
    }
    if (formats & SBL_FMT_I8) pa.out.i8 = out->i8;
    if (formats & SBL_FMT_NM) {
        pa.out.nm_values = out->nm_values;
        pa.out.nm_values_stride = static_cast<int64_t>(sbl_packed_row_bytes(desc, SBL_FMT_NM, SBL_BUF_MAIN));
        pa.out.nm_bitmap = out->nm_bitmap;
        pa.out.nm_bitmap_stride =
            static_cast<int64_t>(sbl_packed_row_bytes(desc, SBL_FMT_NM, SBL_BUF_NM_BITMAP));
    }
    if (formats & SBL_FMT_T24) {
        pa.out.t24_lo = out->t24_lo;
        pa.out.t24_lo_stride = static_cast<int64_t>(sbl_packed_row_bytes(desc, SBL_FMT_T24, SBL_BUF_MAIN));
        pa.out.t24_hi = out->t24_hi;
        pa.out.t24_hi_stride = static_cast<int64_t>(sbl_packed_row_bytes(desc, SBL_FMT_T24, SBL_BUF_T24_HI));
    }
    if (formats & SBL_FMT_SP24) {
        pa.out.sp24_values = out->sp24_values;
        pa.out.sp24_values_stride = static_cast<int64_t>(sbl_packed_row_bytes(desc, SBL_FMT_SP24, SBL_BUF_MAIN));
        pa.out.sp24_meta = out->sp24_meta;
        pa.out.sp24_meta_stride = static_cast<int64_t>(sbl_packed_row_bytes(desc, SBL_FMT_SP24, SBL_BUF_SP24_META));
    }
    const bool want_stats = stats && (stats->keep || stats->flips || stats->near_zero || stats->block_threshold);
    if (want_stats) {
        pa.stats.prev_keep = stats->prev_keep;
        pa.stats.keep = stats->keep;
        pa.stats.keep_stride = static_cast<int64_t>(round_up(K / 8, 16));
        pa.stats.flips = stats->flips;
        pa.stats.near_zero = stats->near_zero;
        pa.stats.threshold = stats->block_threshold;
    }
    if ((formats & (SBL_FMT_PK2 | SBL_FMT_I8 | SBL_FMT_NM | SBL_FMT_SP24 | SBL_FMT_T24)) || want_stats) {
        // programmatic dependent launch behind gamma_kernel (see pack_kernel);
        // a thread covers 16 weights
        const int64_t per_cta = 256 * 16 / desc->m;  // groups per CTA
        const int64_t groups = count / desc->m;
        cudaLaunchConfig_t cfg;
        memset(&cfg, 0, sizeof(cfg));
        cfg.gridDim = dim3(static_cast<unsigned>((groups + per_cta - 1) / per_cta));
        cfg.blockDim = dim3(256);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = gamma_given ? 0 : 1;
        const bool sp = (formats & (SBL_FMT_SP24 | SBL_FMT_T24)) != 0;  // the 2:4 formats' instantiation
        const int opt = (sp ? kPackSp24 : 0) | (want_stats ? kPackStats : 0) |
                        (v.mask_source == SBL_MASK_FROM_QUANTIZED ? kPackMaskQ : 0) | (bf16 ? kPackBf16 : 0);
        const cudaError_t e = desc->m == 8 ? launch_pack<8>(cfg, pa, opt) : launch_pack<4>(cfg, pa, opt);
        if (e != cudaSuccess) return SBL_ERR_CUDA;
        if ((st = launch_status()) != SBL_OK) return st;
    }
    if (formats & SBL_FMT_BF16T) {
        dim3 grid((K + 63) / 64, (O + 63) / 64);
        transpose_i8_to_bf16_kernel<<<grid, 256, 0, stream>>>(out->i8, O, K, out->bf16t);
        if ((st = launch_status()) != SBL_OK) return st;
    }
    return SBL_OK;
}

extern "C" {

sbl_status sbl_quantize_mask_pack(const sbl_layer_desc *desc, const float *W, uint32_t formats,
                                  const sbl_packed *out, void *workspace, size_t workspace_bytes,
                                  void *stream_p)
{
    return quantize_mask_pack_impl(desc, W, formats, out, nullptr, nullptr, workspace, workspace_bytes, stream_p);
}

sbl_status sbl_quantize_mask_pack_stats(const sbl_layer_desc *desc, const float *W, uint32_t formats,
                                        const sbl_packed *out, const sbl_mask_stats *stats, void *workspace,
                                        size_t workspace_bytes, void *stream_p)
{
    return quantize_mask_pack_impl(desc, W, formats, out, stats, nullptr, workspace, workspace_bytes, stream_p);
}

sbl_status sbl_quantize_mask_pack_ex(const sbl_layer_desc *desc, const void *W, const sbl_pack_variant *variant,
                                     uint32_t formats, const sbl_packed *out, const sbl_mask_stats *stats,
                                     void *workspace, size_t workspace_bytes, void *stream_p)
{
    return quantize_mask_pack_impl(desc, W, formats, out, stats, variant, workspace, workspace_bytes, stream_p);
}

size_t sbl_gamma_node_count(const sbl_layer_desc *shard)
{
    if (check_desc(shard) != SBL_OK) return 0;
    const int64_t count = static_cast<int64_t>(shard->out_features) * shard->in_features;
    return static_cast<size_t>((count + kGammaBlock - 1) / kGammaBlock);
}

sbl_status sbl_gamma_partials(const sbl_layer_desc *shard, const float *W, int64_t first_row, double *node_sums,
                              void *workspace, size_t workspace_bytes, void *stream_p)
{
    sbl_status st = check_desc(shard);
    if (st != SBL_OK) return st;
    if (!W || !node_sums) return SBL_ERR_INVALID_ARG;
    const int64_t K = shard->in_features;
    if (first_row < 0 || first_row > kMaxDim || (first_row * K) % kGammaBlock != 0) return SBL_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(node_sums)) return SBL_ERR_ALIGNMENT;
    if (!workspace || workspace_bytes < sbl_workspace_bytes(shard, 0, SBL_OP_QUANTIZE_MASK_PACK))
        return SBL_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return SBL_ERR_ALIGNMENT;
    DeviceInfo *di = nullptr;
    if ((st = current_device(&di)) != SBL_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_p);
    const int64_t count = static_cast<int64_t>(shard->out_features) * K;
    const int nodes = static_cast<int>((count + kGammaBlock - 1) / kGammaBlock);
    GammaWorkspace *ws = static_cast<GammaWorkspace *>(workspace);
    if (cudaMemsetAsync(&ws->counter, 0, sizeof(uint32_t), stream) != cudaSuccess) return SBL_ERR_CUDA;
    gamma_kernel<float, 0><<<nodes, 256, 0, stream>>>(W, count, ws, nullptr, shard->n, count, nullptr);
    if ((st = launch_status()) != SBL_OK) return st;
    if (cudaMemcpyAsync(node_sums, ws->partials, static_cast<size_t>(nodes) * sizeof(double),
                        cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
        return SBL_ERR_CUDA;
    return SBL_OK;
}

sbl_status sbl_gamma_combine(const double *node_sums, int64_t nodes, int64_t total_weights, float *gamma,
                             void *stream_p)
{
    if (!node_sums || !gamma) return SBL_ERR_INVALID_ARG;
    if (total_weights < 1 || total_weights > static_cast<int64_t>(kGammaBlock) * kGammaMaxPartials ||
        nodes != (total_weights + kGammaBlock - 1) / kGammaBlock)
        return SBL_ERR_SHAPE;
    if (!aligned16(node_sums) || !aligned16(gamma)) return SBL_ERR_ALIGNMENT;
    DeviceInfo *di = nullptr;
    sbl_status st = current_device(&di);
    if (st != SBL_OK) return st;
    gamma_combine_kernel<<<1, 256, 0, static_cast<cudaStream_t>(stream_p)>>>(node_sums, static_cast<int>(nodes),
                                                                             total_weights, gamma);
    return launch_status();
}

sbl_status sbl_quantize_mask_pack_shard(const sbl_layer_desc *shard, const float *W, uint32_t formats,
                                        const sbl_packed *out, void *stream_p)
{
    return quantize_mask_pack_impl(shard, W, formats, out, nullptr, nullptr, nullptr, 0, stream_p, true);
}

sbl_status sbl_quantize_act(const uint16_t *X, int32_t T, int32_t K, int8_t *Xq, float *d, void *stream_p)
{
    if (T < 0 || K < 16 || K % 16 != 0 || K > kMaxDim) return SBL_ERR_SHAPE;
    if (T == 0) return SBL_OK;
    if (!X || !Xq || !d) return SBL_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(Xq) || !aligned16(d)) return SBL_ERR_ALIGNMENT;
    DeviceInfo *di = nullptr;
    sbl_status st = current_device(&di);
    if (st != SBL_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_p);
    const int chunks = K / 8;
    int rt = 32;
    while (rt * kActMaxChunks < chunks) rt *= 2;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaSuccess;
    switch (rt) {
#define SBL_ACT_CASE(R)                                                        \
    case R: {                                                                 \
        constexpr int rows = R >= 256 ? 1 : 256 / R;                          \
        cfg.gridDim = dim3(static_cast<unsigned>((T + rows - 1) / rows));     \
        cfg.blockDim = dim3(R > 256 ? R : 256);                               \
        e = cudaLaunchKernelEx(&cfg, act_quant_kernel<R>, X, T, K, Xq, d);    \
        break;                                                                \
    }
        SBL_ACT_CASE(32)
        SBL_ACT_CASE(64)
        SBL_ACT_CASE(128)
        SBL_ACT_CASE(256)
        SBL_ACT_CASE(512)
        SBL_ACT_CASE(1024)
#undef SBL_ACT_CASE
    default: return SBL_ERR_SHAPE;
    }
    if (e != cudaSuccess) return SBL_ERR_CUDA;
    return launch_status();
}

sbl_status sbl_quantize_act_rmsnorm(const uint16_t *X, int32_t T, int32_t K, const uint16_t *g, float eps, int8_t *Xq,
                                    float *d, void *stream_p)
{
    if (T < 0 || K < 16 || K % 16 != 0 || K > kMaxDim) return SBL_ERR_SHAPE;
    if (T == 0) return SBL_OK;
    if (!X || !Xq || !d) return SBL_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || eps > 3.0e38f) return SBL_ERR_INVALID_ARG;  // finite, non-negative
    if (!aligned16(X) || !aligned16(Xq) || !aligned16(d) || (g && !aligned16(g))) return SBL_ERR_ALIGNMENT;
    DeviceInfo *di = nullptr;
    sbl_status st = current_device(&di);
    if (st != SBL_OK) return st;
    // RT threads per row (the layout of the plain quantiser: 16-byte chunks
    // lt + c RT, c < 8), 256 / RT rows per CTA when RT < 256
    const int chunks = K / 8;
    int rt = 32;
    while (rt * kActMaxChunks < chunks) rt *= 2;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.stream = static_cast<cudaStream_t>(stream_p);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaErrorInvalidValue;
    switch (rt) {
#define SBL_NORM_CASE(R)                                                                   \
    case R: {                                                                             \
        constexpr int rows = R >= 256 ? 1 : 256 / R;                                      \
        cfg.gridDim = dim3(static_cast<unsigned>((T + rows - 1) / rows));                 \
        cfg.blockDim = dim3(R > 256 ? R : 256);                                           \
        e = cudaLaunchKernelEx(&cfg, act_norm_quant_kernel<R>, X, T, K, g, eps, Xq, d);   \
        break;                                                                            \
    }
        SBL_NORM_CASE(32)
        SBL_NORM_CASE(64)
        SBL_NORM_CASE(128)
        SBL_NORM_CASE(256)
        SBL_NORM_CASE(512)
        SBL_NORM_CASE(1024)
#undef SBL_NORM_CASE
    }
    return e == cudaSuccess ? launch_status() : SBL_ERR_CUDA;
}

}  // extern "C"

// The fused decode (every CTA quantises X in its prologue) replaces the
// activation kernel only while X is small: measured on B200 against the two
// launches with programmatic dependent launch, it was 4% faster at T K = 2560,
// even at 6912 and 18% slower at 5120 (two tokens).  The kernel itself takes up
// to T K = kDecFuseMaxElems.
constexpr int64_t kLinearFuseMaxElems = 4096;
static_assert(kLinearFuseMaxElems <= kDecFuseMaxElems, "the fused prologue holds at most kDecFuseMaxElems");

// One decode launch: a CTA per 16 output rows; fused: the bf16 activations
// are quantised in the kernel's prologue into T (K + 16) bytes of shared
// memory (at most 8.4 KB: T K <= 8192).
static sbl_status launch_decode(DecodeArgs &a, bool fuse, cudaStream_t stream, bool t24 = false)
{
    a.chunks = (a.K + kDecChunk - 1) / kDecChunk;
    // chunks per warp per round: the whole row in one round up to
    // K = 16384 (more rounds above)
    const int need = (a.chunks + 7) / 8;
    const int cpw = need <= 1 ? 1 : need <= 2 ? 2 : need <= 4 ? 4 : 8;
    const int rg = kDecRowGroups;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>((a.O + kDecRows * rg - 1) / (kDecRows * rg)));
    cfg.blockDim = dim3(static_cast<unsigned>(256 * rg));
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    // programmatic dependent launch: the kernel loads its (read-only)
    // packed weights before waiting on the previous kernel's outputs
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (t24) {
        cfg.dynamicSmemBytes = 4096 * sizeof(uint16_t);  // the pair table
        e = a.T <= 8 ? launch_decode_t24<1>(cfg, a, cpw) : launch_decode_t24<2>(cfg, a, cpw);
    } else if (fuse) {
        a.xs_stride = a.K + kDecXsPad;
        cfg.dynamicSmemBytes = static_cast<size_t>(a.T) * a.xs_stride;
        e = a.T <= 8 ? launch_decode_fused<1>(cfg, a, cpw) : launch_decode_fused<2>(cfg, a, cpw);
    } else {
        e = a.T <= 8 ? launch_decode_nt<1>(cfg, a, cpw) : launch_decode_nt<2>(cfg, a, cpw);
    }
    return e == cudaSuccess ? launch_status() : SBL_ERR_CUDA;
}

static sbl_status forward_impl(const sbl_layer_desc *desc, const int8_t *Xq, const float *d, int32_t T,
                               const sbl_packed *w, sbl_format fmt, void *Y, int32_t y_is_fp32,
                               int32_t *acc_out, const sbl_epilogue *epi, void *stream_p)
{
    sbl_status st = check_desc(desc);
    if (st != SBL_OK) return st;
    if (T < 0) return SBL_ERR_SHAPE;
    if (T == 0) return SBL_OK;
    if (!Xq || !d || !w || !Y || !w->gamma) return SBL_ERR_INVALID_ARG;
    if (!aligned16(Xq) || !aligned16(d) || !aligned16(Y) || !aligned16(w->gamma) ||
        (acc_out && !aligned16(acc_out)) || (epi && epi->residual && !aligned16(epi->residual)))
        return SBL_ERR_ALIGNMENT;
    DeviceInfo *di = nullptr;
    if ((st = current_device(&di)) != SBL_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_p);
    const int32_t O = desc->out_features, K = desc->in_features;

    if (fmt == SBL_FMT_I8) {
        if (!w->i8) return SBL_ERR_INVALID_ARG;
        if (!aligned16(w->i8)) return SBL_ERR_ALIGNMENT;
        GemmArgs a;
        memset(&a, 0, sizeof(a));
        a.out = Y;
        a.ldo = O;
        a.out_fp32 = y_is_fp32 ? 1 : 0;
        a.acc_out = acc_out;
        a.gamma = w->gamma;
        a.row_scale = d;
        if (epi) {
            a.relu2 = epi->relu2 ? 1 : 0;
            a.residual = epi->residual;
        }
        return launch_gemm<kKindI8>(di, Xq, K, w->i8, K, T, O, K, a, stream);
    }
    if (fmt == SBL_FMT_SP24) {
        if (!w->sp24_values || !w->sp24_meta) return SBL_ERR_INVALID_ARG;
        if (!sp24_fits(desc)) return SBL_ERR_UNSUPPORTED;
        if (!aligned16(w->sp24_values) || !aligned16(w->sp24_meta)) return SBL_ERR_ALIGNMENT;
        return choose_pair_bn(O, T, di->num_sms) == 224
                   ? launch_sp24_pair<224>(di, O, K, T, Xq, d, w, Y, y_is_fp32 != 0, acc_out, epi, stream)
                   : launch_sp24_pair<128>(di, O, K, T, Xq, d, w, Y, y_is_fp32 != 0, acc_out, epi, stream);
    }
    if (fmt == SBL_FMT_T24) {
        if (!w->t24_lo || !w->t24_hi) return SBL_ERR_INVALID_ARG;
        if (!aligned16(w->t24_lo) || !aligned16(w->t24_hi)) return SBL_ERR_ALIGNMENT;
        if (T > kDecMaxTokens || K % kDecKUnit != 0 || !sp24_fits(desc)) return SBL_ERR_UNSUPPORTED;
        DecodeArgs a;
        memset(&a, 0, sizeof(a));
        a.pk2 = w->t24_lo;  // the low plane takes the place of the PK2 codes
        a.pk2_stride = static_cast<int64_t>(sbl_packed_row_bytes(desc, SBL_FMT_T24, SBL_BUF_MAIN));
        a.t24_hi = w->t24_hi;
        a.t24_hi_stride = static_cast<int32_t>(sbl_packed_row_bytes(desc, SBL_FMT_T24, SBL_BUF_T24_HI));
        a.xq = Xq;
        a.d = d;
        a.gamma = w->gamma;
        a.out = Y;
        a.out_fp32 = y_is_fp32 ? 1 : 0;
        a.acc_out = acc_out;
        if (epi) {
            a.relu2 = epi->relu2 ? 1 : 0;
            a.residual = epi->residual;
        }
        a.T = T;
        a.K = K;
        a.O = O;
        return launch_decode(a, false, stream, true);
    }
    if (fmt == SBL_FMT_PK2) {
        if (!w->pk2) return SBL_ERR_INVALID_ARG;
        if (!aligned16(w->pk2)) return SBL_ERR_ALIGNMENT;
        if (T > kDecMaxTokens || K % kDecKUnit != 0) return SBL_ERR_UNSUPPORTED;
        DecodeArgs a;
        memset(&a, 0, sizeof(a));
        a.pk2 = w->pk2;
        a.pk2_stride = static_cast<int64_t>(sbl_packed_row_bytes(desc, SBL_FMT_PK2, SBL_BUF_MAIN));
        a.xq = Xq;
        a.d = d;
        a.gamma = w->gamma;
        a.out = Y;
        a.out_fp32 = y_is_fp32 ? 1 : 0;
        a.acc_out = acc_out;
        if (epi) {
            a.relu2 = epi->relu2 ? 1 : 0;
            a.residual = epi->residual;
        }
        a.T = T;
        a.K = K;
        a.O = O;
        return launch_decode(a, false, stream);
    }
    return SBL_ERR_UNSUPPORTED;
}

extern "C" {

sbl_status sbl_forward(const sbl_layer_desc *desc, const int8_t *Xq, const float *d, int32_t T,
                       const sbl_packed *w, sbl_format fmt, void *Y, int32_t y_is_fp32,
                       int32_t *acc_out, void *stream_p)
{
    return forward_impl(desc, Xq, d, T, w, fmt, Y, y_is_fp32, acc_out, nullptr, stream_p);
}

sbl_status sbl_forward_group(const sbl_layer_desc *const *descs, int32_t count, const int8_t *Xq,
                             const float *d, int32_t T, const sbl_packed *const *w, void *const *Y,
                             int32_t y_is_fp32, void *stream_p)
{
    if (!descs || !w || !Y || count < 1 || count > SBL_GROUP_MAX) return SBL_ERR_INVALID_ARG;
    sbl_status st;
    for (int32_t i = 0; i < count; ++i) {
        if ((st = check_desc(descs[i])) != SBL_OK) return st;
        if (descs[i]->in_features != descs[0]->in_features) return SBL_ERR_SHAPE;
    }
    if (T < 0) return SBL_ERR_SHAPE;
    if (T == 0) return SBL_OK;
    if (!Xq || !d) return SBL_ERR_INVALID_ARG;
    if (!aligned16(Xq) || !aligned16(d)) return SBL_ERR_ALIGNMENT;
    for (int32_t i = 0; i < count; ++i) {
        if (!w[i] || !w[i]->i8 || !w[i]->gamma || !Y[i]) return SBL_ERR_INVALID_ARG;
        if (!aligned16(w[i]->i8) || !aligned16(w[i]->gamma) || !aligned16(Y[i])) return SBL_ERR_ALIGNMENT;
    }
    DeviceInfo *di = nullptr;
    if ((st = current_device(&di)) != SBL_OK) return st;
    const int32_t K = descs[0]->in_features;
    int64_t n_total = 0;
    for (int32_t i = 0; i < count; ++i) n_total += descs[i]->out_features;
    const int bn = choose_bn(T, static_cast<int32_t>(n_total), di->num_sms);
    const bool pair = bn == 256 && T > kBM;
    static GemmGroupParams p;  // 1.4 KB of kernel parameters, copied at launch
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    memset(&p, 0, sizeof(p));
    if (!encode_kmajor(&p.a, Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, T, K, kBM)) return SBL_ERR_CUDA;
    int32_t tn = 0;
    for (int32_t i = 0; i < count; ++i) {
        const int32_t O = descs[i]->out_features;
        if (!encode_kmajor(&p.b[i], w[i]->i8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, O, K, pair ? bn / 2 : bn) ||
            !encode_output(&p.y[i], Y[i], y_is_fp32 != 0, T, O, O, !y_is_fp32))
            return SBL_ERR_CUDA;
        p.grp.tn0[i] = tn;
        p.grp.n[i] = O;
        p.grp.gamma[i] = w[i]->gamma;
        tn += (O + bn - 1) / bn;
    }
    p.grp.tn0[count] = tn;
    p.grp.count = count;
    p.args.M = T;
    p.args.N = static_cast<int32_t>(n_total);
    p.args.K = K;
    p.args.k_blocks = (K + kBKBytes - 1) / kBKBytes;
    p.args.out_fp32 = y_is_fp32 ? 1 : 0;
    p.args.row_scale = d;
    p.args.err = di->err;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_p);
    if (pair) return launch_gemm_group<256, true>(di, p, stream);
    return bn == 128 ? launch_gemm_group<128, false>(di, p, stream) : launch_gemm_group<256, false>(di, p, stream);
}

sbl_status sbl_forward_ex(const sbl_layer_desc *desc, const int8_t *Xq, const float *d, int32_t T,
                          const sbl_packed *w, sbl_format fmt, void *Y, int32_t y_is_fp32, int32_t *acc_out,
                          const sbl_epilogue *epi, void *stream_p)
{
    return forward_impl(desc, Xq, d, T, w, fmt, Y, y_is_fp32, acc_out, epi, stream_p);
}

sbl_status sbl_linear_forward(const sbl_layer_desc *desc, const uint16_t *X, int32_t T, const sbl_packed *w,
                              sbl_format fmt, int8_t *Xq, float *d, void *Y, int32_t y_is_fp32,
                              const sbl_epilogue *epi, void *stream_p)
{
    sbl_status st = check_desc(desc);
    if (st != SBL_OK) return st;
    if (T < 0) return SBL_ERR_SHAPE;
    if (T == 0) return SBL_OK;
    if (!X || !Xq || !d || !w || !Y || !w->gamma) return SBL_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(Xq) || !aligned16(d) || !aligned16(Y) || !aligned16(w->gamma) ||
        (epi && epi->residual && !aligned16(epi->residual)))
        return SBL_ERR_ALIGNMENT;
    const int32_t O = desc->out_features, K = desc->in_features;
    if (fmt == SBL_FMT_PK2 && T <= kDecMaxTokens && K % kDecKUnit == 0 &&
        static_cast<int64_t>(T) * K <= kLinearFuseMaxElems) {
        if (!w->pk2) return SBL_ERR_INVALID_ARG;
        if (!aligned16(w->pk2)) return SBL_ERR_ALIGNMENT;
        DeviceInfo *di = nullptr;
        if ((st = current_device(&di)) != SBL_OK) return st;
        DecodeArgs a;
        memset(&a, 0, sizeof(a));
        a.pk2 = w->pk2;
        a.pk2_stride = static_cast<int64_t>(sbl_packed_row_bytes(desc, SBL_FMT_PK2, SBL_BUF_MAIN));
        a.gamma = w->gamma;
        a.out = Y;
        a.out_fp32 = y_is_fp32 ? 1 : 0;
        if (epi) {
            a.relu2 = epi->relu2 ? 1 : 0;
            a.residual = epi->residual;
        }
        a.T = T;
        a.K = K;
        a.O = O;
        a.x = X;
        a.xq_out = Xq;
        a.d_out = d;
        return launch_decode(a, true, static_cast<cudaStream_t>(stream_p));
    }
    // otherwise the activation kernel, then the layer's forward kernel
    if ((st = sbl_quantize_act(X, T, K, Xq, d, stream_p)) != SBL_OK) return st;
    return forward_impl(desc, Xq, d, T, w, fmt, Y, y_is_fp32, nullptr, epi, stream_p);
}

sbl_format sbl_forward_format(const sbl_layer_desc *desc, int32_t tokens)
{
    if (check_desc(desc) != SBL_OK || tokens < 0) return static_cast<sbl_format>(0);
    if (!sp24_fits(desc)) return SBL_FMT_I8;
    const int64_t outputs = static_cast<int64_t>(tokens) * desc->out_features;
    return (desc->in_features >= 1024 && outputs >= 8192LL * 1024) ? SBL_FMT_SP24 : SBL_FMT_I8;
}

}  // extern "C"

// ------------------------------------------------------ batched decode --
static_assert(SBL_GROUP_MAX == kGemmMaxGroups, "the launch parameters hold every map of a group");
static_assert(SBL_BATCH_MAX_LAYERS <= kGvMaxProblems, "the launch parameters hold every layer of a batch");
static_assert(sizeof(GvArgs) <= 32000 && sizeof(GvPrepArgs) <= 32000, "kernel parameters are limited to 32764 bytes");
constexpr int32_t kGvMaxK = 4 * kGvStageBytes / 16 / kDecKUnit * kDecKUnit;  // 16-row items of K / 4 bytes per row fill a stage

static bool batch_has_chain(const sbl_batch_layer *layers, int32_t count)
{
    for (int32_t i = 0; i < count; ++i)
        if (layers[i].input_is_previous_output) return true;
    return false;
}

// Index of the first unchained layer with the same input (activations and
// width) as layer i, so that each distinct input is prepared once.
static int32_t batch_input_owner(const sbl_batch_layer *layers, int32_t i)
{
    for (int32_t j = 0; j < i; ++j)
        if (!layers[j].input_is_previous_output && layers[j].xq == layers[i].xq &&
            layers[j].desc.in_features == layers[i].desc.in_features)
            return j;
    return i;
}

// Workspace layout: [completion words, 128 bytes per layer, when chained]
// [per distinct unchained input: T K bytes of prepared activations rounded to
// 256, then 256 bytes of column sums].
static int64_t batch_workspace_layout(const sbl_batch_layer *layers, int32_t count, int32_t T, int64_t *offsets)
{
    int64_t off = batch_has_chain(layers, count) ? round_up(static_cast<int64_t>(count) * kGvSyncWords * 4, 256) : 0;
    for (int32_t i = 0; i < count; ++i) {
        if (offsets) offsets[i] = -1;
        if (layers[i].input_is_previous_output || batch_input_owner(layers, i) != i) continue;
        if (offsets) offsets[i] = off;
        off += round_up(static_cast<int64_t>(T) * layers[i].desc.in_features, 256) + 256;
    }
    return off;
}

extern "C" {

size_t sbl_forward_batch_workspace_bytes(const sbl_batch_layer *layers, int32_t count, int32_t T)
{
    if (!layers || count < 1 || count > SBL_BATCH_MAX_LAYERS || T < 1 || T > kDecMaxTokens) return 0;
    for (int32_t i = 0; i < count; ++i)
        if (check_desc(&layers[i].desc) != SBL_OK) return 0;
    return static_cast<size_t>(batch_workspace_layout(layers, count, T, nullptr));
}

sbl_status sbl_forward_batch(const sbl_batch_layer *layers, int32_t count, int32_t T, void *workspace,
                             size_t workspace_bytes, void *stream_p)
{
    if (!layers) return SBL_ERR_INVALID_ARG;
    if (count < 1 || count > SBL_BATCH_MAX_LAYERS || T < 1 || T > kDecMaxTokens) return SBL_ERR_SHAPE;
    // launch parameters (18 KB and 9 KB), filled under the lock below
    static GvArgs a;
    static GvPrepArgs prep;
    static int64_t offsets[SBL_BATCH_MAX_LAYERS];
    static std::mutex batch_mutex;
    std::lock_guard<std::mutex> lock(batch_mutex);
    memset(&a, 0, sizeof(a));
    memset(&prep, 0, sizeof(prep));
    int32_t items = 0;
    bool chain = false;
    for (int32_t i = 0; i < count; ++i) {
        const sbl_batch_layer &L = layers[i];
        sbl_status st = check_desc(&L.desc);
        if (st != SBL_OK) return st;
        const int32_t O = L.desc.out_features, K = L.desc.in_features;
        if (K % kDecKUnit != 0 || K > kGvMaxK) return SBL_ERR_UNSUPPORTED;
        if (!L.pk2 || !L.gamma || !L.y) return SBL_ERR_INVALID_ARG;
        if (!aligned16(L.pk2) || !aligned16(L.gamma) || !aligned16(L.y)) return SBL_ERR_ALIGNMENT;
        const bool ch = L.input_is_previous_output != 0;
        if (ch) {
            if (i == 0) return SBL_ERR_INVALID_ARG;
            const sbl_batch_layer &P = layers[i - 1];
            if (P.desc.out_features != K || P.y_is_fp32) return SBL_ERR_INVALID_ARG;
            if ((L.xq_out && !aligned16(L.xq_out)) || (L.d_out && !aligned16(L.d_out))) return SBL_ERR_ALIGNMENT;
            chain = true;
        } else {
            if (!L.xq || !L.d) return SBL_ERR_INVALID_ARG;
            if (!aligned16(L.xq) || !aligned16(L.d)) return SBL_ERR_ALIGNMENT;
        }
        // as many 16-row tiles per item (4, 2 or 1) as one stage holds
        const int32_t tiles = 64 * (K / 4) <= kGvStageBytes ? 4 : 32 * (K / 4) <= kGvStageBytes ? 2 : 1;
        const int32_t item_rows = 16 * tiles;
        GvProblem &g = a.p[i];
        g.pk2 = L.pk2;
        g.gamma = L.gamma;
        g.d = ch ? nullptr : L.d;
        g.y = L.y;
        g.xq_out = ch ? L.xq_out : nullptr;
        g.d_out = ch ? L.d_out : nullptr;
        g.O = O;
        g.K = K;
        g.item0 = items;
        g.flags = (L.y_is_fp32 ? kGvOutFp32 : 0) | (ch ? kGvChained : 0) |
                  ((tiles == 4 ? 2 : tiles == 2 ? 1 : 0) << kGvTilesShift);
        if (ch) a.p[i - 1].flags |= kGvPublish;
        items += (O + item_rows - 1) / item_rows;
    }
    const int64_t need = batch_workspace_layout(layers, count, T, offsets);
    if (!workspace || workspace_bytes < static_cast<size_t>(need)) return SBL_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return SBL_ERR_ALIGNMENT;
    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    for (int32_t i = 0; i < count; ++i) {
        if (layers[i].input_is_previous_output) continue;
        const int32_t owner = batch_input_owner(layers, i);
        const int64_t off = offsets[owner];
        const int32_t K = layers[i].desc.in_features;
        a.p[i].xt = reinterpret_cast<const int8_t *>(wsb + off);
        a.p[i].colsum = reinterpret_cast<const int32_t *>(wsb + off + round_up(static_cast<int64_t>(T) * K, 256));
        if (owner == i) {
            GvPrepInput &in = prep.in[prep.inputs++];
            in.xq = layers[i].xq;
            in.xt = reinterpret_cast<int8_t *>(wsb + off);
            in.colsum = reinterpret_cast<int32_t *>(wsb + off + round_up(static_cast<int64_t>(T) * K, 256));
            in.K = K;
        }
    }
    prep.T = T;
    DeviceInfo *di = nullptr;
    sbl_status st = current_device(&di);
    if (st != SBL_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_p);
    if (chain && cudaMemsetAsync(workspace, 0, static_cast<size_t>(count) * kGvSyncWords * 4, stream) != cudaSuccess)
        return SBL_ERR_CUDA;
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    if (prep.inputs > 0) {
        cudaLaunchConfig_t pc;
        memset(&pc, 0, sizeof(pc));
        pc.gridDim = dim3(static_cast<unsigned>(prep.inputs * T));
        pc.blockDim = dim3(256);
        pc.stream = stream;
        pc.attrs = pdl;
        pc.numAttrs = chain ? 0 : 1;
        if (cudaLaunchKernelEx(&pc, gemv_prep_kernel, prep) != cudaSuccess) return SBL_ERR_CUDA;
        if ((st = launch_status()) != SBL_OK) return st;
    }
    a.count = count;
    a.T = T;
    a.items = items;
    a.early_trigger = chain ? 0 : 1;
    a.sync = chain ? reinterpret_cast<uint32_t *>(wsb) : nullptr;
    a.err = di->err;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(items < di->num_sms ? items : di->num_sms));
    cfg.blockDim = dim3(kGvThreads);
    cfg.dynamicSmemBytes = kGvSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    if (chain) {
        // the CTAs wait on one another: all of them must be resident
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
    } else {
        attr[0] = pdl[0];
    }
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = T <= 8 ? cudaLaunchKernelEx(&cfg, gemv_stream_kernel<1>, a)
                                 : cudaLaunchKernelEx(&cfg, gemv_stream_kernel<2>, a);
    return e == cudaSuccess ? launch_status() : SBL_ERR_CUDA;
}

}  // extern "C"

static sbl_status backward_impl(const sbl_layer_desc *desc, const uint16_t *dY, const int8_t *Xq, const float *d,
                                int32_t T, const sbl_packed *w, void *dX, int32_t dx_is_fp32, float *dW,
                                const uint8_t *dw_keep, void *workspace, size_t workspace_bytes, void *stream_p)
{
    sbl_status st = check_desc(desc);
    if (st != SBL_OK) return st;
    if (T < 0) return SBL_ERR_SHAPE;
    if (!dY || !w || (!dX && !dW)) return SBL_ERR_INVALID_ARG;
    if (dw_keep && !dW) return SBL_ERR_INVALID_ARG;
    if (dX && (!w->bf16t || !w->gamma)) return SBL_ERR_INVALID_ARG;
    if (dW && (!Xq || !d)) return SBL_ERR_INVALID_ARG;
    if (!aligned16(dY) || (dX && (!aligned16(dX) || !aligned16(w->bf16t) || !aligned16(w->gamma))) ||
        (dW && (!aligned16(dW) || !aligned16(Xq) || !aligned16(d))) || (dw_keep && !aligned16(dw_keep)))
        return SBL_ERR_ALIGNMENT;
    if (dW && (!workspace || workspace_bytes < sbl_workspace_bytes(desc, T, SBL_OP_BACKWARD)))
        return SBL_ERR_WORKSPACE;
    if (dW && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SBL_ERR_ALIGNMENT;
    DeviceInfo *di = nullptr;
    if ((st = current_device(&di)) != SBL_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_p);
    const int32_t O = desc->out_features, K = desc->in_features;

    if (dW && T == 0) {
        if (cudaMemsetAsync(dW, 0, static_cast<size_t>(O) * K * 4, stream) != cudaSuccess) return SBL_ERR_CUDA;
    }
    if (T == 0) return SBL_OK;

    if (dX) {
        // dX[T, K] = gamma * dY[T, O] . W_eff[O, K]; B operand = W_eff^T [K, O] (K-major over O)
        GemmArgs a;
        memset(&a, 0, sizeof(a));
        a.out = dX;
        a.ldo = K;
        a.out_fp32 = dx_is_fp32 ? 1 : 0;
        a.gamma = w->gamma;
        st = launch_gemm<kKindBF16>(di, dY, static_cast<int64_t>(O) * 2, w->bf16t, static_cast<int64_t>(O) * 2,
                                    T, K, O, a, stream);
        if (st != SBL_OK) return st;
    }
    if (dW) {
        // dW[O, K] = 2^-s sum_t (dY[t, o] d_t 2^s) q[t, k]: both operands
        // transposed to [*, T_pad] fp16 so the reduction over tokens is
        // K-major; 2^s puts the largest |dY d_t| in fp16's top binade, so
        // gradients of any magnitude keep fp16's 11 bits, and the GEMM's
        // epilogue multiplies by 2^-s (both scalings are exact)
        const int64_t tp = round_up(T, 64);
        uint8_t *wsb = static_cast<uint8_t *>(workspace);
        __half *a_t = reinterpret_cast<__half *>(wsb);
        const int64_t a_bytes = round_up(static_cast<int64_t>(O) * tp * 2, 256);
        __half *b_t = reinterpret_cast<__half *>(wsb + a_bytes);
        uint32_t *pre = reinterpret_cast<uint32_t *>(wsb + a_bytes + round_up(static_cast<int64_t>(K) * tp * 2, 256));
        float *inv_pre = reinterpret_cast<float *>(pre + 1);
        if (cudaMemsetAsync(pre, 0, sizeof(uint32_t), stream) != cudaSuccess) return SBL_ERR_CUDA;
        const int64_t rows_per_cta = 8;
        const int64_t mx_grid = std::min<int64_t>((T + rows_per_cta - 1) / rows_per_cta, 8LL * di->num_sms);
        grad_absmax_kernel<<<static_cast<unsigned>(mx_grid), 256, 0, stream>>>(dY, d, T, O, pre);
        if ((st = launch_status()) != SBL_OK) return st;
        dim3 ga((O + 63) / 64, static_cast<unsigned>(tp / 64));
        transpose_to_f16_kernel<0><<<ga, 256, 0, stream>>>(dY, T, O, d, pre, inv_pre, a_t, tp);
        if ((st = launch_status()) != SBL_OK) return st;
        dim3 gb((K + 63) / 64, static_cast<unsigned>(tp / 64));
        transpose_to_f16_kernel<1><<<gb, 256, 0, stream>>>(Xq, T, K, nullptr, nullptr, nullptr, b_t, tp);
        if ((st = launch_status()) != SBL_OK) return st;
        GemmArgs a;
        memset(&a, 0, sizeof(a));
        a.out = dW;
        a.ldo = K;
        a.out_fp32 = 1;
        a.gamma = inv_pre;
        a.col_keep = dw_keep;
        a.keep_stride = round_up(K / 8, 16);
        st = launch_gemm<kKindF16>(di, a_t, tp * 2, b_t, tp * 2, O, K, static_cast<int32_t>(tp), a, stream);
        if (st != SBL_OK) return st;
    }
    return SBL_OK;
}

extern "C" {

sbl_status sbl_backward_dual_ste(const sbl_layer_desc *desc, const uint16_t *dY, const int8_t *Xq,
                                 const float *d, int32_t T, const sbl_packed *w, void *dX,
                                 int32_t dx_is_fp32, float *dW, void *workspace, size_t workspace_bytes,
                                 void *stream_p)
{
    return backward_impl(desc, dY, Xq, d, T, w, dX, dx_is_fp32, dW, nullptr, workspace, workspace_bytes, stream_p);
}

sbl_status sbl_backward_dual_ste_ex(const sbl_layer_desc *desc, const uint16_t *dY, const int8_t *Xq,
                                    const float *d, int32_t T, const sbl_packed *w, void *dX,
                                    int32_t dx_is_fp32, float *dW, const uint8_t *dw_keep, void *workspace,
                                    size_t workspace_bytes, void *stream_p)
{
    return backward_impl(desc, dY, Xq, d, T, w, dX, dx_is_fp32, dW, dw_keep, workspace, workspace_bytes, stream_p);
}

}  // extern "C"

// ------------------------------------------------ no-allocation variant --
// File-scope scratch for sbl_quantize_mask_pack_noalloc: holds the gamma
// partial sums and the finishing counter.  In host code the symbol is only a
// handle; its device address comes from cudaGetSymbolAddress, looked up once
// per device on the first call.
namespace sbl {
static_assert(SBL_NOALLOC_SCRATCH_BYTES >= (sizeof(GammaWorkspace) + 255) / 256 * 256,
              "scratch smaller than the workspace sbl_workspace_bytes asks for");
static_assert(SBL_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size must keep 256-byte granularity");
static __device__ __align__(256) uint8_t g_noalloc_scratch[SBL_NOALLOC_SCRATCH_BYTES];
static std::mutex g_noalloc_mutex;
static void *g_noalloc_ptr[kMaxDevices];

// Self-test of the bounded waits: one thread waits, through the same
// mbar_wait every kernel uses, on a fresh mbarrier that nothing arrives at.
// After kWaitLimitNs the wait records SBL_DEVICE_ERROR_SELFTEST and the
// kernel returns.  No copy, MMA or tensor memory is outstanding when it does.
static_assert((SBL_DEVICE_ERROR_SELFTEST & (kErrGemmProducer | kErrGemmMma | kErrGemmEpilogue | kErrDecode |
                                            kErrPack | kErrGemv)) == 0,
              "the self-test bit is distinct from every kernel family's bit");
__global__ void __launch_bounds__(32) wait_expiry_kernel(uint32_t *err)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    const uint32_t b = smem_addr(&bar);
    mbar_init(b, 1);
    fence_barrier_init();
    mbar_wait(b, 0, err, SBL_DEVICE_ERROR_SELFTEST);
}
}  // namespace sbl

extern "C" {

sbl_status sbl_quantize_mask_pack_noalloc(const sbl_layer_desc *desc, const float *W, uint32_t formats,
                                          const sbl_packed *out, void *stream)
{
    sbl_status st = check_desc(desc);
    if (st != SBL_OK) return st;
    // the scratch holds kGammaMaxPartials partial sums of kGammaBlock weights
    const int64_t count = static_cast<int64_t>(desc->out_features) * desc->in_features;
    if (count > static_cast<int64_t>(kGammaBlock) * kGammaMaxPartials) return SBL_ERR_SHAPE;
    // an sm_100 device first (other devices get SBL_ERR_DEVICE, as every call)
    DeviceInfo *di = nullptr;
    if ((st = current_device(&di)) != SBL_OK) return st;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SBL_ERR_DEVICE;
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mutex);
        if (!g_noalloc_ptr[dev]) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
                cudaGetLastError();  // leave no pending error for the thread's next launch check
                return SBL_ERR_CUDA;
            }
            g_noalloc_ptr[dev] = p;
        }
        scratch = g_noalloc_ptr[dev];
    }
    return sbl_quantize_mask_pack(desc, W, formats, out, scratch, SBL_NOALLOC_SCRATCH_BYTES, stream);
}

sbl_status sbl_selftest_wait_expiry(void *stream)
{
    DeviceInfo *di = nullptr;
    sbl_status st = current_device(&di);
    if (st != SBL_OK) return st;
    wait_expiry_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(di->err);
    return launch_status();
}

sbl_status sbl_device_error(uint32_t *code, int32_t clear)
{
    if (!code) return SBL_ERR_INVALID_ARG;
    DeviceInfo *di = nullptr;
    sbl_status st = current_device(&di);
    if (st != SBL_OK) return st;
    if (cudaDeviceSynchronize() != cudaSuccess) return SBL_ERR_CUDA;
    if (cudaMemcpy(code, di->err, sizeof(uint32_t), cudaMemcpyDeviceToHost) != cudaSuccess) return SBL_ERR_CUDA;
    if (clear && cudaMemset(di->err, 0, sizeof(uint32_t)) != cudaSuccess) return SBL_ERR_CUDA;
    return SBL_OK;
}

}  // extern "C"
