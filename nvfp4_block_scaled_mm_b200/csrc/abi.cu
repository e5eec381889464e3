// C ABI of the NVFP4 + LoRA GEMM library (declared in include/nvfp4lora.h).
//
// Host side: argument rules (flashinfer.gemm.mm_nvfp4_lora, Notes: Shape rules; Parameters),
// adapter pins and stale checks (Parameters: lora_adapter; Notes: CUDA graphs), the eager
// prepare's single host read and checks (prepare_nvfp4_lora_adapter, Parameters: alpha,
// Returns), TMA descriptor encoding, and kernel launch.  Every rule is checked before any
// CUDA call, so a rejected call enqueues nothing.  This is the library's only translation
// unit: it includes the kernels and the device error word they set.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <set>
#include <string>

#include "../../include/nvfp4lora.h"
#include "bgmv.cuh"
#include "fold.cuh"
#include "gemm.cuh"
#include "gemm_decode.cuh"
#include "gemm_pair.cuh"
#include "ptx.cuh"
#include "quantize.cuh"
#include "selftest.cuh"

namespace nvfp4lora {
namespace {

thread_local std::string t_last_error;

nvfp4lora_status fail(nvfp4lora_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return st;
}

nvfp4lora_status cuda_fail(cudaError_t e, const char* what) {
    return fail(NVFP4LORA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ---------------------------------------------------------------------------------------
// device facts, cached per device
// ---------------------------------------------------------------------------------------

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool init = false;
    bool supported = false;
    int sms = 0;
    int major = 0, minor = 0;
    std::set<const void*> smem_attr_set;   // kernels whose dynamic shared memory limit is raised
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

nvfp4lora_status device_info(int* dev_out, DeviceInfo** info_out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(NVFP4LORA_ERR_CUDA, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.init) {
        if ((e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute");
        d.supported = (d.major == 10 && d.minor == 0);
        d.init = true;
    }
    if (!d.supported)
        return fail(NVFP4LORA_ERR_UNSUPPORTED_ARCH,
                    "device %d is sm_%d%d; this library runs on sm_100 (B200) only", dev, d.major, d.minor);
    *dev_out = dev;
    *info_out = &d;
    return NVFP4LORA_OK;
}

template <typename Kernel>
nvfp4lora_status ensure_smem_attr(DeviceInfo* info, Kernel kernel, int smem, bool max_carveout = true) {
    std::lock_guard<std::mutex> lock(g_mu);
    const void* key = reinterpret_cast<const void*>(kernel);
    if (info->smem_attr_set.count(key)) return NVFP4LORA_OK;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    // the whole unified L1 / shared array as shared memory, so co-resident CTAs fit
    if (e == cudaSuccess && max_carveout)
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    info->smem_attr_set.insert(key);
    return NVFP4LORA_OK;
}

// ---------------------------------------------------------------------------------------
// TMA descriptors
// ---------------------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
cudaError_t g_encode_err = cudaSuccess;

nvfp4lora_status get_encoder(PFN_cuTensorMapEncodeTiled_v12000* out) {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        g_encode_err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (g_encode_err == cudaSuccess && q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (g_encode == nullptr)
        return fail(NVFP4LORA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)",
                    cudaGetErrorString(g_encode_err));
    *out = g_encode;
    return NVFP4LORA_OK;
}

// 2-D row-major tensor [rows, cols] of `esize`-byte elements, read in boxes of
// box_cols x box_rows with the 128-byte swizzle; out-of-range elements read as zero.
// The LoRA operands d [M, r] and lora_b / b_folded [N, r] of the tiled kernels are read with no L2
// promotion.  Their boxes are 64 columns wide and zero-filled past r; where r is not a multiple of
// 16 a row's in-bounds part ends inside a 32-byte sector, and with 256-byte promotion those loads
// arrived late enough to stall the tile's end: raw path, M = 256, N = 14336, K = 4096, r = 8 ran
// 18.3 us on the SM-pair kernel with promotion and 16.9 without (r = 16: 14.9 either way).
constexpr CUtensorMapL2promotion kLoraPromotion = CU_TENSOR_MAP_L2_PROMOTION_NONE;

nvfp4lora_status encode_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int esize,
                           uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
                           CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B,
                           CUtensorMapL2promotion promotion = CU_TENSOR_MAP_L2_PROMOTION_L2_256B) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
    nvfp4lora_status st = get_encoder(&enc);
    if (st != NVFP4LORA_OK) return st;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * (uint64_t)esize};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promotion, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(NVFP4LORA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    return NVFP4LORA_OK;
}

// 3-D view of a row-major [rows, cols] uint8 matrix as (128-byte chunk, row, chunk index), used
// to name one 128-row block across several K chunks in a single box (L2 prefetch only).
nvfp4lora_status encode_rows_by_chunks(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                                       uint32_t box_rows, uint32_t box_chunks) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
    nvfp4lora_status st = get_encoder(&enc);
    if (st != NVFP4LORA_OK) return st;
    cuuint64_t dims[3] = {128, rows, cols / 128};
    cuuint64_t strides[2] = {cols, 128};
    cuuint32_t box[3] = {128, box_rows, box_chunks};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(NVFP4LORA_ERR_CUDA, "cuTensorMapEncodeTiled (3-D) failed (CUresult %d)", (int)r);
    return NVFP4LORA_OK;
}

// ---------------------------------------------------------------------------------------
// argument rules
// ---------------------------------------------------------------------------------------

constexpr int64_t kMaxDim = (int64_t)1 << 30;   // keeps every tile coordinate in int32
constexpr int64_t kMaxK = (int64_t)1 << 20;

nvfp4lora_status check_rank(int64_t r) {
    if (r < 8 || r > 128 || r % 8 != 0)
        return fail(NVFP4LORA_ERR_INVALID_ARG,
                    "LoRA rank r = %lld: r must be a multiple of 8 in [8, 128]", (long long)r);
    return NVFP4LORA_OK;
}

nvfp4lora_status check_base(const uint8_t* a, const uint8_t* b, const uint8_t* a_sf, int64_t a_sf_bytes,
                            const uint8_t* b_sf, int64_t b_sf_bytes, const float* alpha,
                            const uint16_t* bias, const uint16_t* out, int64_t M, int64_t N, int64_t K) {
    if (M < 1) return fail(NVFP4LORA_ERR_INVALID_ARG, "M = %lld: M >= 1 is required", (long long)M);
    if (N < 1) return fail(NVFP4LORA_ERR_INVALID_ARG, "N = %lld: N >= 1 is required", (long long)N);
    if (K < 256 || K % 256 != 0)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "K = %lld: K must be a positive multiple of 256", (long long)K);
    if (M > kMaxDim || N > kMaxDim || K > kMaxK)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "M, N <= 2^30 and K <= 2^20 are required");
    if (!a || !b || !a_sf || !b_sf || !alpha || !out)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "a, b, a_sf, b_sf, alpha and out must be non-null");
    if (!aligned(a, 16) || !aligned(b, 16) || !aligned(a_sf, 16) || !aligned(b_sf, 16) || !aligned(out, 16))
        return fail(NVFP4LORA_ERR_INVALID_ARG, "a, b, a_sf, b_sf and out must be 16-byte aligned");
    if (!aligned(alpha, 4)) return fail(NVFP4LORA_ERR_INVALID_ARG, "alpha must be 4-byte aligned");
    if (bias && !aligned(bias, 2)) return fail(NVFP4LORA_ERR_INVALID_ARG, "bias must be 2-byte aligned");
    const int64_t need_a = (M + 127) / 128 * 128 * (K / 16);
    const int64_t need_b = (N + 127) / 128 * 128 * (K / 16);
    if (a_sf_bytes < need_a)
        return fail(NVFP4LORA_ERR_INVALID_ARG,
                    "a_sf has %lld bytes; the 128x4 layout with rows padded to 128 needs %lld",
                    (long long)a_sf_bytes, (long long)need_a);
    if (b_sf_bytes < need_b)
        return fail(NVFP4LORA_ERR_INVALID_ARG,
                    "b_sf has %lld bytes; the 128x4 layout with rows padded to 128 needs %lld",
                    (long long)b_sf_bytes, (long long)need_b);
    return NVFP4LORA_OK;
}

// ---------------------------------------------------------------------------------------
// GEMM launch
// ---------------------------------------------------------------------------------------

constexpr int kStages = 3;

// The tiled kernels split their registers by warpgroup (setmaxnreg); the split assumes the per-
// thread count the compiler gave the kernel at launch.  A smaller count would leave the epilogue
// warpgroups waiting for registers that never come, so a build that differs is refused here.
template <typename Kernel>
nvfp4lora_status check_split_regs(Kernel kernel, int expected, std::atomic<int>& checked, const char* what) {
    if (checked.load(std::memory_order_relaxed)) return NVFP4LORA_OK;
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return cuda_fail(e, what);
    if (fa.numRegs != expected)
        return fail(NVFP4LORA_ERR_CUDA, "%s built with %d registers per thread, its register split assumes %d", what,
                    fa.numRegs, expected);
    checked.store(1, std::memory_order_relaxed);
    return NVFP4LORA_OK;
}

template <Mode MODE>
nvfp4lora_status launch_gemm(const uint8_t* a, const uint8_t* b, const uint8_t* a_sf, const uint8_t* b_sf,
                             const float* alpha, const float* scale, const uint16_t* d,
                             const uint16_t* lb, int64_t r, const uint16_t* bias, uint16_t* out,
                             int64_t M, int64_t N, int64_t K, cudaStream_t stream) {
    int dev = 0;
    DeviceInfo* info = nullptr;
    nvfp4lora_status st = device_info(&dev, &info);
    if (st != NVFP4LORA_OK) return st;

    auto kernel = nvfp4_gemm_kernel<kStages, MODE>;
    constexpr int smem = GemmSmem<kStages>::DYN_BYTES;
    if ((st = ensure_smem_attr(info, kernel, smem)) != NVFP4LORA_OK) return st;
    static std::atomic<int> regs_ok{0};            // one per instantiation
    if ((st = check_split_regs(kernel, kGemmRegsLaunch, regs_ok, "GEMM")) != NVFP4LORA_OK) return st;

    CUtensorMap tm_a, tm_b, tm_d, tm_lb, tm_out;
    std::memset(&tm_d, 0, sizeof(tm_d));
    std::memset(&tm_lb, 0, sizeof(tm_lb));
    std::memset(&tm_out, 0, sizeof(tm_out));
    if ((st = encode_2d(&tm_a, a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, M, 128, kTileM)) != NVFP4LORA_OK) return st;
    if ((st = encode_2d(&tm_b, b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, N, 128, kTileN)) != NVFP4LORA_OK) return st;
    if (MODE != Mode::Off) {
        if ((st = encode_2d(&tm_d, d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, r, M, 64, kTileM, CU_TENSOR_MAP_SWIZZLE_128B, kLoraPromotion)) != NVFP4LORA_OK) return st;
        if ((st = encode_2d(&tm_lb, lb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, r, N, 64, kTileN, CU_TENSOR_MAP_SWIZZLE_128B, kLoraPromotion)) != NVFP4LORA_OK) return st;
    }
    // rows of out 16-byte aligned: the epilogue writes 32 x 32 bf16 boxes with TMA stores
    const bool vec_out = (N % 8 == 0 && (bias == nullptr || aligned(bias, 16)));
    if (vec_out &&
        (st = encode_2d(&tm_out, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, M, kOutBoxCols, kOutBoxRows,
                        CU_TENSOR_MAP_SWIZZLE_NONE)) != NVFP4LORA_OK)
        return st;

    GemmArgs args;
    args.a_sf = a_sf;
    args.b_sf = b_sf;
    args.alpha = alpha;
    args.scale = scale;
    args.bias = bias;
    args.out = out;
    args.M = (int)M;
    args.N = (int)N;
    args.K = (int)K;
    args.r = (int)r;
    args.m_tiles = (int)((M + kTileM - 1) / kTileM);
    args.n_tiles = (int)((N + kTileN - 1) / kTileN);
    const int64_t tiles = (int64_t)args.m_tiles * args.n_tiles;
    if (tiles > INT32_MAX) return fail(NVFP4LORA_ERR_INVALID_ARG, "too many output tiles (M x N too large)");
    args.num_tiles = (int)tiles;
    args.k_stages = (int)(K / 256);
    args.sf_atoms_k = (int)(K / 64);
    args.sf_row_blocks_b = (int)((N + 127) / 128);
    args.vec_out = vec_out ? 1 : 0;
    args.m_indptr = nullptr;
    args.num_experts = 0;

    const int grid = (int)std::min<int64_t>(tiles, info->sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, tm_a, tm_b, tm_d, tm_lb, tm_out, args);
    if (e != cudaSuccess) return cuda_fail(e, "GEMM launch");
    return NVFP4LORA_OK;
}

// Grouped call (nvfp4lora_grouped_mm): the single-SM tiled kernel over 128-row blocks whose expert
// comes from m_indptr on the device.  `rows` is the row count of a, d and out; b and lora_b are
// [E * N, .] row-major; alpha is [E].
template <Mode MODE>
nvfp4lora_status launch_gemm_grouped(const uint8_t* a, const uint8_t* b, const uint8_t* a_sf, const uint8_t* b_sf,
                                     const int* m_indptr, int64_t E, const float* alpha, const float* scale,
                                     const uint16_t* d, const uint16_t* lb, int64_t r, const uint16_t* bias,
                                     uint16_t* out, int64_t rows, int64_t N, int64_t K, cudaStream_t stream) {
    int dev = 0;
    DeviceInfo* info = nullptr;
    nvfp4lora_status st = device_info(&dev, &info);
    if (st != NVFP4LORA_OK) return st;

    auto kernel = nvfp4_gemm_kernel<kStages, MODE, true>;
    constexpr int smem = GemmSmem<kStages>::DYN_BYTES;
    if ((st = ensure_smem_attr(info, kernel, smem)) != NVFP4LORA_OK) return st;
    static std::atomic<int> regs_ok{0};            // one per instantiation
    if ((st = check_split_regs(kernel, kGemmRegsLaunch, regs_ok, "grouped GEMM")) != NVFP4LORA_OK) return st;

    CUtensorMap tm_a, tm_b, tm_d, tm_lb, tm_out;
    std::memset(&tm_d, 0, sizeof(tm_d));
    std::memset(&tm_lb, 0, sizeof(tm_lb));
    std::memset(&tm_out, 0, sizeof(tm_out));
    if ((st = encode_2d(&tm_a, a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, rows, 128, kTileM)) != NVFP4LORA_OK) return st;
    if ((st = encode_2d(&tm_b, b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, E * N, 128, kTileN)) != NVFP4LORA_OK) return st;
    if (MODE != Mode::Off) {
        if ((st = encode_2d(&tm_d, d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, r, rows, 64, kTileM, CU_TENSOR_MAP_SWIZZLE_128B, kLoraPromotion)) != NVFP4LORA_OK) return st;
        if ((st = encode_2d(&tm_lb, lb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, r, E * N, 64, kTileN, CU_TENSOR_MAP_SWIZZLE_128B, kLoraPromotion)) != NVFP4LORA_OK) return st;
    }
    const bool vec_out = (N % 8 == 0 && (bias == nullptr || aligned(bias, 16)));
    if (vec_out &&
        (st = encode_2d(&tm_out, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, rows, kOutBoxCols, kOutBoxRows,
                        CU_TENSOR_MAP_SWIZZLE_NONE)) != NVFP4LORA_OK)
        return st;

    GemmArgs args;
    args.a_sf = a_sf;
    args.b_sf = b_sf;
    args.alpha = alpha;
    args.scale = scale;
    args.bias = bias;
    args.out = out;
    args.M = (int)rows;
    args.N = (int)N;
    args.K = (int)K;
    args.r = (int)r;
    args.m_tiles = (int)((rows + kTileM - 1) / kTileM);     // bound: the kernel reads m_indptr[E]
    args.n_tiles = (int)((N + kTileN - 1) / kTileN);
    const int64_t tiles = (int64_t)args.m_tiles * args.n_tiles;
    if (tiles > INT32_MAX) return fail(NVFP4LORA_ERR_INVALID_ARG, "too many output tiles (rows x N too large)");
    args.num_tiles = (int)tiles;
    args.k_stages = (int)(K / 256);
    args.sf_atoms_k = (int)(K / 64);
    args.sf_row_blocks_b = (int)((N + 127) / 128);         // per expert
    args.vec_out = vec_out ? 1 : 0;
    args.m_indptr = m_indptr;
    args.num_experts = (int)E;

    const int grid = (int)std::min<int64_t>(tiles, info->sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, tm_a, tm_b, tm_d, tm_lb, tm_out, args);
    if (e != cudaSuccess) return cuda_fail(e, "grouped GEMM launch");
    return NVFP4LORA_OK;
}

// ---------------------------------------------------------------------------------------
// decode launch (M <= kDecodeMaxM): swapped operands, split-K over a cluster
// ---------------------------------------------------------------------------------------

constexpr int kDecodeMaxM = 32;

// Largest cluster split S <= max_s (a power of two) that keeps n_tiles * S CTAs within one wave
// and divides the K stages.
int decode_splits(int n_tiles, int k_stages, int sms, int max_s) {
    for (int s = max_s; s > 1; s >>= 1)
        if (k_stages % s == 0 && (int64_t)n_tiles * s <= sms) return s;
    return 1;
}

// STAGES ring slots (all of a split's K stages in flight where they fit); MAXS - 1 peer partial
// slots plus one for the LoRA accumulator on rank 0.
template <int MT, int STAGES, int MAXS, Mode MODE>
nvfp4lora_status launch_decode_plan(DeviceInfo* info, int splits, const uint8_t* a, const uint8_t* b,
                                    const uint8_t* a_sf, const uint8_t* b_sf, const float* alpha,
                                    const float* scale, const uint16_t* d, const uint16_t* lb, int64_t r,
                                    const uint16_t* bias, uint16_t* out, int64_t M, int64_t N, int64_t K,
                                    cudaStream_t stream) {
    nvfp4lora_status st;
    auto kernel = nvfp4_decode_kernel<MT, STAGES, MAXS, MODE>;
    constexpr int smem = DecodeSmem<MT, STAGES, MAXS>::DYN_BYTES;
    if ((st = ensure_smem_attr(info, kernel, smem)) != NVFP4LORA_OK) return st;

    CUtensorMap tm_a, tm_b, tm_d, tm_lb;
    std::memset(&tm_d, 0, sizeof(tm_d));
    std::memset(&tm_lb, 0, sizeof(tm_lb));
    if ((st = encode_2d(&tm_a, a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, M, 128, MT)) != NVFP4LORA_OK) return st;
    if ((st = encode_2d(&tm_b, b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, N, 128, 128)) != NVFP4LORA_OK) return st;
    if (MODE != Mode::Off) {
        if ((st = encode_2d(&tm_d, d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, r, M, 64, MT)) != NVFP4LORA_OK) return st;
        if ((st = encode_2d(&tm_lb, lb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, r, N, 64, 128)) != NVFP4LORA_OK) return st;
    }
    DecodeArgs args;
    args.a_sf = a_sf;
    args.b_sf = b_sf;
    args.alpha = alpha;
    args.scale = scale;
    args.lb = lb;
    args.bias = bias;
    args.out = out;
    args.M = (int)M;
    args.N = (int)N;
    args.K = (int)K;
    args.r = (int)r;
    args.n_tiles = (int)((N + 127) / 128);
    const int k_stages = (int)(K / 256);
    args.splits = splits;
    args.stages_per_split = k_stages / args.splits;
    args.sf_atoms_k = (int)(K / 64);
    args.sf_row_blocks_b = (int)((N + 127) / 128);

    CUtensorMap tm_b3;
    // one prefetch box covers up to 8 chunks (128 KB, within the tensor-map box limit)
    args.pf_chunks = std::min(args.stages_per_split, 8);
    if ((st = encode_rows_by_chunks(&tm_b3, b, K / 2, N, 128, args.pf_chunks)) != NVFP4LORA_OK) return st;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(args.n_tiles, args.splits);
    cfg.blockDim = dim3(kDecodeThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (args.splits > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = 1;
        attr[1].val.clusterDim.y = args.splits;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, tm_a, tm_b, tm_d, tm_lb, tm_b3, args);
    if (e != cudaSuccess) return cuda_fail(e, "decode GEMM launch");
    return NVFP4LORA_OK;
}

// A split cluster (S > 1) streams few K stages per CTA: 4 slots hold them all at the workload
// shapes.  Without a split (many weight row blocks) one CTA streams the whole of K, and the ring is
// as deep as shared memory allows, since a CTA's streaming rate is its bytes in flight over the
// memory latency (M = 1, N = 14336, K = 4096: 10.0 us per call with 4 slots, 8.6 with 8).
template <int MT, Mode MODE>
nvfp4lora_status launch_decode_mt(DeviceInfo* info, const uint8_t* a, const uint8_t* b, const uint8_t* a_sf,
                                  const uint8_t* b_sf, const float* alpha, const float* scale, const uint16_t* d,
                                  const uint16_t* lb, int64_t r, const uint16_t* bias, uint16_t* out,
                                  int64_t M, int64_t N, int64_t K, cudaStream_t stream) {
    constexpr int MAXS = 4;
    constexpr int DEEP = (MT == 16) ? 8 : 6;
    const int n_tiles = (int)((N + 127) / 128);
    const int splits = decode_splits(n_tiles, (int)(K / 256), info->sms, MAXS);
    if (splits > 1)
        return launch_decode_plan<MT, 4, MAXS, MODE>(info, splits, a, b, a_sf, b_sf, alpha, scale, d, lb, r, bias,
                                                     out, M, N, K, stream);
    return launch_decode_plan<MT, DEEP, 1, MODE>(info, 1, a, b, a_sf, b_sf, alpha, scale, d, lb, r, bias, out, M,
                                                 N, K, stream);
}

template <Mode MODE>
nvfp4lora_status launch_decode(const uint8_t* a, const uint8_t* b, const uint8_t* a_sf, const uint8_t* b_sf,
                               const float* alpha, const float* scale, const uint16_t* d, const uint16_t* lb,
                               int64_t r, const uint16_t* bias, uint16_t* out, int64_t M, int64_t N, int64_t K,
                               cudaStream_t stream) {
    int dev = 0;
    DeviceInfo* info = nullptr;
    nvfp4lora_status st = device_info(&dev, &info);
    if (st != NVFP4LORA_OK) return st;
    if (M <= 16)
        return launch_decode_mt<16, MODE>(info, a, b, a_sf, b_sf, alpha, scale, d, lb, r, bias, out, M, N, K, stream);
    return launch_decode_mt<32, MODE>(info, a, b, a_sf, b_sf, alpha, scale, d, lb, r, bias, out, M, N, K, stream);
}

// ---------------------------------------------------------------------------------------
// SM-pair tiled launch: clusters of 2 CTAs, 256 x 256 tiles
// ---------------------------------------------------------------------------------------

template <Mode MODE>
nvfp4lora_status launch_gemm_pair(const uint8_t* a, const uint8_t* b, const uint8_t* a_sf, const uint8_t* b_sf,
                                  const float* alpha, const float* scale, const uint16_t* d, const uint16_t* lb,
                                  int64_t r, const uint16_t* bias, uint16_t* out, int64_t M, int64_t N, int64_t K,
                                  cudaStream_t stream) {
    int dev = 0;
    DeviceInfo* info = nullptr;
    nvfp4lora_status st = device_info(&dev, &info);
    if (st != NVFP4LORA_OK) return st;
    auto kernel = nvfp4_gemm_pair_kernel<kPairStages, MODE>;
    constexpr int smem = PairSmem<kPairStages>::DYN_BYTES;
    if ((st = ensure_smem_attr(info, kernel, smem)) != NVFP4LORA_OK) return st;

    static std::atomic<int> regs_ok{0};            // one per instantiation
    if ((st = check_split_regs(kernel, kPairRegsLaunch, regs_ok, "pair GEMM")) != NVFP4LORA_OK) return st;

    CUtensorMap tm_a, tm_b, tm_d, tm_lb, tm_out;
    std::memset(&tm_d, 0, sizeof(tm_d));
    std::memset(&tm_lb, 0, sizeof(tm_lb));
    std::memset(&tm_out, 0, sizeof(tm_out));
    if ((st = encode_2d(&tm_a, a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, M, 128, 128)) != NVFP4LORA_OK) return st;
    if ((st = encode_2d(&tm_b, b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, N, 128, 128)) != NVFP4LORA_OK) return st;
    if (MODE != Mode::Off) {
        if ((st = encode_2d(&tm_d, d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, r, M, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B, kLoraPromotion)) != NVFP4LORA_OK) return st;
        // raw: per N-half, 64 of each CTA's 128 lora_b rows; prepared: all 128
        const int lb_rows = (MODE == Mode::Raw) ? 64 : 128;
        if ((st = encode_2d(&tm_lb, lb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, r, N, 64, lb_rows, CU_TENSOR_MAP_SWIZZLE_128B, kLoraPromotion)) != NVFP4LORA_OK) return st;
    }
    const bool vec_out = (N % 8 == 0 && (bias == nullptr || aligned(bias, 16)));
    if (vec_out &&
        (st = encode_2d(&tm_out, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, M, kOutBoxCols, kOutBoxRows,
                        CU_TENSOR_MAP_SWIZZLE_NONE)) != NVFP4LORA_OK)
        return st;

    PairArgs args;
    args.alpha = alpha;
    args.scale = scale;
    args.a_sf = a_sf;
    args.b_sf = b_sf;
    args.bias = bias;
    args.out = out;
    args.M = (int)M;
    args.N = (int)N;
    args.K = (int)K;
    args.r = (int)r;
    args.m_pairs = (int)((M + kPairTileM - 1) / kPairTileM);
    args.n_tiles = (int)((N + kTileN - 1) / kTileN);
    const int64_t tiles = (int64_t)args.m_pairs * args.n_tiles;
    if (tiles > INT32_MAX) return fail(NVFP4LORA_ERR_INVALID_ARG, "too many output tiles (M x N too large)");
    args.num_tiles = (int)tiles;
    args.k_stages = (int)(K / 256);
    args.sf_atoms_k = (int)(K / 64);
    args.sf_row_blocks_a = (int)((M + 127) / 128);
    args.sf_row_blocks_b = (int)((N + 127) / 128);
    args.vec_out = vec_out ? 1 : 0;

    const int pairs = (int)std::min<int64_t>(tiles, info->sms / 2);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(kPairThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, tm_a, tm_b, tm_d, tm_lb, tm_out, args);
    if (e != cudaSuccess) return cuda_fail(e, "pair GEMM launch");
    return NVFP4LORA_OK;
}

// The SM-pair kernel measured faster than the single-SM one on every shape with M >= 128 where both
// run the same number of waves (2-6 % at M = 128..384, N = 14336; 20-30 % at M >= 2048 since it
// stages scales with register stores and halves each SM's B traffic), and slower where its 256-row
// tiles add a wave (4736 x 1024 x 8192: 31.8 against 20.9 us).  It is used from M = 128 on when its
// wave count over the SM pairs is no larger than the single-SM kernel's over the SMs.
//
// One exception, measured on the raw path with a rank below 32 that is not a multiple of 16 (the
// narrow-row LoRA loads above) at M <= 256: 256 x 14336 x 4096, r = 8 ran 15.5 us on the single-SM
// kernel against 16.9 on the pair kernel (128 rows: 15.2 against 16.1), so those calls stay on the
// single-SM kernel.
bool use_pair_kernel(int64_t M, int64_t N, bool raw, int64_t r) {
    if (M < 128) return false;
    if (raw && r % 16 != 0 && r < 32 && M <= 256) return false;
    int dev = 0;
    DeviceInfo* info = nullptr;
    if (device_info(&dev, &info) != NVFP4LORA_OK) return false;
    const int64_t n_tiles = (N + kTileN - 1) / kTileN;
    const int64_t t1 = (M + kTileM - 1) / kTileM * n_tiles, t2 = (M + kPairTileM - 1) / kPairTileM * n_tiles;
    const int64_t sms = info->sms, pairs = info->sms / 2;
    return (t2 + pairs - 1) / pairs <= (t1 + sms - 1) / sms;
}

// Chooses the decode kernel for M <= 32, the SM-pair kernel where use_pair_kernel says so, and the
// single-SM tiled kernel otherwise.
template <Mode MODE>
nvfp4lora_status launch(const uint8_t* a, const uint8_t* b, const uint8_t* a_sf, const uint8_t* b_sf,
                        const float* alpha, const float* scale, const uint16_t* d, const uint16_t* lb, int64_t r,
                        const uint16_t* bias, uint16_t* out, int64_t M, int64_t N, int64_t K, cudaStream_t stream) {
    if (M <= kDecodeMaxM)
        return launch_decode<MODE>(a, b, a_sf, b_sf, alpha, scale, d, lb, r, bias, out, M, N, K, stream);
    if (use_pair_kernel(M, N, MODE == Mode::Raw, r))
        return launch_gemm_pair<MODE>(a, b, a_sf, b_sf, alpha, scale, d, lb, r, bias, out, M, N, K, stream);
    return launch_gemm<MODE>(a, b, a_sf, b_sf, alpha, scale, d, lb, r, bias, out, M, N, K, stream);
}

// ---------------------------------------------------------------------------------------
// fold launch
// ---------------------------------------------------------------------------------------

nvfp4lora_status launch_fold(const uint16_t* lora_b, const float* lora_scale, const float* alpha,
                             uint16_t* b_folded, float* ratio, int64_t N, int64_t r, cudaStream_t stream) {
    int dev = 0;
    DeviceInfo* info = nullptr;
    nvfp4lora_status st = device_info(&dev, &info);
    if (st != NVFP4LORA_OK) return st;
    const int64_t groups = N * r / 8;
    const int64_t want = (groups + kFoldThreads - 1) / kFoldThreads;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)info->sms * 8));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kFoldThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, fold_kernel, lora_b, lora_scale, alpha, b_folded, ratio, groups);
    if (e != cudaSuccess) return cuda_fail(e, "fold launch");
    return NVFP4LORA_OK;
}

nvfp4lora_status check_fold_args(const uint16_t* lora_b, const float* lora_scale, const float* alpha,
                                  int64_t N, int64_t r, const uint16_t* b_folded, const float* ratio) {
    if (N < 1) return fail(NVFP4LORA_ERR_INVALID_ARG, "N = %lld: N >= 1 is required", (long long)N);
    if (N > kMaxDim) return fail(NVFP4LORA_ERR_INVALID_ARG, "N <= 2^30 is required");
    nvfp4lora_status st = check_rank(r);
    if (st != NVFP4LORA_OK) return st;
    if (!lora_b || !lora_scale || !alpha || !b_folded || !ratio)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "lora_b, lora_scale, alpha, b_folded and ratio must be non-null");
    if (!aligned(lora_b, 16) || !aligned(b_folded, 16))
        return fail(NVFP4LORA_ERR_INVALID_ARG, "lora_b and b_folded must be 16-byte aligned");
    if (!aligned(lora_scale, 4) || !aligned(alpha, 4) || !aligned(ratio, 4))
        return fail(NVFP4LORA_ERR_INVALID_ARG, "lora_scale, alpha and ratio must be 4-byte aligned");
    if (ratio == lora_scale || ratio == alpha)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "ratio must not alias lora_scale or alpha");
    return NVFP4LORA_OK;
}

}  // namespace
}  // namespace nvfp4lora

using namespace nvfp4lora;

extern "C" {

nvfp4lora_status nvfp4lora_mm(const uint8_t* a, const uint8_t* b, const uint8_t* a_sf, int64_t a_sf_bytes,
                              const uint8_t* b_sf, int64_t b_sf_bytes, const float* alpha,
                              const uint16_t* d, const uint16_t* lora_b, const float* lora_scale, int64_t r,
                              const uint16_t* bias, uint16_t* out, int64_t M, int64_t N, int64_t K,
                              nvfp4lora_stream stream) {
    t_last_error.clear();
    nvfp4lora_status st = check_base(a, b, a_sf, a_sf_bytes, b_sf, b_sf_bytes, alpha, bias, out, M, N, K);
    if (st != NVFP4LORA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (lora_scale == nullptr)
        return launch<Mode::Off>(a, b, a_sf, b_sf, alpha, nullptr, nullptr, nullptr, 0, bias, out, M, N, K, s);
    if ((st = check_rank(r)) != NVFP4LORA_OK) return st;
    if (!d || !lora_b) return fail(NVFP4LORA_ERR_INVALID_ARG, "lora_scale given: d and lora_b must be non-null");
    if (!aligned(d, 16) || !aligned(lora_b, 16))
        return fail(NVFP4LORA_ERR_INVALID_ARG, "d and lora_b must be 16-byte aligned");
    if (!aligned(lora_scale, 4)) return fail(NVFP4LORA_ERR_INVALID_ARG, "lora_scale must be 4-byte aligned");
    return launch<Mode::Raw>(a, b, a_sf, b_sf, alpha, lora_scale, d, lora_b, r, bias, out, M, N, K, s);
}

nvfp4lora_status nvfp4lora_prepare(const uint16_t* lora_b, const float* lora_scale, const float* alpha,
                                   int64_t N, int64_t r, uint16_t* b_folded, float* ratio,
                                   uint64_t src_version, nvfp4lora_adapter* adapter_out,
                                   nvfp4lora_stream stream) {
    t_last_error.clear();
    if (!adapter_out) return fail(NVFP4LORA_ERR_INVALID_ARG, "adapter_out must be non-null");
    nvfp4lora_status st = check_fold_args(lora_b, lora_scale, alpha, N, r, b_folded, ratio);
    if (st != NVFP4LORA_OK) return st;
    int dev = 0;
    DeviceInfo* info = nullptr;
    if ((st = device_info(&dev, &info)) != NVFP4LORA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // The single host read of the adapter switch: (lora_scale, alpha).
    float host[2] = {0.0f, 0.0f};
    cudaError_t e = cudaMemcpyAsync(&host[0], lora_scale, sizeof(float), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(&host[1], alpha, sizeof(float), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "reading lora_scale and alpha");
    if (host[1] == 0.0f)
        return fail(NVFP4LORA_ERR_ALPHA_ZERO, "alpha == 0: lora_scale / alpha is undefined "
                                              "(the alpha == 0 LoRA-only call is the raw path)");
    volatile float q = host[0] / host[1];
    if (!std::isfinite((float)q))
        return fail(NVFP4LORA_ERR_ALPHA_ZERO, "lora_scale / alpha = %g is not finite", (double)q);
    if ((st = launch_fold(lora_b, lora_scale, alpha, b_folded, ratio, N, r, s)) != NVFP4LORA_OK) return st;
    adapter_out->b_folded = b_folded;
    adapter_out->ratio = ratio;
    adapter_out->alpha = alpha;
    adapter_out->lora_b = lora_b;
    adapter_out->lora_scale = lora_scale;
    adapter_out->N = N;
    adapter_out->r = r;
    adapter_out->src_version = src_version;
    adapter_out->device = dev;
    adapter_out->reserved = 0;
    return NVFP4LORA_OK;
}

nvfp4lora_status nvfp4lora_refold(nvfp4lora_adapter* adapter, const uint16_t* lora_b, const float* lora_scale,
                                  const float* alpha, int64_t N, int64_t r, uint64_t src_version,
                                  nvfp4lora_stream stream) {
    t_last_error.clear();
    if (!adapter) return fail(NVFP4LORA_ERR_INVALID_ARG, "adapter must be non-null");
    nvfp4lora_status st = check_fold_args(lora_b, lora_scale, alpha, N, r, adapter->b_folded, adapter->ratio);
    if (st != NVFP4LORA_OK) return st;
    if (alpha != adapter->alpha)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "alpha must be the adapter's own alpha tensor");
    if (N != adapter->N || r != adapter->r)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "lora_b must keep the adapter's [N, r] = [%lld, %lld]",
                    (long long)adapter->N, (long long)adapter->r);
    int dev = 0;
    DeviceInfo* info = nullptr;
    if ((st = device_info(&dev, &info)) != NVFP4LORA_OK) return st;
    if (dev != adapter->device)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "lora_b must stay on the adapter's device %d", adapter->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = launch_fold(lora_b, lora_scale, alpha, adapter->b_folded, adapter->ratio, N, r, s)) != NVFP4LORA_OK)
        return st;
    adapter->lora_b = lora_b;
    adapter->lora_scale = lora_scale;
    adapter->src_version = src_version;
    return NVFP4LORA_OK;
}

nvfp4lora_status nvfp4lora_mm_prepared(const uint8_t* a, const uint8_t* b, const uint8_t* a_sf, int64_t a_sf_bytes,
                                       const uint8_t* b_sf, int64_t b_sf_bytes, const float* alpha,
                                       const uint16_t* d, const nvfp4lora_adapter* adapter,
                                       const uint16_t* cur_lora_b, const float* cur_lora_scale,
                                       uint64_t cur_src_version, const uint16_t* bias, uint16_t* out,
                                       int64_t M, int64_t N, int64_t K, nvfp4lora_stream stream) {
    t_last_error.clear();
    nvfp4lora_status st = check_base(a, b, a_sf, a_sf_bytes, b_sf, b_sf_bytes, alpha, bias, out, M, N, K);
    if (st != NVFP4LORA_OK) return st;
    if (!adapter) return fail(NVFP4LORA_ERR_INVALID_ARG, "adapter must be non-null");
    if (!adapter->b_folded || !adapter->ratio)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "adapter has no b_folded / ratio buffers");
    if (adapter->N != N)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "adapter has N = %lld, the call N = %lld",
                    (long long)adapter->N, (long long)N);
    if ((st = check_rank(adapter->r)) != NVFP4LORA_OK) return st;
    if (!d) return fail(NVFP4LORA_ERR_INVALID_ARG, "the prepared path still requires d");
    if (!aligned(d, 16) || !aligned(adapter->b_folded, 16))
        return fail(NVFP4LORA_ERR_INVALID_ARG, "d and b_folded must be 16-byte aligned");
    if (alpha != adapter->alpha)
        return fail(NVFP4LORA_ERR_STALE_ADAPTER,
                    "the adapter was prepared for another alpha tensor; re-prepare when alpha changes");
    if (cur_lora_b != adapter->lora_b || cur_lora_scale != adapter->lora_scale)
        return fail(NVFP4LORA_ERR_STALE_ADAPTER, "the adapter's lora_b / lora_scale moved since the prepare");
    if (cur_src_version != adapter->src_version)
        return fail(NVFP4LORA_ERR_STALE_ADAPTER, "the adapter's lora_b / lora_scale were written since the prepare");
    int dev = 0;
    DeviceInfo* info = nullptr;
    if ((st = device_info(&dev, &info)) != NVFP4LORA_OK) return st;
    if (dev != adapter->device)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "the adapter lives on device %d, the call runs on %d",
                    adapter->device, dev);
    return launch<Mode::Prepared>(a, b, a_sf, b_sf, alpha, adapter->ratio, d, adapter->b_folded,
                                       adapter->r, bias, out, M, N, K, reinterpret_cast<cudaStream_t>(stream));
}

nvfp4lora_status nvfp4lora_grouped_mm(const uint8_t* a, const uint8_t* b, const uint8_t* a_sf, int64_t a_sf_bytes,
                                      const uint8_t* b_sf, int64_t b_sf_bytes, const int32_t* m_indptr,
                                      int64_t num_experts, const float* alpha, const uint16_t* d,
                                      const uint16_t* lora_b, const float* lora_scale, int64_t r,
                                      const uint16_t* bias, uint16_t* out, int64_t rows, int64_t N, int64_t K,
                                      nvfp4lora_stream stream) {
    t_last_error.clear();
    if (num_experts < 1 || num_experts > kMaxExperts)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "num_experts = %lld: 1 <= num_experts <= %d is required",
                    (long long)num_experts, kMaxExperts);
    if (rows > kMaxDim || (int64_t)num_experts * N > kMaxDim)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "rows and num_experts x N must be at most 2^30");
    // the per-expert scale buffers of b are consecutive, ceil(N/128)*128*K/16 bytes each
    const int64_t per_expert_sf = (N + 127) / 128 * 128 * (K / 16);
    nvfp4lora_status st = check_base(a, b, a_sf, a_sf_bytes, b_sf, per_expert_sf, alpha, bias, out, rows, N, K);
    if (st != NVFP4LORA_OK) return st;
    if (b_sf_bytes < num_experts * per_expert_sf)
        return fail(NVFP4LORA_ERR_INVALID_ARG,
                    "b_sf has %lld bytes; num_experts consecutive 128x4 buffers of N rows need %lld",
                    (long long)b_sf_bytes, (long long)(num_experts * per_expert_sf));
    if (!m_indptr || !aligned(m_indptr, 4))
        return fail(NVFP4LORA_ERR_INVALID_ARG, "m_indptr must be a non-null, 4-byte aligned int32 array");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (lora_scale == nullptr)
        return launch_gemm_grouped<Mode::Off>(a, b, a_sf, b_sf, m_indptr, num_experts, alpha, nullptr, nullptr,
                                              nullptr, 0, bias, out, rows, N, K, s);
    if ((st = check_rank(r)) != NVFP4LORA_OK) return st;
    if (!d || !lora_b) return fail(NVFP4LORA_ERR_INVALID_ARG, "lora_scale given: d and lora_b must be non-null");
    if (!aligned(d, 16) || !aligned(lora_b, 16))
        return fail(NVFP4LORA_ERR_INVALID_ARG, "d and lora_b must be 16-byte aligned");
    if (!aligned(lora_scale, 4)) return fail(NVFP4LORA_ERR_INVALID_ARG, "lora_scale must be 4-byte aligned");
    return launch_gemm_grouped<Mode::Raw>(a, b, a_sf, b_sf, m_indptr, num_experts, alpha, lora_scale, d, lora_b, r,
                                          bias, out, rows, N, K, s);
}

nvfp4lora_status nvfp4lora_device_status(nvfp4lora_stream stream) {
    t_last_error.clear();
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int word = 0;
    e = cudaMemcpyFromSymbol(&word, g_device_error, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    if (word != 0) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
        if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
        if (word == kErrBadIndptr)
            return fail(NVFP4LORA_ERR_INVALID_ARG,
                        "grouped call: m_indptr must start at 0, be non-decreasing, hold multiples of 128 and "
                        "end at most at the row count (no tile was computed)");
        if (word == kErrBadRoute)
            return fail(NVFP4LORA_ERR_INVALID_ARG,
                        "LoRA delta: a routing entry was out of range (expert id outside [0, num_experts), "
                        "permuted index past the activation rows, or a null or misaligned bank address); "
                        "that slot was skipped");
        return fail(NVFP4LORA_ERR_DEVICE_TIMEOUT, "a kernel's bounded wait ran out (pipeline stalled)");
    }
    return NVFP4LORA_OK;
}

nvfp4lora_status nvfp4lora_selftest_wait_timeout(int64_t limit_ns, nvfp4lora_stream stream) {
    t_last_error.clear();
    if (limit_ns <= 0 || limit_ns > 1000000000)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "limit_ns = %lld: 0 < limit_ns <= 1e9 is required", (long long)limit_ns);
    int dev = 0;
    DeviceInfo* info = nullptr;
    nvfp4lora_status st = device_info(&dev, &info);
    if (st != NVFP4LORA_OK) return st;
    wait_timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        (unsigned long long)limit_ns);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
    return NVFP4LORA_OK;
}

nvfp4lora_status nvfp4lora_quantize(const uint16_t* x, int64_t rows, int64_t K, const float* global_scale,
                                    uint8_t* codes, uint8_t* scales, int64_t scales_bytes, nvfp4lora_stream stream) {
    t_last_error.clear();
    if (!x || !global_scale || !codes || !scales)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "x, global_scale, codes and scales must be non-null");
    if (rows < 1 || K < 64 || K % 64 != 0)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "rows >= 1 and K >= 64 with K %% 64 == 0 are required (rows=%lld K=%lld)",
                    (long long)rows, (long long)K);
    if (rows > (int64_t)1 << 40 || K > (int64_t)1 << 30)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "rows x K too large");
    const int64_t need = (rows + 127) / 128 * 128 * (K / 16);
    if (scales_bytes < need)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "scales needs %lld bytes (rows padded to 128 x K/16), got %lld",
                    (long long)need, (long long)scales_bytes);
    if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, 16))
        return fail(NVFP4LORA_ERR_INVALID_ARG, "x, codes and scales must be 16-byte aligned");
    if (!aligned(global_scale, 4)) return fail(NVFP4LORA_ERR_INVALID_ARG, "global_scale must be 4-byte aligned");
    int dev = 0;
    DeviceInfo* info = nullptr;
    nvfp4lora_status st = device_info(&dev, &info);
    if (st != NVFP4LORA_OK) return st;
    const int64_t total = (rows + 127) / 128 * 128 * (K / 16);             // one thread per block per step
    const int64_t want = (total + kQuantThreads - 1) / kQuantThreads;
    // a grid-stride loop over one wave: the launch bounds keep 8 CTAs resident per SM
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)info->sms * 8));
    quantize_kernel<<<grid, kQuantThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, rows, K, global_scale,
                                                                                          codes, scales);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
    return NVFP4LORA_OK;
}

nvfp4lora_status nvfp4lora_bgmv_moe_gemm2_lora_delta(
    const void* act, int64_t padded_rows, int64_t I, const int32_t* perm, const int64_t* w_ptr_a,
    int64_t lora_stride_a, const int64_t* w_ptr_b, int64_t lora_stride_b, const int32_t* topk_ids,
    const float* topk_weights, const int32_t* lora_ids, int64_t num_tokens, int64_t top_k, int64_t num_experts,
    int64_t rank, int64_t hidden_size, int32_t lora_dtype, float scale, int32_t out_dtype, void* out,
    nvfp4lora_stream stream) {
    t_last_error.clear();
    const int64_t kMaxDim = (int64_t)1 << 30;
    if (num_tokens < 0 || num_tokens > kMaxDim)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "num_tokens = %lld out of range", (long long)num_tokens);
    if (top_k < 1 || top_k > kBgmvMaxTopK)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "top_k = %lld: 1 <= top_k <= %d is required", (long long)top_k,
                    kBgmvMaxTopK);
    if (rank < 8 || rank > kBgmvMaxRank || rank % 8 != 0)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "rank = %lld: 8 <= rank <= %d with rank %% 8 == 0 is required",
                    (long long)rank, kBgmvMaxRank);
    if (I < 8 || I % 8 != 0 || I > kMaxDim)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "I = %lld: I >= 8 with I %% 8 == 0 is required", (long long)I);
    if (hidden_size < 1 || hidden_size > kMaxDim)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "hidden_size = %lld out of range", (long long)hidden_size);
    if (num_experts < 1 || num_experts > kMaxDim)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "num_experts = %lld out of range", (long long)num_experts);
    if (padded_rows < 0 || padded_rows > kMaxDim)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "padded_rows = %lld out of range", (long long)padded_rows);
    if (num_tokens * top_k > kMaxDim)
        return fail(NVFP4LORA_ERR_INVALID_ARG, "num_tokens * top_k too large");
    if (lora_stride_a < 0 || lora_stride_b < 0 || lora_stride_a % 8 != 0 || lora_stride_b % 8 != 0)
        return fail(NVFP4LORA_ERR_INVALID_ARG,
                    "lora_stride_a = %lld, lora_stride_b = %lld: non-negative multiples of 8 are required "
                    "(adapter blocks start on 16-byte boundaries)", (long long)lora_stride_a, (long long)lora_stride_b);
    if ((lora_dtype != NVFP4LORA_DTYPE_BF16 && lora_dtype != NVFP4LORA_DTYPE_FP16) ||
        (out_dtype != NVFP4LORA_DTYPE_BF16 && out_dtype != NVFP4LORA_DTYPE_FP16))
        return fail(NVFP4LORA_ERR_INVALID_ARG, "lora_dtype and out_dtype must be NVFP4LORA_DTYPE_BF16 or _FP16");
    if (num_tokens == 0) return NVFP4LORA_OK;
    if (!perm || !w_ptr_a || !w_ptr_b || !topk_ids || !topk_weights || !lora_ids || !out ||
        (!act && padded_rows > 0))
        return fail(NVFP4LORA_ERR_INVALID_ARG, "every pointer argument must be non-null");
    if (!aligned(act, 16)) return fail(NVFP4LORA_ERR_INVALID_ARG, "act must be 16-byte aligned");
    if (!aligned(w_ptr_a, 8) || !aligned(w_ptr_b, 8))
        return fail(NVFP4LORA_ERR_INVALID_ARG, "w_ptr_a and w_ptr_b must be 8-byte aligned");
    if (!aligned(perm, 4) || !aligned(topk_ids, 4) || !aligned(topk_weights, 4) || !aligned(lora_ids, 4) ||
        !aligned(out, 2))
        return fail(NVFP4LORA_ERR_INVALID_ARG, "routing tables must be 4-byte aligned and out 2-byte aligned");
    int dev = 0;
    DeviceInfo* info = nullptr;
    nvfp4lora_status st = device_info(&dev, &info);
    if (st != NVFP4LORA_OK) return st;

    // A cluster of cs CTAs per token splits I (shrink) and H (expand): the smallest power of two
    // that gives about two CTAs per SM, capped by the cluster limit and by I / 8 and H; raised
    // further if one CTA's shared memory (the shrink's cells for its I slice) would not fit.
    const int64_t len = top_k * rank;
    auto fits = [&](int64_t c) { return bgmv_smem_floats(len, (I / 8 + c - 1) / c, c) * 4 <= kBgmvSmemLimit; };
    auto can_grow = [&](int64_t c) { return c < kBgmvMaxCluster && 2 * c <= I / 8 && 2 * c <= hidden_size; };
    int cs = 1;
    while (can_grow(cs) && num_tokens * cs < 2 * (int64_t)info->sms) cs *= 2;
    while (!fits(cs) && can_grow(cs)) cs *= 2;
    if (!fits(cs))
        return fail(NVFP4LORA_ERR_INVALID_ARG,
                    "top_k * rank * I too large: one CTA's share (I / %d columns, %lld rows of the adapters) needs more "
                    "than %d bytes of shared memory", cs, (long long)len, kBgmvSmemLimit);
    BgmvArgs args;
    args.act = act;
    args.perm = perm;
    args.w_ptr_a = w_ptr_a;
    args.w_ptr_b = w_ptr_b;
    args.topk_ids = topk_ids;
    args.topk_w = topk_weights;
    args.lora_ids = lora_ids;
    args.out = out;
    args.stride_a = lora_stride_a;
    args.stride_b = lora_stride_b;
    args.rows = (int)padded_rows;
    args.I = (int)I;
    args.top_k = (int)top_k;
    args.num_experts = (int)num_experts;
    args.rank = (int)rank;
    args.H = (int)hidden_size;
    args.cs = cs;
    args.scale = scale;
    const int smem = (int)(bgmv_smem_floats(len, (I / 8 + cs - 1) / cs, cs) * (int64_t)sizeof(float));

    auto pick = [&](auto kernel) -> nvfp4lora_status {
        // the delta's shared memory can exceed the 48 KB default; the L1 carve-out stays the
        // driver's choice (the activation rows are re-read through L1)
        nvfp4lora_status sa = ensure_smem_attr(info, kernel, kBgmvSmemLimit, false);
        if (sa != NVFP4LORA_OK) return sa;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(num_tokens * cs));
        cfg.blockDim = dim3(kBgmvThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = reinterpret_cast<cudaStream_t>(stream);
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cs > 1) {
            attr[1].id = cudaLaunchAttributeClusterDimension;
            attr[1].val.clusterDim.x = cs;
            attr[1].val.clusterDim.y = 1;
            attr[1].val.clusterDim.z = 1;
            cfg.numAttrs = 2;
        }
        cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args);
        if (e != cudaSuccess) return cuda_fail(e, "LoRA delta launch");
        return NVFP4LORA_OK;
    };
    const bool f16_in = lora_dtype == NVFP4LORA_DTYPE_FP16, f16_out = out_dtype == NVFP4LORA_DTYPE_FP16;
    if (f16_in)
        return f16_out ? pick(bgmv_delta_kernel<true, true>) : pick(bgmv_delta_kernel<true, false>);
    return f16_out ? pick(bgmv_delta_kernel<false, true>) : pick(bgmv_delta_kernel<false, false>);
}

const char* nvfp4lora_last_error(void) { return t_last_error.c_str(); }

const char* nvfp4lora_version(void) { return "nvfp4lora 0.1.0 (sm_100a)"; }

}  // extern "C"
