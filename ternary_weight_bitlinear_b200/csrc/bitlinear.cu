// bitlinear.cu -- the C ABI of libbitlinear.so: argument checks, dispatch and
// launches of the sm_100a kernels.  One translation unit so the kernels share
// the device status word without relocatable device code.
#include "bitlinear.h"

#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cstdio>
#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "decode.cuh"
#include "glue.cuh"
#include "pack.cuh"
#include "quant.cuh"

namespace {

using namespace bl;

constexpr int kQuantThreads = 256;

// ---- device properties and per-kernel launch settings ---------------------
struct DeviceInfo {
    int sms = 0;
    int major = 0;
    int smem_optin = 0;
};

std::mutex g_mu;

bl_status current_device(int* dev, DeviceInfo* info) {
    static DeviceInfo cache[64];
    static bool have[64] = {};
    if (cudaGetDevice(dev) != cudaSuccess) { cudaGetLastError(); return BL_ERR_DEVICE; }
    if (*dev < 0 || *dev >= 64) return BL_ERR_DEVICE;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!have[*dev]) {
        DeviceInfo d;
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, *dev) !=
                cudaSuccess ||
            cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, *dev) !=
                cudaSuccess) {
            cudaGetLastError();
            return BL_ERR_DEVICE;
        }
        cache[*dev] = d;
        have[*dev] = true;
    }
    *info = cache[*dev];
    return info->major == 10 ? BL_OK : BL_ERR_DEVICE;
}

thread_local char g_last_error[256] = "";

void record_cuda_error(cudaError_t e, const char* where) {
    snprintf(g_last_error, sizeof g_last_error, "%s: %s (%s)", where, cudaGetErrorName(e),
             cudaGetErrorString(e));
}

// Opt a kernel in to all the dynamic shared memory the device allows next to
// its static shared memory (once per device) and return how many of its CTAs
// fit on one SM with `smem` dynamic bytes; -1 on a CUDA error.
int prepare_kernel(const void* fn, int dev, const DeviceInfo& info, int threads, int64_t smem) {
    static std::map<std::tuple<const void*, int, int64_t>, int> occ;
    static std::map<std::pair<const void*, int>, int64_t> max_dyn;
    std::lock_guard<std::mutex> lk(g_mu);
    auto mk = std::make_pair(fn, dev);
    if (!max_dyn.count(mk)) {
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, fn);
        if (e != cudaSuccess) { record_cuda_error(e, "cudaFuncGetAttributes"); cudaGetLastError(); return -1; }
        const int64_t dyn = (int64_t)info.smem_optin - (int64_t)fa.sharedSizeBytes;
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
        if (e != cudaSuccess) { record_cuda_error(e, "cudaFuncSetAttribute"); cudaGetLastError(); return -1; }
        max_dyn[mk] = dyn;
    }
    if (smem > max_dyn[mk]) {
        snprintf(g_last_error, sizeof g_last_error, "kernel needs %lld B of shared memory, %lld allowed",
                 (long long)smem, (long long)max_dyn[mk]);
        return -1;
    }
    auto key = std::make_tuple(fn, dev, smem);
    auto it = occ.find(key);
    if (it != occ.end()) return it->second;
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, (size_t)smem);
    if (e != cudaSuccess) { record_cuda_error(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor"); cudaGetLastError(); return -1; }
    n = std::max(n, 1);
    occ[key] = n;
    return n;
}

// Launch with programmatic dependent launch enabled: the kernel may begin
// while the previous kernel in the stream drains; every kernel here calls
// griddepcontrol.wait before touching data another kernel may have written.
template <typename... KArgs, typename... Args>
bl_status launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                 cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    if (e != cudaSuccess) {
        record_cuda_error(e, "cudaLaunchKernelEx");
        cudaGetLastError();
        return BL_ERR_CUDA;
    }
    return BL_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bl_status check_shape(int64_t M, int64_t K, int64_t N) {
    if (M < 0 || K <= 0 || N <= 0) return BL_ERR_SHAPE;
    if (K % 16 != 0 || N % 4 != 0 || K > BL_MAX_K) return BL_ERR_SHAPE;
    if (M > INT32_MAX || N / 4 > INT32_MAX) return BL_ERR_SHAPE;
    return BL_OK;
}

bool decode_eligible(int64_t M, int64_t K) { return M <= kDecMaxTokens && M * K <= kDecMaxQBytes; }

int64_t ws_q_bytes(int64_t M, int64_t K) { return round_up(M * K, 256); }
int64_t ws_vec_bytes(int64_t M) { return round_up(4 * M, 256); }

// ---- decode launches --------------------------------------------------------
template <int MT, int EPI, bool FUSED>
bl_status launch_decode_mt(const DecodeArgs& a, int dev, const DeviceInfo& info,
                           cudaStream_t stream) {
    const int64_t smem = decode_smem_bytes(MT, a.K, a.chunk);
    auto fn = decode_kernel<MT, EPI, FUSED>;
    const int per_sm = prepare_kernel(reinterpret_cast<const void*>(fn), dev, info, kDecThreads,
                                      smem);
    if (per_sm < 0) return BL_ERR_CUDA;
    const int64_t grid = std::min<int64_t>(a.R, (int64_t)info.sms * per_sm);
    return launch(fn, dim3((unsigned)grid), dim3(kDecThreads), (size_t)smem, stream, a);
}

template <int EPI, bool FUSED>
bl_status launch_decode(int mt, const DecodeArgs& a, int dev, const DeviceInfo& info,
                        cudaStream_t stream) {
    switch (mt) {
        case 1: return launch_decode_mt<1, EPI, FUSED>(a, dev, info, stream);
        case 2: return launch_decode_mt<2, EPI, FUSED>(a, dev, info, stream);
        case 3: return launch_decode_mt<3, EPI, FUSED>(a, dev, info, stream);
        case 4: return launch_decode_mt<4, EPI, FUSED>(a, dev, info, stream);
        default: return BL_ERR_SHAPE;
    }
}

template <bool FUSED>
bl_status launch_decode_epi(int epi, int mt, const DecodeArgs& a, int dev, const DeviceInfo& info,
                            cudaStream_t stream) {
    switch (epi) {
        case kEpiF32: return launch_decode<kEpiF32, FUSED>(mt, a, dev, info, stream);
        case kEpiBF16: return launch_decode<kEpiBF16, FUSED>(mt, a, dev, info, stream);
        case kEpiI32: return launch_decode<kEpiI32, FUSED>(mt, a, dev, info, stream);
        default: return BL_ERR_DTYPE;
    }
}

int decode_chunk(int64_t K) { return (int)std::min<int64_t>(K, kDecChunkMax); }

// Matmul + epilogue on pre-quantised activations, any M: token groups of up
// to four rows through the decode kernel.
bl_status run_quantized(const int8_t* q, const float* s_x, const int32_t* rowsum, const uint8_t* P,
                        float beta, int64_t M, int64_t K, int64_t N, void* y, int epi,
                        const uint16_t* residual, int dev, const DeviceInfo& info,
                        cudaStream_t stream) {
    const int64_t max_mt = std::max<int64_t>(1, std::min<int64_t>(kDecMaxTokens, kDecMaxQBytes / K));
    const size_t ysz = epi == kEpiBF16 ? 2 : 4;
    for (int64_t m0 = 0; m0 < M; m0 += max_mt) {
        const int mt = (int)std::min<int64_t>(max_mt, M - m0);
        DecodeArgs a = {};
        a.q = q + m0 * K;
        a.s_x = s_x ? s_x + m0 : nullptr;
        a.rowsum = rowsum + m0;
        a.P = P;
        a.beta = beta;
        a.K = (int)K;
        a.chunk = decode_chunk(K);
        a.R = N / 4;
        a.N = N;
        a.y = static_cast<char*>(y) + (size_t)(m0 * N) * ysz;
        a.residual = residual ? residual + m0 * N : nullptr;
        bl_status st = launch_decode_epi<false>(epi, mt, a, dev, info, stream);
        if (st != BL_OK) return st;
    }
    return BL_OK;
}

int epi_of(bl_out_dtype d) {
    return d == BL_OUT_BF16 ? kEpiBF16 : d == BL_OUT_F32 ? kEpiF32 : -1;
}


// ---- fixed scratch for bitlinear_forward_noalloc ----------------------------
// One array per device, allocated with the module; its device address is
// looked up once per device.  (The name is a host-side stand-in in host code:
// only the looked-up address may be given to kernels.)
static __device__ __align__(256) uint8_t g_noalloc_scratch[BL_NOALLOC_SCRATCH_BYTES];

bl_status noalloc_scratch(int dev, void** ptr) {
    static void* addr[64] = {};
    std::lock_guard<std::mutex> lk(g_mu);
    if (!addr[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            record_cuda_error(e, "cudaGetSymbolAddress");
            cudaGetLastError();
            return BL_ERR_CUDA;
        }
        addr[dev] = p;
    }
    *ptr = addr[dev];
    return BL_OK;
}

}  // namespace

// =============================================================================
extern "C" {

int bitlinear_abi_version(void) { return BL_ABI_VERSION; }

const char* bitlinear_last_error(void) { return g_last_error; }

const char* bitlinear_status_string(bl_status s) {
    switch (s) {
        case BL_OK: return "ok";
        case BL_ERR_NULL: return "a required pointer is NULL";
        case BL_ERR_SHAPE: return "invalid shape (need M>=0, K>0, K%16==0, K<=BL_MAX_K, N>0, N%4==0)";
        case BL_ERR_ALIGN: return "a tensor pointer is not 16-byte aligned";
        case BL_ERR_DTYPE: return "invalid output dtype or dtype/option combination";
        case BL_ERR_WORKSPACE: return "workspace missing or too small";
        case BL_ERR_CUDA: return "CUDA launch or runtime error";
        case BL_ERR_TIMEOUT: return "a device-side bounded wait expired";
        case BL_ERR_DEVICE: return "no usable sm_100 CUDA device is current";
    }
    return "unknown status";
}

bl_status bitlinear_pack_workspace_size(int64_t N, int64_t K, size_t* bytes) {
    if (!bytes) return BL_ERR_NULL;
    bl_status st = check_shape(0, K, N);
    if (st != BL_OK) return st;
    *bytes = sizeof(PackWorkspace);
    return BL_OK;
}

bl_status bitlinear_pack(const float* W, int64_t N, int64_t K, uint8_t* P, float* beta_out,
                         void* workspace, size_t workspace_bytes, void* stream) {
    bl_status st = check_shape(0, K, N);
    if (st != BL_OK) return st;
    if (!W || !P || !beta_out) return BL_ERR_NULL;
    if (!workspace || workspace_bytes < sizeof(PackWorkspace)) return BL_ERR_WORKSPACE;
    if (!aligned16(W) || !aligned16(P) || !aligned16(workspace)) return BL_ERR_ALIGN;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    PackWorkspace* ws = static_cast<PackWorkspace*>(workspace);
    const int64_t n = N * K;
    if ((st = launch(absmean_partial_kernel, dim3(kPackPartials), dim3(kPackThreads), 0, s, W, n,
                     ws)) != BL_OK)
        return st;
    if ((st = launch(absmean_finalize_kernel, dim3(1), dim3(32), 0, s, n, kPackPartials, ws,
                     beta_out)) != BL_OK)
        return st;
    const int64_t R = N / 4, work = R * (K / 16);
    return launch(ternarize_pack_kernel, dim3((unsigned)((work + kPackThreads - 1) / kPackThreads)),
                  dim3(kPackThreads), 0, s, W, R, K, (const PackWorkspace*)ws, P);
}

bl_status bitlinear_pack_ternary(const int8_t* t, int64_t N, int64_t K, uint8_t* P, void* stream) {
    bl_status st = check_shape(0, K, N);
    if (st != BL_OK) return st;
    if (!t || !P) return BL_ERR_NULL;
    if (!aligned16(t) || !aligned16(P)) return BL_ERR_ALIGN;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    const int64_t R = N / 4, work = R * (K / 16);
    return launch(pack_ternary_kernel, dim3((unsigned)((work + kPackThreads - 1) / kPackThreads)),
                  dim3(kPackThreads), 0, static_cast<cudaStream_t>(stream), t, R, K, P);
}

bl_status bitlinear_unpack(const uint8_t* P, int64_t N, int64_t K, int8_t* t, void* stream) {
    bl_status st = check_shape(0, K, N);
    if (st != BL_OK) return st;
    if (!t || !P) return BL_ERR_NULL;
    if (!aligned16(t) || !aligned16(P)) return BL_ERR_ALIGN;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    const int64_t R = N / 4, work = R * (K / 16);
    return launch(unpack_kernel, dim3((unsigned)((work + kPackThreads - 1) / kPackThreads)),
                  dim3(kPackThreads), 0, static_cast<cudaStream_t>(stream), P, R, K, t);
}

bl_status bitlinear_act_quant(const uint16_t* x, const uint16_t* gain, float eps, int64_t M,
                              int64_t K, int8_t* q, float* s_x, int32_t* rowsum, void* stream) {
    bl_status st = check_shape(M, K, 4);
    if (st != BL_OK) return st;
    if (M == 0) return BL_OK;
    if (!x || !q || !s_x) return BL_ERR_NULL;
    if (!aligned16(x) || !aligned16(q) || (gain && !aligned16(gain))) return BL_ERR_ALIGN;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    return launch(act_quant_kernel<kQuantThreads>, dim3((unsigned)M), dim3(kQuantThreads), 0,
                  static_cast<cudaStream_t>(stream), x, gain, eps, (int)K, q, s_x, rowsum);
}

bl_status bitlinear_forward_workspace_size(int64_t M, int64_t K, int64_t N, size_t* bytes) {
    if (!bytes) return BL_ERR_NULL;
    bl_status st = check_shape(M, K, N);
    if (st != BL_OK) return st;
    *bytes = (M == 0 || decode_eligible(M, K))
                 ? 0
                 : (size_t)(ws_q_bytes(M, K) + 2 * ws_vec_bytes(M));
    return BL_OK;
}

bl_status bitlinear_forward(const uint16_t* x, const uint16_t* gain, float eps, const uint8_t* P,
                            float beta, int64_t M, int64_t K, int64_t N, void* y,
                            bl_out_dtype y_dtype, void* workspace, size_t workspace_bytes,
                            void* stream) {
    bl_status st = check_shape(M, K, N);
    if (st != BL_OK) return st;
    const int epi = epi_of(y_dtype);
    if (epi < 0) return BL_ERR_DTYPE;
    if (M == 0) return BL_OK;
    if (!x || !P || !y) return BL_ERR_NULL;
    if (!aligned16(x) || !aligned16(P) || !aligned16(y) || (gain && !aligned16(gain)))
        return BL_ERR_ALIGN;
    size_t need = 0;
    bitlinear_forward_workspace_size(M, K, N, &need);
    if (need > 0) {
        if (!workspace || workspace_bytes < need) return BL_ERR_WORKSPACE;
        if (!aligned16(workspace)) return BL_ERR_ALIGN;
    }
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    if (decode_eligible(M, K)) {
        DecodeArgs a = {};
        a.x = x;
        a.gain = gain;
        a.eps = eps;
        a.P = P;
        a.beta = beta;
        a.K = (int)K;
        a.chunk = decode_chunk(K);
        a.R = N / 4;
        a.N = N;
        a.y = y;
        return launch_decode_epi<true>(epi, (int)M, a, dev, info, s);
    }
    char* w = static_cast<char*>(workspace);
    int8_t* q = reinterpret_cast<int8_t*>(w);
    float* sx = reinterpret_cast<float*>(w + ws_q_bytes(M, K));
    int32_t* rs = reinterpret_cast<int32_t*>(w + ws_q_bytes(M, K) + ws_vec_bytes(M));
    if ((st = launch(act_quant_kernel<kQuantThreads>, dim3((unsigned)M), dim3(kQuantThreads), 0, s,
                     x, gain, eps, (int)K, q, sx, rs)) != BL_OK)
        return st;
    return run_quantized(q, sx, rs, P, beta, M, K, N, y, epi, nullptr, dev, info, s);
}

bl_status bitlinear_forward_quantized(const int8_t* q, const float* s_x, const int32_t* rowsum,
                                      const uint8_t* P, float beta, int64_t M, int64_t K,
                                      int64_t N, void* y, bl_out_dtype y_dtype,
                                      const uint16_t* residual, void* stream) {
    bl_status st = check_shape(M, K, N);
    if (st != BL_OK) return st;
    const int epi = epi_of(y_dtype);
    if (epi < 0 || (residual && epi != kEpiBF16)) return BL_ERR_DTYPE;
    if (M == 0) return BL_OK;
    if (!q || !s_x || !rowsum || !P || !y) return BL_ERR_NULL;
    if (!aligned16(q) || !aligned16(P) || !aligned16(y) || (residual && !aligned16(residual)))
        return BL_ERR_ALIGN;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    return run_quantized(q, s_x, rowsum, P, beta, M, K, N, y, epi, residual, dev, info,
                         static_cast<cudaStream_t>(stream));
}

bl_status bitlinear_accumulate(const int8_t* q, const int32_t* rowsum, const uint8_t* P, int64_t M,
                               int64_t K, int64_t N, int32_t* acc, void* stream) {
    bl_status st = check_shape(M, K, N);
    if (st != BL_OK) return st;
    if (M == 0) return BL_OK;
    if (!q || !rowsum || !P || !acc) return BL_ERR_NULL;
    if (!aligned16(q) || !aligned16(P) || !aligned16(acc)) return BL_ERR_ALIGN;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    return run_quantized(q, nullptr, rowsum, P, 1.0f, M, K, N, acc, kEpiI32, nullptr, dev, info,
                         static_cast<cudaStream_t>(stream));
}

bl_status bitlinear_relu2_mul(const uint16_t* a, const uint16_t* b, int64_t n, uint16_t* z,
                              void* stream) {
    if (n < 0) return BL_ERR_SHAPE;
    if (n == 0) return BL_OK;
    if (!a || !b || !z) return BL_ERR_NULL;
    if (!aligned16(a) || !aligned16(b) || !aligned16(z)) return BL_ERR_ALIGN;
    int dev;
    DeviceInfo info;
    bl_status st;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    const int64_t threads = (n + 7) / 8;
    return launch(relu2_mul_kernel, dim3((unsigned)((threads + kGlueThreads - 1) / kGlueThreads)),
                  dim3(kGlueThreads), 0, static_cast<cudaStream_t>(stream), a, b, n, z);
}

bl_status bitlinear_device_status(void* stream) {
    int dev;
    DeviceInfo info;
    bl_status st;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        record_cuda_error(e, "cudaStreamSynchronize");
        cudaGetLastError();
        return BL_ERR_CUDA;
    }
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof v) != cudaSuccess ||
        cudaMemcpyToSymbol(g_status, &zero, sizeof zero) != cudaSuccess) {
        cudaGetLastError();
        return BL_ERR_CUDA;
    }
    return (v & kStatusTimeout) ? BL_ERR_TIMEOUT : BL_OK;
}

bl_status bitlinear_forward_noalloc(const uint16_t* x, const uint16_t* gain, float eps,
                                    const uint8_t* P, float beta, int64_t M, int64_t K,
                                    int64_t N, void* y, bl_out_dtype y_dtype, void* stream) {
    size_t need = 0;
    bl_status st = bitlinear_forward_workspace_size(M, K, N, &need);
    if (st != BL_OK) return st;
    if (need > BL_NOALLOC_SCRATCH_BYTES) {
        snprintf(g_last_error, sizeof g_last_error,
                 "bitlinear_forward_noalloc: this shape needs %zu bytes of scratch; the fixed "
                 "scratch holds %u",
                 need, (unsigned)BL_NOALLOC_SCRATCH_BYTES);
        return BL_ERR_WORKSPACE;
    }
    void* scratch = nullptr;
    if (need > 0) {
        int dev;
        DeviceInfo info;
        if ((st = current_device(&dev, &info)) != BL_OK) return st;
        if ((st = noalloc_scratch(dev, &scratch)) != BL_OK) return st;
    }
    return bitlinear_forward(x, gain, eps, P, beta, M, K, N, y, y_dtype, scratch,
                             need > 0 ? (size_t)BL_NOALLOC_SCRATCH_BYTES : 0, stream);
}

}  // extern "C"
