// bitlinear.cu -- the C ABI of libbitlinear.so: argument checks, dispatch and
// launches of the sm_100a kernels.  One translation unit so the kernels share
// the device status word without relocatable device code.
#include "bitlinear.h"

#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <climits>
#include <cmath>
#include <cstdio>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "common.cuh"
#include "decode.cuh"
#include "gemm_tc.cuh"
#include "glue.cuh"
#include "pack.cuh"
#include "quant.cuh"
#include "skinny.cuh"
#include "ste.cuh"
#include "chain.cuh"
#include "attn.cuh"

namespace {

using namespace bl;

constexpr int kQuantThreads = 256;
constexpr int kSmallBatch = 8;  // parameter-table size of small batches
constexpr int64_t kQuantWarpMinRows = 1024;  // rows from which a warp per row pays off
// many rows: one CTA of W warps per row, VPT 16-byte vectors per thread, at
// least MINB CTAs per SM (the register budget)
constexpr int kQuantRowW1 = 2, kQuantRowVpt1 = 5, kQuantRowMinB1 = 12;  // K <= 2560
constexpr int kQuantRowW2 = 4, kQuantRowVpt2 = 7, kQuantRowMinB2 = 4;   // K <= 7168

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

// Cooperative launch: every CTA of the grid is resident at once (or the
// launch fails), which a kernel with a grid-wide barrier needs.
template <typename... KArgs, typename... Args>
bl_status launch_coop(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    if (e != cudaSuccess) {
        record_cuda_error(e, "cudaLaunchKernelEx (cooperative)");
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

int64_t ws_q_bytes(int64_t M, int64_t K) { return round_up(M * K, 256); }
int64_t ws_vec_bytes(int64_t M) { return round_up(4 * M, 256); }
// workspace of one problem: codes | s_x | rowsum
int64_t ws_problem_bytes(int64_t M, int64_t K) { return ws_q_bytes(M, K) + 2 * ws_vec_bytes(M); }

struct WsSlices {
    int8_t* q;
    float* s_x;
    int32_t* rowsum;
};

// Tail of a forward workspace used by the 5..64-token kernel when a row tile
// is shared by several CTAs: one counter and two blocks of int32 partial sums
// (128 x npad: the tile a CTA's share enters part-way, and the one it leaves
// part-way) per CTA.
bool skinny_m(int64_t M) { return M >= kSkMinTokens && M <= kSkMaxTokens; }
int64_t sk_npad(int64_t M) { return (M + 15) / 16 * 16; }
int64_t sk_ctr_bytes() { return round_up(8 * kSkMaxGrid, 256); }
int64_t sk_ws_bytes(int64_t M) {
    return skinny_m(M) ? sk_ctr_bytes() + (int64_t)kSkMaxGrid * 2 * 128 * sk_npad(M) * 4 : 0;
}

WsSlices ws_slices(char* w, int64_t M, int64_t K) {
    return {reinterpret_cast<int8_t*>(w), reinterpret_cast<float*>(w + ws_q_bytes(M, K)),
            reinterpret_cast<int32_t*>(w + ws_q_bytes(M, K) + ws_vec_bytes(M))};
}

// ---- quantisation launches --------------------------------------------------
template <int CAP>
bl_status launch_quant_cap(const QuantProblem* probs, int count, int64_t M, float eps, int dev,
                           const DeviceInfo& info, cudaStream_t stream) {
    QuantBatch<CAP> b{};
    b.count = count;
    b.M = (int)M;
    b.eps = eps;
    int kmax = 16;
    for (int i = 0; i < count; ++i) {
        b.p[i] = probs[i];
        kmax = std::max(kmax, probs[i].K);
    }
    const int64_t rows = (int64_t)count * M;
    if (rows >= kQuantWarpMinRows && kmax <= 8 * 32 * kQuantRowW1 * kQuantRowVpt1) {
        // many rows (prefill), rows up to 2560: two warps per row, held in registers
        auto fn = quant_row_kernel<kQuantRowW1, kQuantRowVpt1, kQuantRowMinB1, CAP>;
        if (prepare_kernel(reinterpret_cast<const void*>(fn), dev, info, 32 * kQuantRowW1, 0) < 0)
            return BL_ERR_CUDA;
        return launch(fn, dim3((unsigned)rows), dim3(32 * kQuantRowW1), 0, stream, b);
    }
    if (rows >= kQuantWarpMinRows && kmax <= 8 * 32 * kQuantRowW2 * kQuantRowVpt2) {
        // many rows, longer rows: four warps per row, held in registers
        auto fn = quant_row_kernel<kQuantRowW2, kQuantRowVpt2, kQuantRowMinB2, CAP>;
        if (prepare_kernel(reinterpret_cast<const void*>(fn), dev, info, 32 * kQuantRowW2, 0) < 0)
            return BL_ERR_CUDA;
        return launch(fn, dim3((unsigned)rows), dim3(32 * kQuantRowW2), 0, stream, b);
    }
    if (kmax <= kQuantWarpMaxK && rows >= kQuantWarpMinRows) {
        // many rows longer than the register kernels hold: one warp per row
        // staged in shared memory, up to 8 rows per CTA; few rows (decode) go
        // to one CTA per row below, which has the lower latency
        const int wpb = (int)std::max<int64_t>(1, std::min<int64_t>(8, 65536 / (4 * (int64_t)kmax)));
        auto fn = quant_warp_kernel<CAP>;
        const int64_t smem = (int64_t)wpb * 4 * kmax;
        if (prepare_kernel(reinterpret_cast<const void*>(fn), dev, info, 32 * wpb, smem) < 0)
            return BL_ERR_CUDA;
        return launch(fn, dim3((unsigned)((rows + wpb - 1) / wpb)), dim3(32 * wpb), (size_t)smem,
                      stream, b, kmax);
    }
    auto fn = quant_batch_kernel<kQuantThreads, CAP>;
    const int64_t smem = 2 * (int64_t)kmax;  // the staged bf16 row
    if (prepare_kernel(reinterpret_cast<const void*>(fn), dev, info, kQuantThreads, smem) < 0)
        return BL_ERR_CUDA;
    return launch(fn, dim3((unsigned)(count * M)), dim3(kQuantThreads), (size_t)smem, stream, b);
}

bl_status run_quant(const QuantProblem* probs, int count, int64_t M, float eps, int dev,
                    const DeviceInfo& info, cudaStream_t stream) {
    if (count <= kSmallBatch)
        return launch_quant_cap<kSmallBatch>(probs, count, M, eps, dev, info, stream);
    return launch_quant_cap<BL_MAX_BATCH>(probs, count, M, eps, dev, info, stream);
}

// ---- decode launches --------------------------------------------------------
// One matmul problem on already-quantised codes.
struct DecodeJob {
    const int8_t* q;
    const float* s_x;
    const int32_t* rowsum;
    const uint8_t* P;
    void* y;
    const uint16_t* residual;
    int64_t K, N;   // N outputs per token
    float beta;
    int epi;
    float beta2 = 0.0f;  // kEpiGateUp: the up projection's scale
    const float* beta_dev = nullptr;  // beta read from device memory instead (online forward)
    // packed rows of P: N/4, or N/2 for a gate/up pair (N = the pair's I outputs)
    int64_t packed_rows() const { return epi == kEpiGateUp ? N / 2 : N / 4; }
};

template <int MT, int CAP>
bl_status launch_decode_mt(const DecBatch<CAP>& b, int64_t rows, int dev, const DeviceInfo& info,
                           cudaStream_t stream) {
    auto fn = decode_batch_kernel<MT, CAP>;
    if (prepare_kernel(reinterpret_cast<const void*>(fn), dev, info, kDecThreads, kDecSmemBytes) < 0)
        return BL_ERR_CUDA;
    // one CTA per SM: leaves room on every SM for the next kernel's CTAs to
    // start prefetching (programmatic dependent launch)
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(rows, info.sms));
    return launch(fn, dim3((unsigned)grid), dim3(kDecThreads), (size_t)kDecSmemBytes, stream, b);
}

template <int CAP>
bl_status launch_decode_cap(const DecodeJob* jobs, int count, int mt, int dev,
                            const DeviceInfo& info, cudaStream_t stream) {
    DecBatch<CAP> b{};
    b.count = count;
    int64_t total = 0, rows = 0;
    for (int i = 0; i < count; ++i) {
        DecProblem& p = b.p[i];
        p.q = jobs[i].q;
        p.s_x = jobs[i].s_x;
        p.rowsum = jobs[i].rowsum;
        p.P = jobs[i].P;
        p.y = jobs[i].y;
        p.residual = jobs[i].residual;
        p.R = jobs[i].packed_rows();
        p.N = jobs[i].N;
        p.byte0 = total;
        p.K = (int)jobs[i].K;
        p.beta = jobs[i].beta;
        p.beta2 = jobs[i].beta2;
        p.beta_dev = jobs[i].beta_dev;
        p.epi = jobs[i].epi;
        total += p.R * p.K;
        rows += p.R;
    }
    b.total = total;
    switch (mt) {
        case 1: return launch_decode_mt<1, CAP>(b, rows, dev, info, stream);
        case 2: return launch_decode_mt<2, CAP>(b, rows, dev, info, stream);
        case 3: return launch_decode_mt<3, CAP>(b, rows, dev, info, stream);
        case 4: return launch_decode_mt<4, CAP>(b, rows, dev, info, stream);
        default: return BL_ERR_SHAPE;
    }
}

// All jobs share the token count mt (1..4); one launch streams every weight once.
bl_status run_decode(const DecodeJob* jobs, int count, int mt, int dev, const DeviceInfo& info,
                     cudaStream_t stream) {
    if (count <= kSmallBatch) return launch_decode_cap<kSmallBatch>(jobs, count, mt, dev, info, stream);
    return launch_decode_cap<BL_MAX_BATCH>(jobs, count, mt, dev, info, stream);
}

// ---- tensor-core GEMM (M > 4) ------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    }
    return fn;
}

// 2-D uint8 tensor [outer, inner] (row stride = inner bytes), tiles of
// box_outer x box_inner; elements outside the tensor read as zero.
bool make_map_2d(CUtensorMap* map, CUtensorMapDataType type, uint64_t elem_bytes, const void* ptr,
                 uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle swizzle);

bool make_map_u8(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t outer,
                 uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
    return make_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ptr, inner, outer, box_inner,
                       box_outer, swizzle);
}

// 2-D tensor [outer, inner] of elem_bytes-wide elements, rows contiguous.
bool make_map_2d(CUtensorMap* map, CUtensorMapDataType type, uint64_t elem_bytes, const void* ptr,
                 uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle swizzle) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) {
        snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled is unavailable");
        return false;
    }
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner * elem_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, type, 2, const_cast<void*>(ptr), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed (%d)", (int)r);
        return false;
    }
    return true;
}

bl_status run_gemm(const DecodeJob& j, int64_t M, int dev, const DeviceInfo& info,
                   cudaStream_t stream) {
    const int8_t* q = j.q;
    const uint8_t* P = j.P;
    void* y = j.y;
    const uint16_t* residual = j.residual;
    const int64_t K = j.K, N = j.N, R = j.packed_rows();
    const int epi = j.epi;
    CUtensorMap map_q, map_p;
    if (!make_map_u8(&map_q, q, (uint64_t)K, (uint64_t)M, kTcBK, kTcBM,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_u8(&map_p, P, (uint64_t)K, (uint64_t)R, kTcBK, kTcPackRows,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
        return BL_ERR_CUDA;
    TcArgs a = {};
    a.P = P;
    a.s_x = j.s_x;
    a.rowsum = j.rowsum;
    a.y = y;
    a.residual = residual;
    a.beta = j.beta;
    a.beta2 = j.beta2;
    a.beta_dev = j.beta_dev;
    a.epi = epi;
    a.M = (int)M;
    a.K = (int)K;
    a.R = (int)R;
    a.N = N;
    a.tiles_n = (int)((R + kTcPackRows - 1) / kTcPackRows);
    a.tiles_m = (int)((M + kTcBM - 1) / kTcBM);
    // 16-byte output accesses need every run of 32 outputs to start 16-byte aligned
    const int64_t out_bytes = (epi == kEpiBF16 || epi == kEpiGateUp) ? 2 : 4;
    a.vec_ok = (R * out_bytes % 16 == 0) && (N * out_bytes % 16 == 0) &&
               (reinterpret_cast<uintptr_t>(y) % 16 == 0) &&
               (!residual || reinterpret_cast<uintptr_t>(residual) % 16 == 0);
    // bf16 y without a residual leaves through TMA stores of 32 x 32 chunks
    // (column offsets i*R + r are multiples of 8 elements when vec_ok holds)
    CUtensorMap map_y = map_q;
    if (a.vec_ok && (epi == kEpiBF16 || epi == kEpiGateUp) && !residual) {
        if (!make_map_2d(&map_y, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, y, (uint64_t)N, (uint64_t)M, 32,
                         32, CU_TENSOR_MAP_SWIZZLE_64B))
            return BL_ERR_CUDA;
        a.tma_store = 1;
    }
    if (prepare_kernel(reinterpret_cast<const void*>(gemm_tc_kernel), dev, info, kTcThreads,
                       kTcSmemBytes) < 0)
        return BL_ERR_CUDA;
    const int64_t tiles = (int64_t)a.tiles_n * a.tiles_m;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(tiles, info.sms));
    // a last wave less than half full runs as N-halves, twice as many units
    const int64_t tail = tiles % grid;
    a.full_units = (tiles > grid && tail > 0 && 2 * tail <= grid) ? tiles - tail : tiles;
    a.units = a.full_units + 2 * (tiles - a.full_units);
    return launch(gemm_tc_kernel, dim3((unsigned)grid), dim3(kTcThreads), (size_t)kTcSmemBytes,
                  stream, map_q, map_p, map_y, a);
}

// A launch epoch for the split-tile counters: never 0, and distinct between
// launches of one process.
unsigned long long next_epoch() {
    static std::atomic<unsigned long long> e{
        0x9E3779B97F4A7C15ull ^
        (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count()};
    unsigned long long v;
    do { v = e.fetch_add(1); } while (v == 0);
    return v;
}

// 5..64 tokens: the weight-streaming tensor-core kernel over up to kSkCap
// problems per launch.  With a workspace of sk_ws_bytes(M) the CTA shares are
// exactly equal (row tiles may be split); without one they are cut at row-tile
// boundaries.
bl_status run_skinny(const DecodeJob* jobs, int count, int64_t M, void* ws, size_t ws_bytes, int dev,
                     const DeviceInfo& info, cudaStream_t stream) {
    const int npad = (int)sk_npad(M);
    const bool ew4 = sk_epi_warps(npad) == 4;
    const int threads = sk_threads(sk_epi_warps(npad));
    const void* kfn = ew4 ? reinterpret_cast<const void*>(skinny_tc_kernel<4>)
                          : reinterpret_cast<const void*>(skinny_tc_kernel<8>);
    if (prepare_kernel(kfn, dev, info, threads, kSkSmemBytes) < 0) return BL_ERR_CUDA;
    static thread_local SkBatch b;  // ~22 KB: kept off the stack
    const bool split = ws && ws_bytes >= (size_t)sk_ws_bytes(M);
    for (int c0 = 0; c0 < count; c0 += kSkCap) {
        const int n = std::min(kSkCap, count - c0);
        b = SkBatch{};
        b.count = n;
        b.M = (int)M;
        b.npad = npad;
        int64_t items = 0;
        for (int i = 0; i < n; ++i) {
            const DecodeJob& j = jobs[c0 + i];
            SkProblem& p = b.p[i];
            p.s_x = j.s_x;
            p.rowsum = j.rowsum;
            p.y = j.y;
            p.residual = j.residual;
            p.N = j.N;
            p.R = (int)j.packed_rows();
            p.K = (int)j.K;
            p.tiles = (p.R + kSkRows - 1) / kSkRows;
            p.kst = (p.K + kSkItemK - 1) / kSkItemK;
            p.beta = j.beta;
            p.beta2 = j.beta2;
            p.beta_dev = j.beta_dev;
            p.epi = j.epi;
            p.item0 = items;
            items += (int64_t)p.tiles * p.kst;
            if (!make_map_u8(&b.tmap_p[i], j.P, (uint64_t)j.K, (uint64_t)p.R, kSkBK, kSkRows,
                             CU_TENSOR_MAP_SWIZZLE_128B) ||
                !make_map_u8(&b.tmap_q[i], j.q, (uint64_t)j.K, (uint64_t)M, kSkBK, (uint32_t)npad,
                             CU_TENSOR_MAP_SWIZZLE_128B))
                return BL_ERR_CUDA;
        }
        b.total = items;
        b.split = split ? 1 : 0;
        if (split) {
            b.ctr = static_cast<unsigned long long*>(ws);
            b.part = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + sk_ctr_bytes());
        }
        b.epoch = next_epoch();
        const int64_t grid = std::max<int64_t>(
            1, std::min<int64_t>(items, std::min<int64_t>(info.sms, kSkMaxGrid)));
        bl_status st = ew4 ? launch(skinny_tc_kernel<4>, dim3((unsigned)grid), dim3((unsigned)threads),
                                    (size_t)kSkSmemBytes, stream, b)
                           : launch(skinny_tc_kernel<8>, dim3((unsigned)grid), dim3((unsigned)threads),
                                    (size_t)kSkSmemBytes, stream, b);
        if (st != BL_OK) return st;
    }
    return BL_OK;
}

// Matmul + epilogue on pre-quantised activations, any M: the decode kernel
// for up to four tokens, the weight-streaming tensor-core kernel for 5..64,
// the tensor-core GEMM beyond.  sk_ws: the optional split workspace of the
// 5..64-token kernel.
bl_status run_job(const DecodeJob& j, int64_t M, int dev, const DeviceInfo& info,
                  cudaStream_t stream, void* sk_ws = nullptr, size_t sk_ws_len = 0) {
    if (M > kSkMaxTokens) return run_gemm(j, M, dev, info, stream);
    if (M > kDecMaxTokens) return run_skinny(&j, 1, M, sk_ws, sk_ws_len, dev, info, stream);
    return run_decode(&j, 1, (int)M, dev, info, stream);
}

bl_status run_quantized(const int8_t* q, const float* s_x, const int32_t* rowsum, const uint8_t* P,
                        float beta, int64_t M, int64_t K, int64_t N, void* y, int epi,
                        const uint16_t* residual, int dev, const DeviceInfo& info,
                        cudaStream_t stream, void* sk_ws = nullptr, size_t sk_ws_len = 0) {
    const DecodeJob j = {q, s_x, rowsum, P, y, residual, K, N, beta, epi};
    return run_job(j, M, dev, info, stream, sk_ws, sk_ws_len);
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
    PackSlots sl;
    for (int i = 0; i < 4; ++i) {
        sl.src[i] = W + (int64_t)i * R * K;
        sl.ws[i] = ws;
    }
    return launch(ternarize_pack_kernel, dim3((unsigned)((work + kPackThreads - 1) / kPackThreads)),
                  dim3(kPackThreads), 0, s, sl, R, K, P);
}

bl_status bitlinear_pack_gate_up_workspace_size(int64_t I, int64_t K, size_t* bytes) {
    if (!bytes) return BL_ERR_NULL;
    bl_status st = check_shape(0, K, 2 * I);
    if (st != BL_OK) return st;
    if (I % 2 != 0) return BL_ERR_SHAPE;
    *bytes = 2 * sizeof(PackWorkspace);
    return BL_OK;
}

bl_status bitlinear_pack_gate_up(const float* W_gate, const float* W_up, int64_t I, int64_t K,
                                 uint8_t* P2, float* beta_out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    size_t need = 0;
    bl_status st = bitlinear_pack_gate_up_workspace_size(I, K, &need);
    if (st != BL_OK) return st;
    if (!W_gate || !W_up || !P2 || !beta_out) return BL_ERR_NULL;
    if (!workspace || workspace_bytes < need) return BL_ERR_WORKSPACE;
    if (!aligned16(W_gate) || !aligned16(W_up) || !aligned16(P2) || !aligned16(workspace))
        return BL_ERR_ALIGN;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    PackWorkspace* ws = static_cast<PackWorkspace*>(workspace);
    const float* W[2] = {W_gate, W_up};
    const int64_t n = I * K;
    for (int h = 0; h < 2; ++h) {  // each projection's own absmean scale
        if ((st = launch(absmean_partial_kernel, dim3(kPackPartials), dim3(kPackThreads), 0, s, W[h],
                         n, ws + h)) != BL_OK)
            return st;
        if ((st = launch(absmean_finalize_kernel, dim3(1), dim3(32), 0, s, n, kPackPartials, ws + h,
                         beta_out + h)) != BL_OK)
            return st;
    }
    const int64_t R = I / 2, work = R * (K / 16);  // packed rows of the [2I, K] concatenation
    PackSlots sl;
    for (int i = 0; i < 4; ++i) {
        sl.src[i] = W[i >> 1] + (int64_t)(i & 1) * R * K;
        sl.ws[i] = ws + (i >> 1);
    }
    return launch(ternarize_pack_kernel, dim3((unsigned)((work + kPackThreads - 1) / kPackThreads)),
                  dim3(kPackThreads), 0, s, sl, R, K, P2);
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
    QuantProblem qp = {x, gain, q, s_x, rowsum, (int)K};
    return run_quant(&qp, 1, M, eps, dev, info, static_cast<cudaStream_t>(stream));
}

bl_status bitlinear_forward_workspace_size(int64_t M, int64_t K, int64_t N, size_t* bytes) {
    if (!bytes) return BL_ERR_NULL;
    bl_status st = check_shape(M, K, N);
    if (st != BL_OK) return st;
    *bytes = M == 0 ? 0 : (size_t)(ws_problem_bytes(M, K) + sk_ws_bytes(M));
    return BL_OK;
}

}  // extern "C"

namespace {

// The forward behind bitlinear_forward and bitlinear_forward_noalloc.  The
// workspace holds the codes, scales and row sums (ws_problem_bytes) and, when
// `need_split` (or when it is large enough anyway), the split-tile tail of the
// 5..64-token kernel; without that tail the kernel cuts its CTA shares at
// row-tile boundaries, with the same results.
bl_status forward_impl(const uint16_t* x, const uint16_t* gain, float eps, const uint8_t* P,
                       float beta, int64_t M, int64_t K, int64_t N, void* y, bl_out_dtype y_dtype,
                       void* workspace, size_t workspace_bytes, bool need_split, void* stream) {
    bl_status st = check_shape(M, K, N);
    if (st != BL_OK) return st;
    const int epi = epi_of(y_dtype);
    if (epi < 0) return BL_ERR_DTYPE;
    if (M == 0) return BL_OK;
    if (!x || !P || !y) return BL_ERR_NULL;
    if (!aligned16(x) || !aligned16(P) || !aligned16(y) || (gain && !aligned16(gain)))
        return BL_ERR_ALIGN;
    const int64_t own = ws_problem_bytes(M, K);
    const int64_t need = own + (need_split ? sk_ws_bytes(M) : 0);
    if (!workspace || workspace_bytes < (size_t)need) return BL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return BL_ERR_ALIGN;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    const WsSlices w = ws_slices(static_cast<char*>(workspace), M, K);
    QuantProblem qp = {x, gain, w.q, w.s_x, w.rowsum, (int)K};
    if ((st = run_quant(&qp, 1, M, eps, dev, info, s)) != BL_OK) return st;
    return run_quantized(w.q, w.s_x, w.rowsum, P, beta, M, K, N, y, epi, nullptr, dev, info, s,
                         static_cast<char*>(workspace) + own, workspace_bytes - (size_t)own);
}

}  // namespace

namespace {

// Positions per split: enough splits for two CTAs per SM over the key/value
// heads, at least 32 positions (one pass of the CTA's four warps) each; more
// splits make the merge, which reads every split's partial, the longer part.
int64_t attn_chunk(int64_t L, int64_t kv_heads, int sms) {
    const int64_t target = std::max<int64_t>(1, (2 * (int64_t)sms + kv_heads - 1) / kv_heads);
    const int64_t per = (L + target - 1) / target;
    return std::max<int64_t>(32, (per + 31) / 32 * 32);
}

bl_status attn_check(int64_t L, int64_t q_heads, int64_t kv_heads, int64_t head_dim) {
    if (L <= 0 || L > INT32_MAX || kv_heads <= 0 || q_heads <= 0 || q_heads % kv_heads != 0)
        return BL_ERR_SHAPE;
    const int64_t group = q_heads / kv_heads;
    if (group != 1 && group != 2 && group != 4 && group != 8) return BL_ERR_SHAPE;
    if (head_dim != 64 && head_dim != 128) return BL_ERR_SHAPE;
    if (kv_heads > 65535 || q_heads > 65535) return BL_ERR_SHAPE;
    // splits <= L / 32 must fit the merge kernel's table
    if ((L + 31) / 32 > kAttnMaxSplits) return BL_ERR_SHAPE;
    return BL_OK;
}

template <int D>
bl_status attn_launch_d(const AttnArgs& a, int group, int64_t splits, int64_t q_heads, uint16_t* out,
                        cudaStream_t stream) {
    const dim3 grid((unsigned)splits, (unsigned)a.kv_heads);
    bl_status st;
    switch (group) {
        case 1: st = launch(attn_split_kernel<D, 1>, grid, dim3(kAttnThreads), 0, stream, a); break;
        case 2: st = launch(attn_split_kernel<D, 2>, grid, dim3(kAttnThreads), 0, stream, a); break;
        case 4: st = launch(attn_split_kernel<D, 4>, grid, dim3(kAttnThreads), 0, stream, a); break;
        default: st = launch(attn_split_kernel<D, 8>, grid, dim3(kAttnThreads), 0, stream, a); break;
    }
    if (st != BL_OK) return st;
    return launch(attn_combine_kernel<D>, dim3((unsigned)q_heads), dim3(D), 0, stream,
                  (const float*)a.part, (int)splits, (int)q_heads, out);
}

}  // namespace

extern "C" {

bl_status bitlinear_forward(const uint16_t* x, const uint16_t* gain, float eps, const uint8_t* P,
                            float beta, int64_t M, int64_t K, int64_t N, void* y,
                            bl_out_dtype y_dtype, void* workspace, size_t workspace_bytes,
                            void* stream) {
    return forward_impl(x, gain, eps, P, beta, M, K, N, y, y_dtype, workspace, workspace_bytes,
                        true, stream);
}

bl_status bitlinear_forward_batch_workspace_size(const bl_problem* probs, int count, int64_t M,
                                                 size_t* bytes) {
    if (!bytes || !probs) return BL_ERR_NULL;
    if (count < 1 || count > BL_MAX_BATCH || M < 0 || M * count > INT32_MAX) return BL_ERR_SHAPE;
    int64_t total = 0;
    for (int i = 0; i < count; ++i) {
        bl_status st = check_shape(M, probs[i].K, probs[i].N);
        if (st != BL_OK) return st;
        total += M == 0 ? 0 : ws_problem_bytes(M, probs[i].K);
    }
    total += sk_ws_bytes(M);
    *bytes = (size_t)total;
    return BL_OK;
}

bl_status bitlinear_forward_batch(const bl_problem* probs, int count, int64_t M, float eps,
                                  void* workspace, size_t workspace_bytes, void* stream) {
    size_t need = 0;
    bl_status st = bitlinear_forward_batch_workspace_size(probs, count, M, &need);
    if (st != BL_OK) return st;
    for (int i = 0; i < count; ++i) {
        const bl_problem& p = probs[i];
        const int epi = epi_of(p.y_dtype);
        if (epi < 0 || (p.residual && epi != kEpiBF16)) return BL_ERR_DTYPE;
        if (M == 0) continue;
        if (!p.x || !p.P || !p.y) return BL_ERR_NULL;
        if (!aligned16(p.x) || !aligned16(p.P) || !aligned16(p.y) ||
            (p.gain && !aligned16(p.gain)) || (p.residual && !aligned16(p.residual)))
            return BL_ERR_ALIGN;
    }
    if (M == 0) return BL_OK;
    if (!workspace || workspace_bytes < need) return BL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return BL_ERR_ALIGN;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    QuantProblem qp[BL_MAX_BATCH];
    DecodeJob jobs[BL_MAX_BATCH];
    char* w = static_cast<char*>(workspace);
    for (int i = 0; i < count; ++i) {
        const bl_problem& p = probs[i];
        const WsSlices sl = ws_slices(w, M, p.K);
        w += ws_problem_bytes(M, p.K);
        qp[i] = {p.x, p.gain, sl.q, sl.s_x, sl.rowsum, (int)p.K};
        jobs[i] = {sl.q, sl.s_x, sl.rowsum, p.P, p.y, p.residual, p.K, p.N, p.beta,
                   epi_of(p.y_dtype)};
    }
    if ((st = run_quant(qp, count, M, eps, dev, info, s)) != BL_OK) return st;
    if (M <= kDecMaxTokens) return run_decode(jobs, count, (int)M, dev, info, s);
    if (skinny_m(M)) return run_skinny(jobs, count, M, w, (size_t)sk_ws_bytes(M), dev, info, s);
    for (int i = 0; i < count; ++i) {
        const DecodeJob& j = jobs[i];
        st = run_quantized(j.q, j.s_x, j.rowsum, j.P, j.beta, M, j.K, j.N, j.y, j.epi, j.residual,
                           dev, info, s);
        if (st != BL_OK) return st;
    }
    return BL_OK;
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

bl_status bitlinear_forward_gate_up(const int8_t* q, const float* s_x, const int32_t* rowsum,
                                    const uint8_t* P2, float beta_gate, float beta_up, int64_t M,
                                    int64_t K, int64_t I, uint16_t* z, void* workspace,
                                    size_t workspace_bytes, void* stream) {
    bl_status st = check_shape(M, K, 2 * I);
    if (st != BL_OK) return st;
    if (I % 2 != 0) return BL_ERR_SHAPE;
    if (M == 0) return BL_OK;
    if (!q || !s_x || !rowsum || !P2 || !z) return BL_ERR_NULL;
    if (!aligned16(q) || !aligned16(P2) || !aligned16(z) || (workspace && !aligned16(workspace)))
        return BL_ERR_ALIGN;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    DecodeJob j = {q, s_x, rowsum, P2, z, nullptr, K, I, beta_gate, kEpiGateUp};
    j.beta2 = beta_up;
    return run_job(j, M, dev, info, static_cast<cudaStream_t>(stream), workspace,
                   workspace ? workspace_bytes : 0);
}

bl_status bitlinear_forward_online_workspace_size(int64_t M, int64_t K, int64_t N,
                                                  size_t* bytes) {
    if (!bytes) return BL_ERR_NULL;
    bl_status st = check_shape(M, K, N);
    if (st != BL_OK) return st;
    *bytes = (size_t)(round_up((int64_t)sizeof(PackWorkspace), 256) + sk_ws_bytes(M));
    return BL_OK;
}

bl_status bitlinear_forward_online(const uint16_t* x, const uint16_t* gain, float eps,
                                   const float* W, int64_t M, int64_t K, int64_t N, void* y,
                                   bl_out_dtype y_dtype, uint8_t* P, float* beta, int8_t* q,
                                   float* s_x, int32_t* rowsum, void* workspace,
                                   size_t workspace_bytes, void* stream) {
    size_t need = 0;
    bl_status st = bitlinear_forward_online_workspace_size(M, K, N, &need);
    if (st != BL_OK) return st;
    const int epi = epi_of(y_dtype);
    if (epi < 0) return BL_ERR_DTYPE;
    if (!W || !P || !beta) return BL_ERR_NULL;
    if (M > 0 && (!x || !y || !q || !s_x || !rowsum)) return BL_ERR_NULL;
    if (!workspace || workspace_bytes < need) return BL_ERR_WORKSPACE;
    if (!aligned16(W) || !aligned16(P) || !aligned16(workspace) || (x && !aligned16(x)) ||
        (y && !aligned16(y)) || (q && !aligned16(q)) || (gain && !aligned16(gain)))
        return BL_ERR_ALIGN;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the weight scale and the packed ternary weights of this call
    PackWorkspace* pw = static_cast<PackWorkspace*>(workspace);
    const int64_t n = N * K, R = N / 4, work = R * (K / 16);
    if ((st = launch(absmean_partial_kernel, dim3(kPackPartials), dim3(kPackThreads), 0, s, W, n,
                     pw)) != BL_OK)
        return st;
    if ((st = launch(absmean_finalize_kernel, dim3(1), dim3(32), 0, s, n, kPackPartials, pw,
                     beta)) != BL_OK)
        return st;
    PackSlots sl;
    for (int i = 0; i < 4; ++i) {
        sl.src[i] = W + (int64_t)i * R * K;
        sl.ws[i] = pw;
    }
    if ((st = launch(ternarize_pack_kernel,
                     dim3((unsigned)((work + kPackThreads - 1) / kPackThreads)),
                     dim3(kPackThreads), 0, s, sl, R, K, P)) != BL_OK)
        return st;
    if (M == 0) return BL_OK;
    // then the forward on them, the rescale reading beta from device memory
    QuantProblem qp = {x, gain, q, s_x, rowsum, (int)K};
    if ((st = run_quant(&qp, 1, M, eps, dev, info, s)) != BL_OK) return st;
    DecodeJob j = {q, s_x, rowsum, P, y, nullptr, K, N, 1.0f, epi};
    j.beta_dev = beta;
    const int64_t own = round_up((int64_t)sizeof(PackWorkspace), 256);
    return run_job(j, M, dev, info, s, static_cast<char*>(workspace) + own,
                   workspace_bytes - (size_t)own);
}

bl_status bitlinear_backward_ste(const float* grad_y, const int8_t* q, const float* s_x,
                                 const uint8_t* P, const float* beta, int64_t M, int64_t K,
                                 int64_t N, float* grad_x, float* grad_w, void* stream) {
    bl_status st = check_shape(M, K, N);
    if (st != BL_OK) return st;
    if (M == 0) return BL_OK;
    if (!grad_y || !beta || (!grad_x && !grad_w)) return BL_ERR_NULL;
    if ((grad_x && !P) || (grad_w && (!q || !s_x))) return BL_ERR_NULL;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const unsigned tk = (unsigned)((K + kSteTile - 1) / kSteTile);
    if (grad_x &&
        (st = launch(ste_grad_input_kernel,
                     dim3(tk, (unsigned)((M + kSteTile - 1) / kSteTile)), dim3(kSteThreads), 0, s,
                     grad_y, P, beta, M, K, N, grad_x)) != BL_OK)
        return st;
    if (grad_w &&
        (st = launch(ste_grad_weight_kernel,
                     dim3(tk, (unsigned)((N + kSteTile - 1) / kSteTile)), dim3(kSteThreads), 0, s,
                     grad_y, q, s_x, M, K, N, grad_w)) != BL_OK)
        return st;
    return BL_OK;
}

bl_status bitlinear_decode_chain_workspace_size(int nsteps, size_t* bytes) {
    if (!bytes) return BL_ERR_NULL;
    if (nsteps < 1 || nsteps > BL_MAX_CHAIN_STEPS) return BL_ERR_SHAPE;
    *bytes = (size_t)(256 + (int64_t)nsteps * (int64_t)sizeof(ChainStep));
    return BL_OK;
}

bl_status bitlinear_decode_chain_prepare(const bl_chain_step* steps, int nsteps, void* workspace,
                                         size_t workspace_bytes) {
    size_t need = 0;
    bl_status st = bitlinear_decode_chain_workspace_size(nsteps, &need);
    if (st != BL_OK) return st;
    if (!steps) return BL_ERR_NULL;
    if (!workspace || workspace_bytes < need) return BL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return BL_ERR_ALIGN;
    std::vector<ChainStep> host((size_t)nsteps);
    for (int i = 0; i < nsteps; ++i) {
        const bl_chain_step& in = steps[i];
        ChainStep& cs = host[(size_t)i];
        if (in.count < 1 || in.count > BL_CHAIN_MAX_PROBLEMS) return BL_ERR_SHAPE;
        if (in.K <= 0 || in.K % 16 != 0 || in.K > kChMaxK) return BL_ERR_SHAPE;
        if (!in.x) return BL_ERR_NULL;
        if (!aligned16(in.x) || (in.gain && !aligned16(in.gain))) return BL_ERR_ALIGN;
        cs = ChainStep{};
        cs.x = in.x;
        cs.gain = in.gain;
        cs.eps = in.eps;
        cs.K = (int)in.K;
        cs.count = in.count;
        int64_t total = 0;
        for (int j = 0; j < in.count; ++j) {
            const bl_chain_problem& pj = in.p[j];
            ChainProblem& cp = cs.p[j];
            if (!pj.P || !pj.y) return BL_ERR_NULL;
            if (!aligned16(pj.P)) return BL_ERR_ALIGN;
            if (pj.kind == BL_CHAIN_GATE_UP) {
                if (pj.N <= 0 || pj.N % 2 != 0 || pj.residual) return BL_ERR_SHAPE;
                cp.epi = kEpiGateUp;
                cp.R = pj.N / 2;
            } else if (pj.kind == BL_CHAIN_BF16 || pj.kind == BL_CHAIN_F32) {
                if (pj.N <= 0 || pj.N % 4 != 0) return BL_ERR_SHAPE;
                if (pj.kind == BL_CHAIN_F32 && pj.residual) return BL_ERR_DTYPE;
                cp.epi = pj.kind == BL_CHAIN_BF16 ? kEpiBF16 : kEpiF32;
                cp.R = pj.N / 4;
            } else {
                return BL_ERR_DTYPE;
            }
            cp.P = pj.P;
            cp.y = pj.y;
            cp.residual = pj.residual;
            cp.N = pj.N;
            cp.beta = pj.beta;
            cp.beta2 = pj.beta_up;
            cp.byte0 = total;
            total += cp.R * in.K;
        }
        cs.total = total;
    }
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    cudaError_t e = cudaMemcpy(static_cast<char*>(workspace) + 256, host.data(),
                               sizeof(ChainStep) * (size_t)nsteps, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        record_cuda_error(e, "cudaMemcpy");
        cudaGetLastError();
        return BL_ERR_CUDA;
    }
    return BL_OK;
}

bl_status bitlinear_decode_chain_run(void* workspace, size_t workspace_bytes, int nsteps,
                                     void* stream) {
    size_t need = 0;
    bl_status st = bitlinear_decode_chain_workspace_size(nsteps, &need);
    if (st != BL_OK) return st;
    if (!workspace || workspace_bytes < need) return BL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return BL_ERR_ALIGN;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int occ = prepare_kernel(reinterpret_cast<const void*>(chain_decode_kernel), dev, info,
                                   kChThreads, kChSmemBytes);
    if (occ < 1) return BL_ERR_CUDA;
    unsigned int* bar = static_cast<unsigned int*>(workspace);
    cudaError_t e = cudaMemsetAsync(bar, 0, sizeof(unsigned int), s);
    if (e != cudaSuccess) {
        record_cuda_error(e, "cudaMemsetAsync");
        cudaGetLastError();
        return BL_ERR_CUDA;
    }
    ChainArgs args;
    args.steps = reinterpret_cast<const ChainStep*>(static_cast<char*>(workspace) + 256);
    args.nsteps = nsteps;
    args.bar = bar;
    return launch_coop(chain_decode_kernel, dim3((unsigned)info.sms), dim3(kChThreads),
                       (size_t)kChSmemBytes, s, args);
}

bl_status bitlinear_quantized_batch_workspace_size(int64_t M, size_t* bytes) {
    if (!bytes) return BL_ERR_NULL;
    if (M < 0) return BL_ERR_SHAPE;
    *bytes = (size_t)sk_ws_bytes(M);
    return BL_OK;
}

bl_status bitlinear_forward_quantized_batch(const bl_quantized_problem* probs, int count,
                                            int64_t M, void* workspace, size_t workspace_bytes,
                                            void* stream) {
    if (!probs) return BL_ERR_NULL;
    if (count < 1 || count > BL_MAX_BATCH || M < 0) return BL_ERR_SHAPE;
    DecodeJob jobs[BL_MAX_BATCH];
    for (int i = 0; i < count; ++i) {
        const bl_quantized_problem& p = probs[i];
        bl_status st = check_shape(M, p.K, p.N);
        if (st != BL_OK) return st;
        const int epi = epi_of(p.y_dtype);
        if (epi < 0 || (p.residual && epi != kEpiBF16)) return BL_ERR_DTYPE;
        if (M == 0) continue;
        if (!p.q || !p.s_x || !p.rowsum || !p.P || !p.y) return BL_ERR_NULL;
        if (!aligned16(p.q) || !aligned16(p.P) || !aligned16(p.y) ||
            (p.residual && !aligned16(p.residual)))
            return BL_ERR_ALIGN;
        jobs[i] = {p.q, p.s_x, p.rowsum, p.P, p.y, p.residual, p.K, p.N, p.beta, epi};
    }
    if (M == 0) return BL_OK;
    int dev;
    DeviceInfo info;
    bl_status st;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M <= kDecMaxTokens) return run_decode(jobs, count, (int)M, dev, info, s);
    if (skinny_m(M)) {
        if (workspace && !aligned16(workspace)) return BL_ERR_ALIGN;
        return run_skinny(jobs, count, M, workspace, workspace_bytes, dev, info, s);
    }
    for (int i = 0; i < count; ++i) {
        const DecodeJob& j = jobs[i];
        st = run_quantized(j.q, j.s_x, j.rowsum, j.P, j.beta, M, j.K, j.N, j.y, j.epi, j.residual,
                           dev, info, s);
        if (st != BL_OK) return st;
    }
    return BL_OK;
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

// ---- attention block: RoPE and grouped-query decode attention ----------------

bl_status bitlinear_rope(const uint16_t* x, const int32_t* pos, int64_t M, int64_t heads,
                         int64_t head_dim, float theta, uint16_t* y, void* stream) {
    if (M < 0 || heads <= 0 || head_dim <= 0 || head_dim % 2 != 0 || head_dim > 1024 ||
        heads > 65535 || M > 65535)
        return BL_ERR_SHAPE;
    if (!(theta > 0.0f) || !std::isfinite(theta)) return BL_ERR_SHAPE;
    if (M == 0) return BL_OK;
    if (!x || !pos || !y) return BL_ERR_NULL;
    int dev;
    DeviceInfo info;
    bl_status st;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    return launch(rope_kernel, dim3((unsigned)heads, (unsigned)M), dim3((unsigned)(head_dim / 2)), 0,
                  static_cast<cudaStream_t>(stream), x, pos, (int)heads, (int)head_dim,
                  std::log((double)theta), y);
}


bl_status bitlinear_attn_decode_workspace_size(int64_t L, int64_t q_heads, int64_t kv_heads,
                                               int64_t head_dim, size_t* bytes) {
    if (!bytes) return BL_ERR_NULL;
    bl_status st;
    if ((st = attn_check(L, q_heads, kv_heads, head_dim)) != BL_OK) return st;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    const int64_t chunk = attn_chunk(L, kv_heads, info.sms);
    const int64_t splits = (L + chunk - 1) / chunk;
    *bytes = (size_t)(splits * q_heads * (head_dim + 2) * 4);
    return BL_OK;
}

bl_status bitlinear_attn_decode(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                                int64_t L, int64_t q_heads, int64_t kv_heads, int64_t head_dim,
                                float scale, uint16_t* out, void* workspace, size_t workspace_bytes,
                                void* stream) {
    bl_status st;
    if ((st = attn_check(L, q_heads, kv_heads, head_dim)) != BL_OK) return st;
    if (!std::isfinite(scale)) return BL_ERR_SHAPE;
    if (!q || !k_cache || !v_cache || !out) return BL_ERR_NULL;
    if (!aligned16(k_cache) || !aligned16(v_cache)) return BL_ERR_ALIGN;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    const int64_t chunk = attn_chunk(L, kv_heads, info.sms);
    const int64_t splits = (L + chunk - 1) / chunk;
    const size_t need = (size_t)(splits * q_heads * (head_dim + 2) * 4);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return BL_ERR_WORKSPACE;
    AttnArgs a = {};
    a.q = q;
    a.k = k_cache;
    a.v = v_cache;
    a.part = static_cast<float*>(workspace);
    a.L = (int)L;
    a.kv_heads = (int)kv_heads;
    a.chunk = (int)chunk;
    a.qscale = scale * kLog2e;
    const int group = (int)(q_heads / kv_heads);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return head_dim == 128 ? attn_launch_d<128>(a, group, splits, q_heads, out, s)
                           : attn_launch_d<64>(a, group, splits, q_heads, out, s);
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

bl_status bitlinear_selftest_wait_timeout(int64_t limit_ns, void* stream) {
    int dev;
    DeviceInfo info;
    bl_status st;
    if ((st = current_device(&dev, &info)) != BL_OK) return st;
    const unsigned long long lim =
        (unsigned long long)std::min<int64_t>(std::max<int64_t>(limit_ns, 1000), 10000000000ll);
    return launch(wait_selftest_kernel, dim3(1), dim3(32), 0, static_cast<cudaStream_t>(stream), lim);
}

bl_status bitlinear_forward_noalloc(const uint16_t* x, const uint16_t* gain, float eps,
                                    const uint8_t* P, float beta, int64_t M, int64_t K,
                                    int64_t N, void* y, bl_out_dtype y_dtype, void* stream) {
    bl_status st = check_shape(M, K, N);
    if (st != BL_OK) return st;
    // the scratch must hold the codes, scales and row sums; the split-tile
    // tail of the 5..64-token kernel is used only when it fits as well
    const int64_t need = M == 0 ? 0 : ws_problem_bytes(M, K);
    if (need > (int64_t)BL_NOALLOC_SCRATCH_BYTES) {
        snprintf(g_last_error, sizeof g_last_error,
                 "bitlinear_forward_noalloc: this shape needs %lld bytes of scratch; the fixed "
                 "scratch holds %u",
                 (long long)need, (unsigned)BL_NOALLOC_SCRATCH_BYTES);
        return BL_ERR_WORKSPACE;
    }
    void* scratch = nullptr;
    if (need > 0) {
        int dev;
        DeviceInfo info;
        if ((st = current_device(&dev, &info)) != BL_OK) return st;
        if ((st = noalloc_scratch(dev, &scratch)) != BL_OK) return st;
    }
    return forward_impl(x, gain, eps, P, beta, M, K, N, y, y_dtype, scratch,
                        need > 0 ? (size_t)BL_NOALLOC_SCRATCH_BYTES : 0, false, stream);
}

}  // extern "C"
