// pack.cuh -- weight preparation: absmean scale, ternary rounding, 2-bit packing.
//
// "Transformers 实战 BitNet 1.58 位量化" walkthrough: section "BitLinear 的三步量化"
// steps 1-2 (scale from the mean of |W| clamped at 1e-5; round, clamp to [-1,1])
// and section "推理侧 BitLinear" (pack_weights: values+1 in two bits, four per
// byte, a quarter of the rows; unpack_weights: mask 3 << 2i, shift, minus one).
// Layout ("block"): bit pair i of packed row r holds output row i*N/4 + r.
//
// The absmean is computed in two deterministic stages: kPackPartials CTAs each
// reduce a fixed strided share of |W| with error-free binary64 accumulation,
// then one CTA merges the partials in index order.  Load-time work; untimed.
#pragma once

#include "common.cuh"
#include "quant.cuh"

namespace bl {

constexpr int kPackThreads = 256;
constexpr int kPackPartials = 296;  // 2 x 148 SMs

struct PackWorkspace {
    double part_hi[kPackPartials];
    double part_lo[kPackPartials];
    float s_w;  // RN32(1 / beta)
};

__global__ void __launch_bounds__(kPackThreads) absmean_partial_kernel(
    const float* __restrict__ W, int64_t n, PackWorkspace* __restrict__ ws) {
    __shared__ QuantScratch<kPackThreads> sc;
    pdl_wait();
    double hi = 0.0, lo = 0.0;
    const int64_t nvec = n >> 2;  // n % 16 == 0
    const float4* wv = reinterpret_cast<const float4*>(W);
    const int64_t stride = (int64_t)gridDim.x * kPackThreads;
    for (int64_t v = (int64_t)blockIdx.x * kPackThreads + threadIdx.x; v < nvec; v += stride) {
        const float4 f = __ldcg(wv + v);
        dd_add(hi, lo, fabs((double)f.x));
        dd_add(hi, lo, fabs((double)f.y));
        dd_add(hi, lo, fabs((double)f.z));
        dd_add(hi, lo, fabs((double)f.w));
    }
    // block_sum_dd returns RN64(hi + lo); keep the pair instead for the merge
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double ohi = __shfl_down_sync(0xffffffffu, hi, o);
        const double olo = __shfl_down_sync(0xffffffffu, lo, o);
        dd_merge(hi, lo, ohi, olo);
    }
    if (lane == 0) { sc.dhi[warp] = hi; sc.dlo[warp] = lo; }
    __syncthreads();
    if (threadIdx.x == 0) {
        double h = sc.dhi[0], l = sc.dlo[0];
        for (int w = 1; w < kPackThreads / 32; ++w) dd_merge(h, l, sc.dhi[w], sc.dlo[w]);
        ws->part_hi[blockIdx.x] = h;
        ws->part_lo[blockIdx.x] = l;
    }
}

// beta = max(RN32(RN64(sum|W|) / (N*K)), 1e-5);  s_w = RN32(1 / beta).
__global__ void absmean_finalize_kernel(int64_t n, int parts, PackWorkspace* __restrict__ ws,
                                        float* __restrict__ beta_out) {
    pdl_wait();
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    double h = __ldcg(&ws->part_hi[0]), l = __ldcg(&ws->part_lo[0]);
    for (int p = 1; p < parts; ++p) dd_merge(h, l, __ldcg(&ws->part_hi[p]), __ldcg(&ws->part_lo[p]));
    const double sum = __dadd_rn(h, l);
    const double mean = __ddiv_rn(sum, (double)n);
    const float beta = fmaxf(__double2float_rn(mean), kScaleFloor);
    ws->s_w = __fdiv_rn(1.0f, beta);
    beta_out[0] = beta;
}

__device__ __forceinline__ uint32_t ternary_code(float w, float s_w) {
    int t = __float2int_rn(__fmul_rn(w, s_w));  // round half to even (saturating)
    t = min(max(t, -1), 1);
    return (uint32_t)(t + 1);
}

// Source of each bit pair (slot) of the packed rows: slot i of packed row r
// takes row r of src[i], ternarised with the scale of ws[i].  One matrix:
// src[i] = W + i*R*K (rows i*N/4 + r), one workspace.  A gate/up pair packed
// as the concatenation [gate; up]: slots 0, 1 from the gate's two row halves
// with the gate's scale, slots 2, 3 from the up projection's with its own.
struct PackSlots {
    const float* src[4];
    const PackWorkspace* ws[4];
};

// One thread: 16 consecutive columns of one packed row (four source rows).
__global__ void __launch_bounds__(kPackThreads) ternarize_pack_kernel(
    const __grid_constant__ PackSlots sl, int64_t R, int64_t K, uint8_t* __restrict__ P) {
    pdl_wait();
    const int64_t cols16 = K >> 4;
    const int64_t idx = (int64_t)blockIdx.x * kPackThreads + threadIdx.x;
    if (idx >= R * cols16) return;
    const int64_t r = idx / cols16, c = idx - r * cols16;
    uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float s_w = __ldcg(&sl.ws[i]->s_w);
        const float4* src = reinterpret_cast<const float4*>(sl.src[i] + r * K + c * 16);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const float4 f = __ldcg(src + v);
            const float e[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)  // column c*16 + 4v + j -> byte 4v + j
                out[v] |= ternary_code(e[j], s_w) << (8 * j + 2 * i);
        }
    }
    reinterpret_cast<uint4*>(P + r * K)[c] = make_uint4(out[0], out[1], out[2], out[3]);
}

__global__ void __launch_bounds__(kPackThreads) pack_ternary_kernel(
    const int8_t* __restrict__ t, int64_t R, int64_t K, uint8_t* __restrict__ P) {
    pdl_wait();
    const int64_t cols16 = K >> 4;
    const int64_t idx = (int64_t)blockIdx.x * kPackThreads + threadIdx.x;
    if (idx >= R * cols16) return;
    const int64_t r = idx / cols16, c = idx - r * cols16;
    uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 u = __ldcg(reinterpret_cast<const uint4*>(t + (i * R + r) * K) + c);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            // each byte b of w[v] is t in {-1,0,1}; code t+1 per byte without carries:
            // (b + 1) & 3 maps 0xFF->0, 0x00->1, 0x01->2
            const uint32_t codes = ((w[v] & 0x7F7F7F7Fu) + 0x01010101u) & 0x03030303u;
            out[v] |= codes << (2 * i);
        }
    }
    reinterpret_cast<uint4*>(P + r * K)[c] = make_uint4(out[0], out[1], out[2], out[3]);
}

__global__ void __launch_bounds__(kPackThreads) unpack_kernel(
    const uint8_t* __restrict__ P, int64_t R, int64_t K, int8_t* __restrict__ t) {
    pdl_wait();
    const int64_t cols16 = K >> 4;
    const int64_t idx = (int64_t)blockIdx.x * kPackThreads + threadIdx.x;
    if (idx >= R * cols16) return;
    const int64_t r = idx / cols16, c = idx - r * cols16;
    const uint4 u = __ldcg(reinterpret_cast<const uint4*>(P + r * K) + c);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t o[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            // per byte: code in {0..3}; code - 1 without borrows between bytes:
            // (code | 0x80) - 1 stays in [0x7F, 0x82], then flip bit 7 back.
            const uint32_t code = (w[v] >> (2 * i)) & 0x03030303u;
            o[v] = ((code | 0x80808080u) - 0x01010101u) ^ 0x80808080u;
        }
        reinterpret_cast<uint4*>(t + (i * R + r) * K)[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace bl
