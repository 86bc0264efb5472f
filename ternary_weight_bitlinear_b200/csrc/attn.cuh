// attn.cuh -- the attention block of the BitNet b1.58 decoder layer around its
// BitLinear projections: rotary position embeddings on q and k, and the
// grouped-query attention of one decode token over its key/value cache.
//
// "BitNet" model doc, model details: the decoder uses rotary position
// embeddings; BitNetConfig: 20 attention heads over hidden 2560 (head
// dimension 128), 5 key/value heads (grouped-query attention), at most 2048
// positions.  The pages give no formulas; these are the textbook ones:
//   RoPE (rotate-half): pair (x[i], x[i + d/2]) of every head turned by
//     a = pos * theta^(-2i/d):  (x[i] cos a - x[i+d/2] sin a, x[i+d/2] cos a + x[i] sin a);
//   attention: query head h reads key/value head h / (H / H_kv);
//     out_h = sum_j softmax_j((q_h . k_j) * scale) v_j over the L cached positions.
// (attn_sub_norm, the RMSNorm in front of o, is the o projection's own
// quantiser norm: bitlinear_forward with a gain.)
//
// Design (B200):
//  * RoPE: one thread per rotated pair; the angle, its sine and cosine and the
//    rotation in binary64, rounded once to bf16 -- the operation is
//    elementwise and tiny next to the projections around it.
//  * Decode attention, split over the cache (one query token is far too
//    little work for one CTA per head): CTA (split, kv head) takes a chunk of
//    positions and all query heads of the group, so each key and value row
//    is read once for the group.  Four lanes score one position against every
//    head of the group (a quarter of the key row each against the group's
//    queries, pre-scaled by scale * log2(e), in shared memory; two shuffles
//    finish the dot products), eight positions a warp pass; the warp keeps an
//    online softmax per head (running max, sum, and output vector: a lane
//    holds d/32 dimensions, the value rows read coalesced by the warp), and
//    the CTA merges its warps into one partial (max, sum, vector) per head in
//    the workspace.  A second kernel merges the splits of each head and
//    writes bf16.  Every step in binary32 with exp2f; tolerance, not bit
//    parity, against the float64 oracle.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace bl {

constexpr int kAttnThreads = 128;  // four warps a CTA
constexpr int kAttnPos = 8;        // positions a warp scores per pass (four lanes each)
constexpr float kLog2e = 1.4426950408889634f;

// y[m, h d + i], y[m, h d + i + d/2] for the pair of thread i of (head h, token m).
__global__ void rope_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ pos, int heads,
                            int d, double log_theta, uint16_t* __restrict__ y) {
    const int h = blockIdx.x, m = blockIdx.y, i = threadIdx.x, half = d >> 1;
    const int64_t base = ((int64_t)m * heads + h) * d;
    pdl_wait();
    pdl_launch_dependents();
    double a = (double)__ldcg(pos + m) * exp(-2.0 * (double)i / (double)d * log_theta);
    // reduce to [-pi, pi] first (a < 2^31 * 1): the error of the reduction,
    // |k| ulp(2 pi), stays far below a bf16 rounding of the result
    const double two_pi = 6.283185307179586;
    a = fma(-rint(a * (1.0 / two_pi)), two_pi, a);
    double s, c;
    sincos(a, &s, &c);
    const double x1 = (double)bf16_bits_to_float(__ldcg(x + base + i));
    const double x2 = (double)bf16_bits_to_float(__ldcg(x + base + i + half));
    y[base + i] = __bfloat16_as_ushort(__double2bfloat16(x1 * c - x2 * s));
    y[base + i + half] = __bfloat16_as_ushort(__double2bfloat16(x2 * c + x1 * s));
}

struct AttnArgs {
    const uint16_t* q;   // bf16 [H * D]
    const uint16_t* k;   // bf16 [L, H_kv, D]
    const uint16_t* v;   // bf16 [L, H_kv, D]
    float* part;         // [splits, H, D + 2]: vector, then max (log2 domain) and sum
    int L;
    int kv_heads;
    int chunk;           // positions per split (a multiple of 32)
    float qscale;        // scale * log2(e)
};

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One split of one key/value head: its NR query heads over positions
// [sp * chunk, min(L, (sp + 1) * chunk)).  A warp takes 8 positions a pass:
// four lanes per position each score a quarter of the head dimension (then
// two shuffles complete the dot products), and each lane accumulates D/32
// output dimensions of the 8 value rows.
template <int D, int NR>
__global__ void __launch_bounds__(kAttnThreads) attn_split_kernel(const AttnArgs a) {
    constexpr int DL = D / 32;      // output dimensions per lane
    constexpr int DP = D / 4;       // score dimensions per lane (a quarter of the head)
    constexpr int NW = kAttnThreads / 32;
    __shared__ float qs[NR][D];
    __shared__ float wm[NW][NR], wl[NW][NR];
    __shared__ float wo[NW][NR][D];
    const int g = blockIdx.y, sp = blockIdx.x;
    const int H = a.kv_heads * NR;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int jl = lane >> 2, part = lane & 3;  // this lane's position in the pass, quarter of the head
    const int j0 = sp * a.chunk, j1 = min(a.L, j0 + a.chunk);
    pdl_wait();
    pdl_launch_dependents();
    for (int t = threadIdx.x; t < NR * D; t += kAttnThreads)
        qs[t / D][t % D] = __fmul_rn(bf16_bits_to_float(__ldcg(a.q + (int64_t)g * NR * D + t)), a.qscale);
    __syncthreads();

    float m[NR], l[NR], o[NR][DL];
#pragma unroll
    for (int h = 0; h < NR; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.0f;
#pragma unroll
        for (int e = 0; e < DL; ++e) o[h][e] = 0.0f;
    }
    const int64_t row_stride = (int64_t)a.kv_heads * D;  // elements between positions
    for (int jb = j0 + kAttnPos * warp; jb < j1; jb += kAttnPos * NW) {
        // every load of the pass in flight at once: this lane's quarter of its
        // position's key row, and its D/32 dimensions of the pass's value rows
        const int j = jb + jl;
        const bool valid = j < j1;
        uint4 kr[DP / 8];
        if (valid) {
            const uint4* kp =
                reinterpret_cast<const uint4*>(a.k + (int64_t)j * row_stride + (int64_t)g * D + part * DP);
#pragma unroll
            for (int c = 0; c < DP / 8; ++c) kr[c] = __ldcg(kp + c);
        }
        uint32_t vr[kAttnPos][DL / 2];
        const uint16_t* vbase = a.v + (int64_t)jb * row_stride + (int64_t)g * D + lane * DL;
#pragma unroll
        for (int b = 0; b < kAttnPos; ++b) {
            if (jb + b < j1) {  // warp-uniform
                const uint16_t* vp = vbase + (int64_t)b * row_stride;
                if constexpr (DL == 4) {
                    const uint2 vv = __ldcg(reinterpret_cast<const uint2*>(vp));
                    vr[b][0] = vv.x;
                    vr[b][1] = vv.y;
                } else {
                    vr[b][0] = __ldcg(reinterpret_cast<const uint32_t*>(vp));
                }
            } else {
#pragma unroll
                for (int e = 0; e < DL / 2; ++e) vr[b][e] = 0u;
            }
        }
        // scores (log2 domain): a quarter dot product per lane, then the four lanes' sum
        float s[NR];
#pragma unroll
        for (int h = 0; h < NR; ++h) s[h] = 0.0f;
        if (valid) {
#pragma unroll
            for (int c = 0; c < DP / 8; ++c) {
                const uint32_t w[4] = {kr[c].x, kr[c].y, kr[c].z, kr[c].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float k0 = bf16_bits_to_float(w[e] & 0xFFFFu), k1 = bf16_bits_to_float(w[e] >> 16);
                    const int dd = part * DP + 8 * c + 2 * e;
#pragma unroll
                    for (int h = 0; h < NR; ++h) {
                        s[h] = fmaf(k0, qs[h][dd], s[h]);
                        s[h] = fmaf(k1, qs[h][dd + 1], s[h]);
                    }
                }
            }
        }
#pragma unroll
        for (int h = 0; h < NR; ++h) {
            s[h] += __shfl_xor_sync(0xffffffffu, s[h], 1);
            s[h] += __shfl_xor_sync(0xffffffffu, s[h], 2);
            if (!valid) s[h] = -INFINITY;
        }
        // online softmax over the pass's positions (position jb is valid)
        float p[NR];
#pragma unroll
        for (int h = 0; h < NR; ++h) {
            const float mn = fmaxf(m[h], warp_max_f(s[h]));
            const float alpha = exp2f(m[h] - mn);  // 0 on the first pass (m = -inf)
            p[h] = exp2f(s[h] - mn);               // 0 for positions past the chunk
            l[h] = fmaf(l[h], alpha, warp_sum_f(part == 0 ? p[h] : 0.0f));
#pragma unroll
            for (int e = 0; e < DL; ++e) o[h][e] *= alpha;
            m[h] = mn;
        }
        // weighted values (rows past the chunk are zeros with weight 0)
#pragma unroll
        for (int b = 0; b < kAttnPos; ++b) {
            float vf[DL];
#pragma unroll
            for (int e = 0; e < DL / 2; ++e) {
                vf[2 * e] = bf16_bits_to_float(vr[b][e] & 0xFFFFu);
                vf[2 * e + 1] = bf16_bits_to_float(vr[b][e] >> 16);
            }
#pragma unroll
            for (int h = 0; h < NR; ++h) {
                const float pj = __shfl_sync(0xffffffffu, p[h], 4 * b);
#pragma unroll
                for (int e = 0; e < DL; ++e) o[h][e] = fmaf(pj, vf[e], o[h][e]);
            }
        }
    }
    // merge the warps: one (max, sum, vector) per head for this split
#pragma unroll
    for (int h = 0; h < NR; ++h) {
        if (lane == 0) {
            wm[warp][h] = m[h];
            wl[warp][h] = l[h];
        }
#pragma unroll
        for (int e = 0; e < DL; ++e) wo[warp][h][lane * DL + e] = o[h][e];
    }
    __syncthreads();
    for (int t = threadIdx.x; t < NR * D; t += kAttnThreads) {
        const int h = t / D, dd = t % D;
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) mx = fmaxf(mx, wm[w][h]);
        float acc = 0.0f, sum = 0.0f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float f = wm[w][h] == -INFINITY ? 0.0f : exp2f(wm[w][h] - mx);  // warps with no position
            acc = fmaf(f, wo[w][h][dd], acc);
            sum = fmaf(f, wl[w][h], sum);
        }
        float* dst = a.part + ((int64_t)sp * H + (int64_t)g * NR + h) * (D + 2);
        dst[dd] = acc;
        if (dd == 0) {
            dst[D] = mx;
            dst[D + 1] = sum;
        }
    }
}

// out[h, :] = bf16(sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s), M = max_s m_s.
// The splits' maxima and sums are staged in shared memory first (one load a
// thread), so the per-dimension loop issues its vector loads back to back.
constexpr int kAttnMaxSplits = 1024;

template <int D>
__global__ void __launch_bounds__(D) attn_combine_kernel(const float* __restrict__ part, int splits, int H,
                                                        uint16_t* __restrict__ out) {
    __shared__ float wsh[kAttnMaxSplits];
    __shared__ float lsh[kAttnMaxSplits];
    __shared__ float mxs;
    const int h = blockIdx.x, dd = threadIdx.x;
    pdl_wait();
    pdl_launch_dependents();
    for (int sp = dd; sp < splits; sp += D) {
        const float* p = part + ((int64_t)sp * H + h) * (D + 2);
        wsh[sp] = __ldcg(p + D);
        lsh[sp] = __ldcg(p + D + 1);
    }
    __syncthreads();
    if (dd < 32) {
        float m = -INFINITY;
        for (int sp = dd; sp < splits; sp += 32) m = fmaxf(m, wsh[sp]);
        m = warp_max_f(m);
        if (dd == 0) mxs = m;
    }
    __syncthreads();
    const float mx = mxs;
    for (int sp = dd; sp < splits; sp += D) wsh[sp] = exp2f(wsh[sp] - mx);
    __syncthreads();
    float num = 0.0f, den = 0.0f;
#pragma unroll 8
    for (int sp = 0; sp < splits; ++sp) {
        const float f = wsh[sp];
        num = fmaf(f, __ldcg(part + ((int64_t)sp * H + h) * (D + 2) + dd), num);
        den = fmaf(f, lsh[sp], den);
    }
    out[(int64_t)h * D + dd] = __bfloat16_as_ushort(__float2bfloat16_rn(num / den));
}

}  // namespace bl
