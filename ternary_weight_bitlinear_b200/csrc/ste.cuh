// ste.cuh -- the backward of a BitLinear layer in quantisation-aware training.
//
// "Transformers 实战 BitNet 1.58 位量化" walkthrough, "BitLinear 的三步量化":
// the weight and activation quantisers are trained with the straight-through
// estimator (their backward passes the gradient on unchanged), so the layer's
// gradients are those of a linear layer on the dequantised operands the
// forward multiplied:
//   W_q[n,k] = RN32(t[n,k] / s_w), s_w = RN32(1/beta)  -> t * RN32(1/s_w)
//   x_q[m,k] = RN32(q[m,k] / s_x[m])
//   gx[m,k] = sum_n gy[m,n] W_q[n,k]      gw[n,k] = sum_m gy[m,n] x_q[m,k]
// Two tiled binary32 kernels (64 x 64 outputs per CTA, 4 x 4 per thread,
// 16-deep chunks of the reduction staged in shared memory; each product is
// added with one fused multiply-add).  The ternary weights are unpacked from
// the 2-bit block layout as the tiles load (row n = i*N/4 + r is bit pair i of
// packed row r); x_q is formed from the int8 codes and the token's scale as
// its tile loads.  Training-side work, off the inference hot path.
#pragma once

#include "common.cuh"

namespace bl {

constexpr int kSteTile = 64;
constexpr int kSteDepth = 16;
constexpr int kSteThreads = 256;

// gx = gy [M,N] x W_q [N,K]; beta read from device memory.
__global__ void __launch_bounds__(kSteThreads) ste_grad_input_kernel(
    const float* __restrict__ gy, const uint8_t* __restrict__ P, const float* __restrict__ beta_dev,
    int64_t M, int64_t K, int64_t N, float* __restrict__ gx) {
    __shared__ float sg[kSteDepth][kSteTile + 1];  // [n][m]
    __shared__ float sw[kSteDepth][kSteTile];      // [n][k]
    pdl_wait();
    pdl_launch_dependents();
    const float s_w = __fdiv_rn(1.0f, __ldcg(beta_dev));
    const float wmag = __fdiv_rn(1.0f, s_w);  // |W_q| of a nonzero ternary weight
    const int64_t R = N / 4;
    const int64_t m0 = (int64_t)blockIdx.y * kSteTile, k0 = (int64_t)blockIdx.x * kSteTile;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;  // 16 x 16 threads, 4 x 4 outputs each
    float acc[4][4] = {};
    for (int64_t n0 = 0; n0 < N; n0 += kSteDepth) {
        for (int e = threadIdx.x; e < kSteDepth * kSteTile; e += kSteThreads) {
            {  // gy: 64 m x 16 n, consecutive threads along n
                const int dn = e % kSteDepth, c = e / kSteDepth;
                const int64_t m = m0 + c, n = n0 + dn;
                sg[dn][c] = (m < M && n < N) ? __ldcg(gy + m * N + n) : 0.0f;
            }
            {  // W_q: 16 n x 64 k, consecutive threads along k
                const int dn = e / kSteTile, c = e % kSteTile;
                const int64_t n = n0 + dn, k = k0 + c;
                float w = 0.0f;
                if (n < N && k < K) {
                    const int64_t i = n / R, r = n - i * R;
                    const int code = (int)((__ldcg(P + r * K + k) >> (2 * i)) & 3u);
                    w = __fmul_rn((float)(code - 1), wmag);  // t * |W_q|, exact
                }
                sw[dn][c] = w;
            }
        }
        __syncthreads();
#pragma unroll
        for (int dn = 0; dn < kSteDepth; ++dn) {
            float a[4], w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = sg[dn][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = sw[dn][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(a[i], w[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t m = m0 + ty * 4 + i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t k = k0 + tx * 4 + j;
            if (k < K) gx[m * K + k] = acc[i][j];
        }
    }
}

// gw = gy^T [N,M] x x_q [M,K].
__global__ void __launch_bounds__(kSteThreads) ste_grad_weight_kernel(
    const float* __restrict__ gy, const int8_t* __restrict__ q, const float* __restrict__ s_x,
    int64_t M, int64_t K, int64_t N, float* __restrict__ gw) {
    __shared__ float sg[kSteDepth][kSteTile + 1];  // [m][n]
    __shared__ float sx[kSteDepth][kSteTile];      // [m][k]
    pdl_wait();
    pdl_launch_dependents();
    const int64_t n0 = (int64_t)blockIdx.y * kSteTile, k0 = (int64_t)blockIdx.x * kSteTile;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4] = {};
    for (int64_t m0 = 0; m0 < M; m0 += kSteDepth) {
        for (int e = threadIdx.x; e < kSteDepth * kSteTile; e += kSteThreads) {
            const int dm = e / kSteTile, c = e % kSteTile;
            const int64_t m = m0 + dm, n = n0 + c, k = k0 + c;
            sg[dm][c] = (m < M && n < N) ? __ldcg(gy + m * N + n) : 0.0f;
            sx[dm][c] = (m < M && k < K)
                            ? __fdiv_rn((float)__ldcg(q + m * K + k), __ldcg(s_x + m))
                            : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int dm = 0; dm < kSteDepth; ++dm) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = sg[dm][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = sx[dm][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t n = n0 + ty * 4 + i;
        if (n >= N) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t k = k0 + tx * 4 + j;
            if (k < K) gw[n * K + k] = acc[i][j];
        }
    }
}

}  // namespace bl
