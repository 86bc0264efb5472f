// glue.cuh -- elementwise FFN glue between BitLinear projections, and the
// self-test kernel of the bounded waits.
//
// "BitNet" transformers model doc, model details: the FFN uses squared ReLU
// (hidden_act "relu2") in a gated form, z = relu(gate)^2 * up, computed here
// as bf16(RN32(RN32(relu(a) * relu(a)) * b)).
#pragma once

#include "common.cuh"

namespace bl {

constexpr int kGlueThreads = 256;

// One thread: 8 consecutive elements (one 16-byte vector), or the scalar tail.
__global__ void __launch_bounds__(kGlueThreads) relu2_mul_kernel(const uint16_t* __restrict__ a,
                                                                 const uint16_t* __restrict__ b,
                                                                 int64_t n,
                                                                 uint16_t* __restrict__ z) {
    pdl_wait();
    pdl_launch_dependents();
    const int64_t base = ((int64_t)blockIdx.x * kGlueThreads + threadIdx.x) * 8;
    if (base >= n) return;
    if (base + 8 <= n) {
        const uint4 ua = __ldcg(reinterpret_cast<const uint4*>(a + base));
        const uint4 ub = __ldcg(reinterpret_cast<const uint4*>(b + base));
        const uint32_t wa[4] = {ua.x, ua.y, ua.z, ua.w};
        const uint32_t wb[4] = {ub.x, ub.y, ub.z, ub.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            o[j] = (uint32_t)relu2_mul_one(wa[j] & 0xFFFFu, wb[j] & 0xFFFFu) |
                   ((uint32_t)relu2_mul_one(wa[j] >> 16, wb[j] >> 16) << 16);
        *reinterpret_cast<uint4*>(z + base) = make_uint4(o[0], o[1], o[2], o[3]);
    } else {
        for (int64_t i = base; i < n; ++i) z[i] = relu2_mul_one(__ldcg(a + i), __ldcg(b + i));
    }
}

// Self-test of the bounded waits: thread 0 waits on a barrier nothing arrives
// on until limit_ns pass, then records the timeout and returns.
__global__ void wait_selftest_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar), 1);
        mbar_init_fence();
    }
    __syncthreads();
    if (threadIdx.x != 0) return;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t n = 0;; ++n) {
        if (mbar_try_wait(smem_addr(&bar), 0)) return;
        if ((n & 255u) == 0 && globaltimer_ns() - t0 > limit_ns) {
            atomicOr(&g_status, kStatusTimeout);
            return;
        }
    }
}

}  // namespace bl
