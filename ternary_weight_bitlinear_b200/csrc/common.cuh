// common.cuh -- device helpers shared by the BitLinear kernels (sm_100a).
//
// Inline PTX for the pieces CUDA C++ does not expose directly: mbarriers,
// bulk asynchronous copies (TMA engine, non-multicast), proxy fences,
// programmatic dependent launch and the global timer used to bound waits.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace bl {

constexpr float kScaleFloor = 1e-5f;  // clamp floor of both scales (absmean, absmax)

// Device status word: bit 0 = a bounded wait expired.  Read and cleared by
// bitlinear_device_status().
__device__ unsigned int g_status;
constexpr unsigned int kStatusTimeout = 1u;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) {
    return __uint_as_float(b << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---- mbarrier --------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async proxy (bulk copies) and the
// rest of the CTA; follow with __syncthreads().
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of the barrier to complete, for at most kWaitLimitNs.
// On expiry records kStatusTimeout and returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 255u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_status, kStatusTimeout);
            return false;
        }
    }
}

// ---- bulk copies (TMA engine, no multicast) ---------------------------------
// Global -> this CTA's shared memory; completion counted in bytes on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Same, with an L2 evict-first hint for data read exactly once (streamed weights).
__device__ __forceinline__ void bulk_g2s_stream(uint32_t dst, const void* src, uint32_t bytes,
                                                uint32_t bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy accesses (a bulk copy refilling a buffer just read).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- asynchronous 16-byte copies (L2 only, so coherent with the previous kernel)
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem_dst)), "l"(gsrc)
                 : "memory");
}
// Wait for every cp.async this thread issued.
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// ---- programmatic dependent launch -----------------------------------------
// Block until the grids this one depends on have completed and their memory
// is visible (no-op when launched without the PDL attribute).
__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Allow the next grid in the stream to begin launching.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- correctly rounded division by a reused divisor ---------------------------
// RN(a / s) for a divisor s > 0 shared by many quotients (a token's scale).
// With y = RN(1/s) computed once, q = RN(a*y) is refined by one FMA step
// (Markstein's correction, q + (a - q*s)*y), which leaves q a faithful
// rounding of a/s.  The remainder a - q*s of a faithful quotient is exactly
// representable, so one more FMA gives it exactly, and q = RN(a/s) holds iff
// |a - q*s| < ulp(q)*s/2: the floats next to q are one ulp(q) away when q is
// not a power of two, and a/s is never a midpoint (it would need more than
// 24 significant bits times s to equal a).  Where that check cannot vouch for
// q -- a zero, tiny, huge or non-finite operand, q a power of two, or the
// bound failing -- the quotient comes from __fdiv_rn instead.
struct RecipDiv {
    float s;
    float y;
};

__device__ __forceinline__ RecipDiv recip_div_init(float s) { return {s, __frcp_rn(s)}; }

__device__ __forceinline__ float recip_div(float a, const RecipDiv& d) {
    float q = __fmul_rn(a, d.y);
    q = __fmaf_rn(__fmaf_rn(-q, d.s, a), d.y, q);
    const float r = __fmaf_rn(-q, d.s, a);
    const uint32_t qb = __float_as_uint(q);
    const uint32_t e = (qb >> 23) & 0xFFu;                  // biased exponent of q
    const float half_ulp = __uint_as_float((e - 24u) << 23);  // ulp(q)/2 = 2^(e-151)
    const float h = __fmul_rn(half_ulp, d.s);               // exact when normal
    const uint32_t ab = __float_as_uint(a) & 0x7FFFFFFFu;
    const bool ok = ab >= 0x0D800000u && ab <= 0x71800000u &&  // 2^-100 <= |a| <= 2^100
                    e >= 25u && e <= 253u && (qb & 0x007FFFFFu) != 0u &&
                    __float_as_uint(h) >= 0x00800000u && fabsf(r) < h;
    if (ok) return q;
    return __fdiv_rn(a, d.s);
}

// The rescale y = RN32(RN32(acc * beta) / s) for many outputs sharing a
// token's divisor s.  Same method as recip_div, split so that the common case
// has no branch: when beta and s both lie in [2^-40, 2^40] and
// 1 <= |acc| <= 2^31, a = RN(acc*beta) lies in [2^-40, 2^71] and q in
// [2^-80, 2^111], so every intermediate is a normal float and only the
// rounding test itself (and q a power of two) is left per output; acc = 0
// gives a = q = +0 exactly (beta > 0).  Outputs whose test fails, or any
// divisor or beta outside the range, go through scale_slow.
struct PairDiv {
    float s;
    float y;   // RN(1/s)
    float ns;  // -s
    bool fast;
};

__device__ __forceinline__ PairDiv pair_div_init(float s, float beta) {
    const bool fast = s >= 0x1p-40f && s <= 0x1p40f && beta >= 0x1p-40f && beta <= 0x1p40f;
    return {s, __frcp_rn(s), -s, fast};
}

// Candidate quotient; ok is set when it is proven to be RN(a/s).
__device__ __forceinline__ float scale_fast(int acc, float beta, const PairDiv& d, bool& ok) {
    const float a = __fmul_rn(__int2float_rn(acc), beta);
    float q = __fmul_rn(a, d.y);
    q = __fmaf_rn(__fmaf_rn(q, d.ns, a), d.y, q);
    const float r = __fmaf_rn(q, d.ns, a);  // exact remainder of the faithful q
    const uint32_t qb = __float_as_uint(q);
    // ulp(q)/2 * s, exact: a power of two times s, normal in this range
    const float h = __fmul_rn(__uint_as_float((qb & 0x7F800000u) - 0x0C000000u), d.s);
    ok = acc == 0 || ((qb & 0x007FFFFFu) != 0u && fabsf(r) < h);
    return q;
}

__device__ __noinline__ float scale_slow(int acc, float beta, float s, float y) {
    return recip_div(__fmul_rn(__int2float_rn(acc), beta), RecipDiv{s, y});
}

// The gated squared-ReLU of the FFN block ("BitNet" transformers model doc,
// model details: hidden_act relu2, gated): z = bf16(RN32(RN32(relu(a)^2) * b))
// for bf16 a (gate output) and b (up output).
__device__ __forceinline__ uint16_t relu2_mul_one(uint32_t a_bits, uint32_t b_bits) {
    const float av = bf16_bits_to_float(a_bits);
    const float ra = av > 0.0f ? av : 0.0f;
    return float_to_bf16_bits(__fmul_rn(__fmul_rn(ra, ra), bf16_bits_to_float(b_bits)));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ---- integer dot products ----------------------------------------------------
// d = c + sum_{j<4} a.u8[j] * b.s8[j]
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// ---- error-free binary64 accumulation ----------------------------------------
// (hi, lo) holds a running sum; add v with TwoSum so the rounding error of the
// hi addition is carried exactly into lo.  Explicit _rn intrinsics keep the
// compiler from contracting or reassociating.
__device__ __forceinline__ void dd_add(double& hi, double& lo, double v) {
    const double s = __dadd_rn(hi, v);
    const double bv = __dsub_rn(s, hi);
    const double av = __dsub_rn(s, bv);
    const double e = __dadd_rn(__dsub_rn(hi, av), __dsub_rn(v, bv));
    hi = s;
    lo = __dadd_rn(lo, e);
}

__device__ __forceinline__ void dd_merge(double& hi, double& lo, double ohi, double olo) {
    dd_add(hi, lo, ohi);
    lo = __dadd_rn(lo, olo);
}

}  // namespace bl
