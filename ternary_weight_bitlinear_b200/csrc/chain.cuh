// chain.cuh -- one token through a chain of dependent BitLinear steps in a
// single persistent launch (decode with the layers in order).
//
// A step is the BitLinear forward ("Transformers 实战 BitNet 1.58 位量化"
// walkthrough, "推理侧 BitLinear": RMSNorm, activation_quant, unpack, F.linear,
// post_quant_process) of up to four projections that share one input row,
// with the outputs of the decode kernel (bf16 / fp32, the residual add of a
// decoder block, the fused gate|up relu^2 of the FFN block, "BitNet" model
// doc, model details).  Step s + 1 may read what step s wrote (its input row,
// its residual), so steps are separated by a grid-wide barrier.
//
// Design (B200):
//  * One CTA per SM, launched cooperatively (all CTAs resident, which the
//    grid barrier needs); 16 warps, each streaming its byte share of every
//    step's packed rows through its own ring of bulk copies, as the decode
//    kernel does.  The walk over a warp's copies runs across step
//    boundaries: weights are constant, so the ring keeps fetching the next
//    steps' rows while the CTA waits at the barrier and quantises the next
//    input -- the weight stream never stops for a launch.
//  * At each step every CTA quantises the step's input row itself (the
//    quantiser's block routine, bit for bit the quantise kernel) into shared
//    memory: no separate quantise launch and no round trip through memory.
//  * The barrier: thread 0 of each CTA counts in on a global counter (zeroed
//    before the launch) after the CTA's outputs are written and fenced, then
//    waits for the count of the step; the wait is bounded (2 s of
//    %globaltimer; on expiry the status word records a timeout and the kernel
//    unwinds).
#pragma once

#include "common.cuh"
#include "decode.cuh"
#include "quant.cuh"

namespace bl {

constexpr int kChMaxProbs = 4;
constexpr int kChMaxK = 8192;
constexpr int kChThreads = kDecThreads;
constexpr int kChWarps = kDecWarps;
constexpr int kChVpt = kChMaxK / (8 * kChThreads);  // 16-byte vectors of the row per thread
// dynamic shared memory: barriers | rings | descriptor queues | codes | gain
constexpr int kChOffRings = kDecBarBytes;
constexpr int kChOffDescs = kChOffRings + kDecSlotBytes;
constexpr int kChOffCodes = kChOffDescs + kDecDescBytes;
constexpr int kChOffGain = kChOffCodes + kChMaxK;
constexpr int kChSmemBytes = kChOffGain + 2 * kChMaxK;
static_assert(kChVpt * 8 * kChThreads == kChMaxK, "row split");
static_assert(kChSmemBytes <= 227 * 1024 - (int)sizeof(QuantScratch<kChThreads>) - 64, "shared memory");

struct ChainProblem {
    const uint8_t* P;          // [R,K] packed
    void* y;                   // [N] output
    const uint16_t* residual;  // bf16 [N] or nullptr
    int64_t R;                 // packed rows
    int64_t N;                 // outputs
    int64_t byte0;             // first byte of this problem within the step
    float beta;
    float beta2;               // kEpiGateUp: the up projection's scale
    int epi;
};

struct ChainStep {
    const uint16_t* x;         // bf16 [K] input row
    const uint16_t* gain;      // bf16 [K] RMSNorm weight or nullptr
    float eps;
    int K;
    int count;
    int64_t total;             // packed bytes of the step
    ChainProblem p[kChMaxProbs];
};

struct ChainArgs {
    const ChainStep* steps;    // device array
    int nsteps;
    unsigned int* bar;         // grid barrier counter, zero at launch
};

// A warp's walk over (step, problem, row, chunk) items: in every step, the
// rows whose first byte lies in the warp's share [gw*T/W, (gw+1)*T/W) of the
// step's T packed bytes; then the next step.
struct ChainWalker {
    const ChainStep* st;
    int nsteps;
    int64_t gw, W;
    int s;          // current step (nsteps once the walk is over)
    int p;          // problem in the step
    int64_t r, r_end, R;
    int c;          // chunk of the row
    int K;
    int max_rows;
    int64_t hi;     // end of the warp's share in this step
    const uint8_t* P;

    __device__ __forceinline__ void enter(int np, int64_t r0) {
        p = np;
        c = 0;
        const ChainProblem& pr = st[s].p[p];
        R = pr.R;
        P = pr.P;
        const int64_t lim = hi - pr.byte0;  // rows with first byte < hi
        r_end = lim <= 0 ? 0 : min((lim + K - 1) / K, R);
        r = min(r0, R);
    }
    __device__ __forceinline__ void enter_step(int ns) {
        for (s = ns; s < nsteps; ++s) {
            const ChainStep& cs = st[s];
            K = cs.K;
            max_rows = K <= kDecChunk ? min(kDecMaxRows, kDecChunk / K) : 1;
            const int64_t lo = gw * cs.total / W;
            hi = (gw + 1) * cs.total / W;
            int pp = 0;
            while (pp + 1 < cs.count && cs.p[pp + 1].byte0 <= lo) ++pp;
            enter(pp, (lo - cs.p[pp].byte0 + K - 1) / K);
            if (settle_in_step()) return;
        }
    }
    // moves past exhausted problems of the step; false when the share ends
    __device__ __forceinline__ bool settle_in_step() {
        while (r >= r_end) {
            if (r_end < R || p + 1 >= st[s].count) return false;  // the share ends here
            enter(p + 1, 0);
        }
        return true;
    }
    __device__ __forceinline__ void start(const ChainStep* steps, int n, int64_t g, int64_t w) {
        st = steps;
        nsteps = n;
        gw = g;
        W = w;
        enter_step(0);
    }
    __device__ __forceinline__ bool valid() const { return s < nsteps; }
    __device__ __forceinline__ int rows() const { return (int)min((int64_t)max_rows, r_end - r); }
    __device__ __forceinline__ int bytes() const {
        return K <= kDecChunk ? rows() * K : min(kDecChunk, K - c * kDecChunk);
    }
    __device__ __forceinline__ bool last_chunk() const {
        return K <= kDecChunk || (c + 1) * kDecChunk >= K;
    }
    __device__ __forceinline__ const uint8_t* src() const { return P + r * K + c * kDecChunk; }
    __device__ __forceinline__ void advance() {
        if (!last_chunk()) { ++c; return; }
        r += rows();
        c = 0;
        if (!settle_in_step()) enter_step(s + 1);
    }
};

__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Per-warp partials of the chain quantiser's three reductions.
struct ChainQuantScratch {
    double d[kChWarps];
    double d2[kChWarps];
    float f[kChWarps];
    int i[kChWarps];
};

// The step's input row quantised by the whole CTA: the same arithmetic as
// quantize_row (the RMS factor decided by the bounded binary64 sum, else the
// error-free sum; max |h|; codes rounded half to even), so the same codes,
// scale and row sum bit for bit, with the row held in registers, the gain
// already in shared memory (gs, or nullptr for no norm) and three CTA barriers.
__device__ void chain_quantize(const uint16_t* __restrict__ x, const uint4* gs, float eps, int K,
                               int8_t* q, ChainQuantScratch& sc, float& s_out, int& rs_out) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nvec = K >> 3;
    const uint4* xv = reinterpret_cast<const uint4*>(x);
    uint4 xr[kChVpt];
#pragma unroll
    for (int j = 0; j < kChVpt; ++j) {
        const int v = threadIdx.x + j * kChThreads;
        xr[j] = v < nvec ? __ldcg(xv + v) : make_uint4(0u, 0u, 0u, 0u);  // zeros add nothing
    }
    float r = 1.0f;
    if (gs) {
        double ss = 0.0;  // plain binary64 sum of the exact squares (any order: bounded below)
#pragma unroll
        for (int j = 0; j < kChVpt; ++j) {
            float f[8];
            unpack8_bf16(xr[j], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = __fma_rn((double)f[e], (double)f[e], ss);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
        if (lane == 0) sc.d[warp] = ss;
        __syncthreads();
        double approx = 0.0;
        for (int w = 0; w < kChWarps; ++w) approx = __dadd_rn(approx, sc.d[w]);
        if (!rms_factor_bounded(approx, K, eps, r)) {  // every thread decides alike
            double hi = 0.0, lo = 0.0;
#pragma unroll
            for (int j = 0; j < kChVpt; ++j) {
                float f[8];
                unpack8_bf16(xr[j], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const double dv = (double)f[e];
                    dd_add(hi, lo, __dmul_rn(dv, dv));  // exact square of a bf16 value
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const double ohi = __shfl_down_sync(0xffffffffu, hi, o);
                const double olo = __shfl_down_sync(0xffffffffu, lo, o);
                dd_merge(hi, lo, ohi, olo);
            }
            __syncthreads();  // every thread has read sc.d
            if (lane == 0) { sc.d[warp] = hi; sc.d2[warp] = lo; }
            __syncthreads();
            double h = sc.d[0], l = sc.d2[0];
            for (int w = 1; w < kChWarps; ++w) dd_merge(h, l, sc.d[w], sc.d2[w]);
            r = rms_factor(__dadd_rn(h, l), K, eps);
        }
    }
    float mx = 0.0f;
#pragma unroll
    for (int j = 0; j < kChVpt; ++j) {
        const int v = threadIdx.x + j * kChThreads;
        float f[8], g[8];
        unpack8_bf16(xr[j], f);
        if (gs) {
            unpack8_bf16(v < nvec ? gs[v] : make_uint4(0u, 0u, 0u, 0u), g);
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = norm_elem(f[e], r, g[e]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(f[e]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) sc.f[warp] = mx;
    __syncthreads();
    float m = sc.f[0];
    for (int w = 1; w < kChWarps; ++w) m = fmaxf(m, sc.f[w]);
    const float s = __fdiv_rn(127.0f, fmaxf(m, kScaleFloor));
    int rs = 0;
#pragma unroll
    for (int j = 0; j < kChVpt; ++j) {
        const int v = threadIdx.x + j * kChThreads;
        if (v >= nvec) continue;
        float f[8], g[8];
        unpack8_bf16(xr[j], f);
        if (gs) {
            unpack8_bf16(gs[v], g);
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = norm_elem(f[e], r, g[e]);
        }
        uint32_t packed[2] = {0u, 0u};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            int c = __float2int_rn(__fmul_rn(f[e], s));  // round half to even
            c = min(max(c, -128), 127);
            rs += c;
            packed[e >> 2] |= (uint32_t)(c & 0xFF) << (8 * (e & 3));
        }
        reinterpret_cast<uint2*>(q)[v] = make_uint2(packed[0], packed[1]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, o);
    if (lane == 0) sc.i[warp] = rs;
    __syncthreads();  // also publishes the codes
    int t = 0;
    for (int w = 0; w < kChWarps; ++w) t += sc.i[w];
    s_out = s;
    rs_out = t;
}

__global__ void __launch_bounds__(kChThreads, 1) chain_decode_kernel(const ChainArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ ChainQuantScratch sc;
    __shared__ int cta_ok;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    uint8_t* rings = smem + kChOffRings;
    ItemDesc* descs = reinterpret_cast<ItemDesc*>(smem + kChOffDescs);
    int8_t* qs = reinterpret_cast<int8_t*>(smem + kChOffCodes);
    uint4* gsm = reinterpret_cast<uint4*>(smem + kChOffGain);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* ring = rings + (size_t)warp * kDecRing;
    ItemDesc* my_descs = descs + warp * kDecSlots;
    const uint32_t bar0 = smem_addr(&bars[warp * kDecSlots]);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kChWarps * kDecSlots; ++i) mbar_init(smem_addr(&bars[i]), 1);
        mbar_init_fence();
        cta_ok = 1;
    }
    __syncthreads();

    const uint64_t policy = policy_evict_first();
    ChainWalker iw;
    iw.start(a.steps, a.nsteps, (int64_t)blockIdx.x * kChWarps + warp, (int64_t)gridDim.x * kChWarps);
    uint32_t issued = 0, done = 0;
    uint32_t ioff = 0, ring_free = kDecRing;
    auto refill = [&]() {
        while (issued - done < (uint32_t)kDecSlots && iw.valid()) {
            const int bytes = iw.bytes();
            const RingSpot spot = ring_spot(ioff, bytes);
            if (spot.used > ring_free) break;
            const uint32_t bar = bar0 + 8u * (issued % kDecSlots);
            if (lane == 0) {
                my_descs[issued % kDecSlots] =
                    ItemDesc{iw.p, (int)iw.r, iw.c, bytes, spot.at, spot.used, iw.rows(), iw.s};
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(bar, (uint32_t)bytes);
                bulk_g2s_stream(smem_addr(ring + spot.at), iw.src(), (uint32_t)bytes, bar, policy);
            }
            ring_free -= spot.used;
            ioff = spot.at + (uint32_t)bytes;
            ++issued;
            iw.advance();
        }
        __syncwarp();
    };
    refill();

    bool ok = true;
    int acc[4];
    for (int s = 0; s < a.nsteps; ++s) {
        // every warp of the CTA is done with step s - 1 (outputs written): count
        // in, load the step's gain (constant) while the others arrive, then wait
        __syncthreads();
        const ChainStep& cs = a.steps[s];
        const bool wait_bar = s > 0 && cta_ok;
        if (wait_bar && threadIdx.x == 0) {
            __threadfence();
            atomicAdd(a.bar, 1u);
        }
        if (cs.gain) {
            const uint4* gv = reinterpret_cast<const uint4*>(cs.gain);
            for (int v = threadIdx.x; v < (cs.K >> 3); v += kChThreads) gsm[v] = __ldg(gv + v);
        }
        if (wait_bar && threadIdx.x == 0) {
            const unsigned int target = (unsigned int)s * gridDim.x;
            const unsigned long long t0 = globaltimer_ns();
            for (uint32_t n = 0; ld_acquire_u32(a.bar) < target; ++n) {
                if ((n & 255u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) {
                    atomicOr(&g_status, kStatusTimeout);
                    cta_ok = 0;
                    break;
                }
            }
        }
        __syncthreads();
        if (!cta_ok) { ok = false; break; }
        // the step's input row, quantised by this CTA into shared memory
        float s_x;
        int rsum;
        chain_quantize(cs.x, cs.gain ? gsm : nullptr, cs.eps, cs.K, qs, sc, s_x, rsum);
        const RecipDiv sx = recip_div_init(s_x);
        const int K = cs.K;
        int cur_p = -1;
        EpiConsts ec{};
        // this warp's items of step s
        while (done < issued) {
            const ItemDesc d = my_descs[done % kDecSlots];
            if (d.pad != s) break;
            if (d.p != cur_p) {
                cur_p = d.p;
                const ChainProblem& pr = cs.p[cur_p];
                ec.y = pr.y;
                ec.residual = pr.residual;
                ec.N = pr.N;
                ec.R = pr.R;
                ec.beta = pr.beta;
                ec.beta2 = pr.beta2;
                ec.epi = pr.epi;
            }
            if (d.c == 0) {
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i] = 0;
            }
            const bool got = mbar_wait(bar0 + 8u * (done % kDecSlots), (done / kDecSlots) & 1u);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            const uint8_t* wbase = ring + d.at;
            const int8_t* qrow = qs + d.c * kDecChunk;
            if (d.rows == 2) {
                const int h = lane >> 4, hl = lane & 15;
                const uint4* wp = reinterpret_cast<const uint4*>(wbase + h * K);
                const int nvec = K >> 4;
#pragma unroll 2
                for (int v = hl; v < nvec; v += 16)
                    dot16(wp[v], reinterpret_cast<const uint4*>(qrow)[v], acc);
            } else {
                const uint4* wp = reinterpret_cast<const uint4*>(wbase);
                const int nvec = d.bytes >> 4;
#pragma unroll 2
                for (int v = lane; v < nvec; v += 32)
                    dot16(wp[v], reinterpret_cast<const uint4*>(qrow)[v], acc);
            }
            __syncwarp();
            ring_free += d.used;
            ++done;
            refill();
            if ((d.c + 1) * kDecChunk >= K || d.rows == 2) {  // the item ends its row(s)
                finish_acc(acc);
                const bool gu = ec.epi == kEpiGateUp;
                if (d.rows == 2) {
                    const int i = (lane >> 2) & 3;
                    const int64_t o = (int64_t)i * ec.R + d.r + (lane >> 4);
                    const int tot = half_reduce4(acc, lane);
                    if (gu) {
                        const int up = __shfl_down_sync(0xffffffffu, tot, 8);
                        if ((lane & 3) == 0 && i < 2)
                            store_gate_up(ec, o, (tot >> (2 * i)) - rsum, (up >> (2 * i + 4)) - rsum, sx);
                    } else if ((lane & 3) == 0) {
                        store_output(ec, o, (tot >> (2 * i)) - rsum, sx);
                    }
                } else {
                    const int i = lane >> 3;
                    const int64_t o = (int64_t)i * ec.R + d.r;
                    const int tot = warp_reduce4(acc, lane);
                    if (gu) {
                        const int up = __shfl_down_sync(0xffffffffu, tot, 16);
                        if ((lane & 7) == 0 && i < 2)
                            store_gate_up(ec, o, (tot >> (2 * i)) - rsum, (up >> (2 * i + 4)) - rsum, sx);
                    } else if ((lane & 7) == 0) {
                        store_output(ec, o, (tot >> (2 * i)) - rsum, sx);
                    }
                }
            }
        }
        // a failed wait ends the launch for the whole CTA at the next step
        // boundary, where every warp checks cta_ok after the same barrier
        if (!ok) cta_ok = 0;
    }
    if (!ok && lane == 0) {
        // drain the copies still in flight into this warp's ring before exiting
        for (uint32_t j = done; j < issued; ++j)
            mbar_wait(bar0 + 8u * (j % kDecSlots), (j / kDecSlots) & 1u);
    }
}

}  // namespace bl
