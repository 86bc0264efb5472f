// decode.cuh -- memory-bound BitLinear GEMV for 1..4 tokens (decode).
//
// Computes acc[m,n] = sum_k q[m,k] t[n,k] straight from the 2-bit packed
// weights ("Transformers 实战 BitNet 1.58 位量化" walkthrough, section
// "推理侧 BitLinear": unpack_weights + F.linear), then the rescale of
// post_quant_process, y = RN32(RN32(acc * beta) / s_x[m]).
//
// Design (B200):
//  * The packed matrix P[N/4, K] is streamed once.  Each CTA owns a contiguous
//    range of packed rows; each warp owns every 8th row of that range and runs
//    its own double-buffered pipeline of bulk copies (TMA engine, L2
//    evict-first) of row chunks into shared memory, signalled by mbarriers.
//    Copies for the first chunks are issued before the kernel waits on the
//    previous grid (programmatic dependent launch), so weight traffic overlaps
//    the previous kernel's tail and this kernel's own activation quantisation.
//  * With FUSED, every CTA quantises the (tiny) activation rows itself (RMSNorm
//    + absmax + int8, identical arithmetic to act_quant_kernel) into shared
//    memory: one launch per forward and no workspace.
//  * Unpacking never materialises ternary values: bit pair i of a packed byte
//    is selected in place with the mask 3 << 2i, so each 32-bit word gives four
//    u8 operands code_i << 2i (code = t+1) for dp4a against four int8 codes.
//    The shift is removed exactly at the end (>> 2i) and t = code - 1 is folded
//    in with the row sum of the codes: sum q*t = sum q*code - sum q.
//  * A warp reduces its 4*MT partial sums with shuffles; lane 4m+i writes
//    output (m, i*N/4 + r).
#pragma once

#include "common.cuh"
#include "quant.cuh"

namespace bl {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecSlots = 2;          // pipeline depth per warp
constexpr int kDecChunkMax = 4096;    // bytes per slot
constexpr int kDecMaxTokens = 4;
constexpr int kDecMaxQBytes = 65536;  // M*K limit of the shared-memory code buffer

enum Epilogue { kEpiF32 = 0, kEpiBF16 = 1, kEpiI32 = 2 };

struct DecodeArgs {
    const uint16_t* x;       // FUSED: bf16 [M,K]
    const uint16_t* gain;    // FUSED: bf16 [K] or nullptr
    float eps;
    const int8_t* q;         // !FUSED: int8 [M,K]
    const float* s_x;        // !FUSED: [M]
    const int32_t* rowsum;   // !FUSED: [M]
    const uint8_t* P;        // [R,K]
    float beta;
    int K;
    int chunk;               // bytes per slot, multiple of 16, <= kDecChunkMax
    int64_t R;               // N/4
    int64_t N;
    void* y;                 // [M,N]
    const uint16_t* residual;  // bf16 [M,N] or nullptr (kEpiBF16 only)
};

__host__ __device__ constexpr int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

// Dynamic shared memory: codes | barriers (128 B) | slots.
__host__ __device__ inline int64_t decode_q_bytes(int mt, int K) { return round_up((int64_t)mt * K, 128); }
__host__ __device__ inline int64_t decode_smem_bytes(int mt, int K, int chunk) {
    return decode_q_bytes(mt, K) + 128 + (int64_t)kDecWarps * kDecSlots * chunk;
}

// acc[i] += sum over the 16 bytes of (bit pair i of w, left in place) * q
__device__ __forceinline__ void dot16(const uint4 w4, const uint4 q4, int (&acc)[4]) {
    const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
    const uint32_t q[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        acc[0] = dp4a_us(w[j] & 0x03030303u, q[j], acc[0]);
        acc[1] = dp4a_us(w[j] & 0x0C0C0C0Cu, q[j], acc[1]);
        acc[2] = dp4a_us(w[j] & 0x30303030u, q[j], acc[2]);
        acc[3] = dp4a_us(w[j] & 0xC0C0C0C0u, q[j], acc[3]);
    }
}

template <int EPI>
__device__ __forceinline__ void store_output(const DecodeArgs& a, int64_t idx, int acc,
                                             float s_x) {
    if (EPI == kEpiI32) {
        static_cast<int32_t*>(a.y)[idx] = acc;
    } else {
        const float y = __fdiv_rn(__fmul_rn(__int2float_rn(acc), a.beta), s_x);
        if (EPI == kEpiF32) {
            static_cast<float*>(a.y)[idx] = y;
        } else {
            uint16_t b = float_to_bf16_bits(y);
            if (a.residual)
                b = float_to_bf16_bits(__fadd_rn(bf16_bits_to_float(a.residual[idx]),
                                                 bf16_bits_to_float(b)));
            static_cast<uint16_t*>(a.y)[idx] = b;
        }
    }
}

template <int MT, int EPI, bool FUSED>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(const DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ QuantScratch<kDecThreads> sc;
    __shared__ float s_sx[MT];
    __shared__ int s_rs[MT];

    const int K = a.K;
    const int chunk = a.chunk;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int8_t* q_s = reinterpret_cast<int8_t*>(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + decode_q_bytes(MT, K));
    uint8_t* slots = smem + decode_q_bytes(MT, K) + 128;

    const int64_t R = a.R;
    const int64_t r_begin = (R * blockIdx.x) / gridDim.x;
    const int64_t r_end = (R * (blockIdx.x + 1)) / gridDim.x;
    const int nck = (K + chunk - 1) / chunk;
    const int64_t cta_rows = r_end - r_begin;
    const int64_t my_rows = cta_rows > warp ? (cta_rows - warp + kDecWarps - 1) / kDecWarps : 0;
    const int64_t n_items = my_rows * nck;  // (row, chunk) pairs of this warp

    if (threadIdx.x == 0) {
        for (int i = 0; i < kDecWarps * kDecSlots; ++i) mbar_init(smem_addr(&bars[i]), 1);
        mbar_init_fence();
    }
    __syncthreads();

    const uint64_t policy = policy_evict_first();
    auto issue = [&](int64_t item) {  // lane 0 only
        const int64_t r = r_begin + warp + (int64_t)kDecWarps * (item / nck);
        const int k0 = (int)(item % nck) * chunk;
        const int bytes = min(chunk, K - k0);
        const int slot = (int)(item % kDecSlots);
        const uint32_t bar = smem_addr(&bars[warp * kDecSlots + slot]);
        mbar_arrive_expect_tx(bar, (uint32_t)bytes);
        bulk_g2s_stream(smem_addr(slots + (size_t)(warp * kDecSlots + slot) * chunk),
                        a.P + r * K + k0, (uint32_t)bytes, bar, policy);
    };
    if (lane == 0)
        for (int64_t it = 0; it < n_items && it < kDecSlots; ++it) issue(it);

    // Everything above touches only the (constant) weights.
    pdl_wait();
    pdl_launch_dependents();

    if (FUSED) {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            float s;
            int rs;
            quantize_row<kDecThreads>(a.x + (int64_t)m * K, a.gain, a.eps, K, q_s + m * K, sc, s,
                                      rs);
            if (threadIdx.x == 0) { s_sx[m] = s; s_rs[m] = rs; }
        }
    } else {
        const int nv = MT * K / 16;
        for (int v = threadIdx.x; v < nv; v += kDecThreads)
            reinterpret_cast<uint4*>(q_s)[v] = __ldg(reinterpret_cast<const uint4*>(a.q) + v);
        if (threadIdx.x < MT) {
            s_sx[threadIdx.x] = a.s_x ? a.s_x[threadIdx.x] : 1.0f;  // unused by kEpiI32
            s_rs[threadIdx.x] = a.rowsum[threadIdx.x];
        }
    }
    __syncthreads();

    int64_t it = 0;
    bool ok = true;
    for (int64_t row = warp; row < cta_rows; row += kDecWarps) {
        int acc[MT][4];
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[m][i] = 0;

        for (int c = 0; c < nck; ++c, ++it) {
            const int slot = (int)(it % kDecSlots);
            const uint32_t parity = (uint32_t)((it / kDecSlots) & 1);
            const bool got = mbar_wait(smem_addr(&bars[warp * kDecSlots + slot]), parity);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            const int k0 = c * chunk;
            const int nvec = min(chunk, K - k0) >> 4;
            const uint4* wp =
                reinterpret_cast<const uint4*>(slots + (size_t)(warp * kDecSlots + slot) * chunk);
            for (int v = lane; v < nvec; v += 32) {
                const uint4 w4 = wp[v];
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const uint4 q4 = *reinterpret_cast<const uint4*>(q_s + m * K + k0 + 16 * v);
                    dot16(w4, q4, acc[m]);
                }
            }
            __syncwarp();
            if (lane == 0 && it + kDecSlots < n_items) {
                fence_proxy_async_smem();  // our reads of this slot precede its refill
                issue(it + kDecSlots);
            }
        }
        if (!ok) break;

#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    acc[m][i] += __shfl_xor_sync(0xffffffffu, acc[m][i], o);

        const int64_t r = r_begin + row;
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (lane == 4 * m + i) {
                    const int exact = (acc[m][i] >> (2 * i)) - s_rs[m];
                    store_output<EPI>(a, (int64_t)m * a.N + (int64_t)i * R + r, exact, s_sx[m]);
                }
    }

    if (!ok && lane == 0) {
        // Drain copies still in flight into this warp's slots before exiting.
        for (int64_t j = it; j < n_items && j < it + kDecSlots; ++j)
            mbar_wait(smem_addr(&bars[warp * kDecSlots + (int)(j % kDecSlots)]),
                      (uint32_t)((j / kDecSlots) & 1));
    }
}

}  // namespace bl
