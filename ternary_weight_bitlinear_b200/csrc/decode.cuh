// decode.cuh -- memory-bound BitLinear GEMV for 1..4 tokens (decode), over a
// batch of independent BitLinear problems in one launch.
//
// Computes acc[m,n] = sum_k q[m,k] t[n,k] straight from the 2-bit packed
// weights ("Transformers 实战 BitNet 1.58 位量化" walkthrough, section
// "推理侧 BitLinear": unpack_weights + F.linear), then the rescale of
// post_quant_process, y = RN32(RN32(acc * beta) / s_x[m]).
//
// Design (B200):
//  * One launch streams the packed weights of every problem in the batch
//    exactly once.  The batch's packed rows are laid end to end as one byte
//    range; every warp of the grid owns an equal share of those bytes (whole
//    rows), so the load is balanced across all 148 SMs whatever the mix of
//    shapes.
//  * Each warp runs its own pipeline of bulk copies (TMA engine, no multicast,
//    L2 evict-first) of row chunks into shared memory, kDecSlots deep,
//    signalled by mbarriers.  The first copies are issued before the kernel
//    waits on the kernel before it (programmatic dependent launch), so weight
//    traffic overlaps the activation quantisation that precedes it.
//  * Unpacking never materialises ternary values: bit pair i of a packed byte
//    is selected in place with the mask 3 << 2i, so each 32-bit word gives
//    u8 operands code_i << 2i (code = t+1) for dp4a against four int8 codes.
//    Only bit pairs 0-2 are masked: the whole byte is sum_i 4^i code_i, so
//    dp4a of the unmasked word accumulates sum_i 4^i S_i and 4^3 S_3 is that
//    total minus the three masked sums (exact integer arithmetic).  The
//    factor 4^i is shifted out at the end and t = code - 1 is folded in with
//    the row sum of the codes: sum q*t = sum q*code - sum q.
//  * After the wait, each CTA stages the int8 codes, scales and row sums of the
//    problems its rows belong to in shared memory (they are reused by every
//    row of a problem); batches too large to stage read them from L2.
//  * Everything another kernel wrote (codes, scales, row sums, residual) is
//    read with ld.global.cg (L2, coherent), never through the non-coherent L1.
//  * A warp reduces its 4*MT partial sums with shuffles; lane 4m+i writes
//    output (m, i*N/4 + r) of its problem.
#pragma once

#include "common.cuh"

namespace bl {

constexpr int kDecThreads = 512;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecSlots = 8;          // copies in flight per warp (one mbarrier each)
constexpr int kDecChunk = 5120;       // largest single copy: 1-2 rows, or a piece of a long row
constexpr int kDecMaxRows = 2;        // rows per copy (one per half-warp)
constexpr int kDecRing = 10240;       // bytes of each warp's ring of copies
constexpr int kDecMaxTokens = 4;
constexpr int kDecQBudget = 48 * 1024;  // shared-memory bytes for staged codes
constexpr int kDecMaxStaged = 16;       // problems whose codes one CTA can stage
// Dynamic shared memory: one 8-byte mbarrier per in-flight copy (padded to 128
// bytes) | rings | staged codes | staged s_x | staged row sums | code offsets.
constexpr int kDecBarBytes = (8 * kDecWarps * kDecSlots + 127) / 128 * 128;
constexpr int kDecSlotBytes = kDecWarps * kDecRing;
static_assert(kDecChunk <= kDecRing && kDecRing % 128 == 0, "ring size");
constexpr int kDecMetaBytes = kDecMaxStaged * kDecMaxTokens * 8 + kDecMaxStaged * 4;
// Per-warp queue of the descriptors of copies in flight (issued, not consumed).
struct ItemDesc {
    int p;          // problem
    int r;          // first row
    int c;          // chunk of the row (rows longer than kDecChunk)
    int bytes;
    uint32_t at;    // ring offset
    uint32_t used;  // ring bytes it holds (skipped tail + bytes)
    int rows;       // whole rows in the copy (1 or 2; 1 for a chunk)
    int pad;
};
constexpr int kDecDescBytes = kDecWarps * kDecSlots * (int)sizeof(ItemDesc);
constexpr int kDecSmemBytes =
    kDecBarBytes + kDecSlotBytes + kDecQBudget + kDecMetaBytes + kDecDescBytes;
static_assert(8 * kDecWarps * kDecSlots <= kDecBarBytes, "barriers overlap the slots");
static_assert(kDecBarBytes % 128 == 0 && kDecChunk % 16 == 0, "copy alignment");
static_assert(kDecSmemBytes <= 227 * 1024, "shared memory budget");

// Output kinds.  kEpiGateUp: the packed matrix is a gate/up pair packed as
// [gate; up] (bit pairs 0, 1 gate rows r and R + r, bit pairs 2, 3 the up rows),
// and the output is z[m, i*R + r] = relu2_mul(bf16 gate, bf16 up) for i = 0, 1
// (N = 2R outputs), the up rows rescaled with their own scale beta2.
enum Epilogue { kEpiF32 = 0, kEpiBF16 = 1, kEpiI32 = 2, kEpiGateUp = 3 };

struct DecProblem {
    const int8_t* q;           // [M,K] codes
    const float* s_x;          // [M] (unused by kEpiI32)
    const int32_t* rowsum;     // [M]
    const uint8_t* P;          // [R,K]
    void* y;                   // [M,N]
    const uint16_t* residual;  // bf16 [M,N] or nullptr (kEpiBF16 only)
    int64_t R;                 // N/4
    int64_t N;
    int64_t byte0;             // sum of R*K over the problems before this one
    int K;
    float beta;
    float beta2;               // up projection's scale (kEpiGateUp)
    int epi;
    const float* beta_dev;     // when set: beta is read from device memory (after the grid wait)
};

template <int CAP>
struct DecBatch {
    int count;
    int64_t total;             // sum of R*K over the batch
    DecProblem p[CAP];
};

__host__ __device__ constexpr int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

// Last problem whose first byte is at or before `pos`.
template <int CAP>
__device__ __forceinline__ int problem_at(const DecBatch<CAP>& b, int64_t pos) {
    int lo_p = 0, hi_p = b.count - 1;
    while (lo_p < hi_p) {
        const int mid = (lo_p + hi_p + 1) >> 1;
        if (b.p[mid].byte0 <= pos) lo_p = mid; else hi_p = mid - 1;
    }
    return lo_p;
}

// A warp's walk over the (problem, row, chunk) items whose rows start in its
// byte range [lo, hi), with the current problem's constants kept in registers.
template <int CAP>
struct Walker {
    int p;      // current problem; b.count once the walk is over
    int r;      // row in p
    int r_end;  // first row of p outside the range
    int c;      // chunk of the row
    int K;
    int max_rows;  // whole rows per copy for this problem (1 when rows are chunked)
    const uint8_t* P;

    __device__ __forceinline__ void enter(const DecBatch<CAP>& b, int np, int64_t r0, int64_t hi) {
        p = np;
        c = 0;
        if (p >= b.count) return;
        const DecProblem& pr = b.p[p];
        K = pr.K;
        max_rows = K <= kDecChunk ? min(kDecMaxRows, kDecChunk / K) : 1;
        P = pr.P;
        const int64_t lim = hi - pr.byte0;  // rows with first byte < hi
        r_end = (int)(lim <= 0 ? 0 : min((lim + K - 1) / K, pr.R));
        r = (int)min(r0, pr.R);
    }
    __device__ __forceinline__ void settle(const DecBatch<CAP>& b, int64_t hi) {
        while (p < b.count && r >= r_end) {
            if (r_end < b.p[p].R) { p = b.count; return; }  // the range ends inside p
            enter(b, p + 1, 0, hi);
        }
    }
    __device__ __forceinline__ void start(const DecBatch<CAP>& b, int64_t lo, int64_t hi) {
        const int pp = problem_at(b, lo);
        const DecProblem& pr = b.p[pp];
        enter(b, pp, (lo - pr.byte0 + pr.K - 1) / pr.K, hi);
        settle(b, hi);
    }
    __device__ __forceinline__ bool valid(const DecBatch<CAP>& b) const { return p < b.count; }
    // whole rows in the next copy (short rows are copied two at a time)
    __device__ __forceinline__ int rows() const {
        return min(max_rows, r_end - r);
    }
    __device__ __forceinline__ int bytes() const {
        return K <= kDecChunk ? rows() * K : min(kDecChunk, K - c * kDecChunk);
    }
    __device__ __forceinline__ bool last_chunk() const {
        return K <= kDecChunk || (c + 1) * kDecChunk >= K;
    }
    __device__ __forceinline__ const uint8_t* src() const {
        return P + (int64_t)r * K + c * kDecChunk;
    }
    __device__ __forceinline__ void advance(const DecBatch<CAP>& b, int64_t hi) {
        if (!last_chunk()) { ++c; return; }
        r += rows();
        c = 0;
        settle(b, hi);
    }
};

// Placement of the next copy in a warp's byte ring: at `off`, or at the
// ring's start when it would run past the end; the skipped tail (possibly 0
// bytes) counts as used until the copy is consumed.
struct RingSpot {
    uint32_t at;    // offset of the copy
    uint32_t used;  // skipped tail + copy bytes
};
__device__ __forceinline__ RingSpot ring_spot(uint32_t off, int bytes) {
    const bool wrap = off + (uint32_t)bytes > (uint32_t)kDecRing;
    return {wrap ? 0u : off, (wrap ? (uint32_t)kDecRing - off : 0u) + (uint32_t)bytes};
}

// acc[i] += sum over the 16 bytes of (bit pair i of w, left in place) * q for
// i < 3; acc[3] += sum of (whole byte) * q.  finish_acc() turns acc[3] into
// the bit-pair-3 sum once the row is complete.
__device__ __forceinline__ void dot16(const uint4 w4, const uint4 q4, int (&acc)[4]) {
    const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
    const uint32_t q[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        acc[0] = dp4a_us(w[j] & 0x03030303u, q[j], acc[0]);
        acc[1] = dp4a_us(w[j] & 0x0C0C0C0Cu, q[j], acc[1]);
        acc[2] = dp4a_us(w[j] & 0x30303030u, q[j], acc[2]);
        acc[3] = dp4a_us(w[j], q[j], acc[3]);
    }
}

// whole-byte sum minus the bit-pair-0..2 sums = 4^3 * (bit-pair-3 sum).  Every
// partial stays below 2^31 in magnitude: a byte is at most 0xAA (codes <= 2),
// 170 * 128 * 65536 < 2^31.
__device__ __forceinline__ void finish_acc(int (&acc)[4]) {
    acc[3] -= acc[0] + acc[1] + acc[2];
}

// The output constants of the problem being consumed, kept in registers.
struct EpiConsts {
    void* y;
    const uint16_t* residual;
    int64_t N;
    int64_t R;
    float beta;
    float beta2;
    int epi;
    __device__ __forceinline__ void load(const DecProblem& pr) {
        y = pr.y;
        residual = pr.residual;
        N = pr.N;
        R = pr.R;
        beta = pr.beta_dev ? __ldcg(pr.beta_dev) : pr.beta;
        beta2 = pr.beta2;
        epi = pr.epi;
    }
};

__device__ __forceinline__ void store_output(const EpiConsts& e, int64_t idx, int acc,
                                             const RecipDiv& s_x) {
    if (e.epi == kEpiI32) {
        static_cast<int32_t*>(e.y)[idx] = acc;
        return;
    }
    const float y = recip_div(__fmul_rn(__int2float_rn(acc), e.beta), s_x);
    if (e.epi == kEpiF32) {
        static_cast<float*>(e.y)[idx] = y;
    } else {
        uint16_t b = float_to_bf16_bits(y);
        if (e.residual)
            b = float_to_bf16_bits(
                __fadd_rn(bf16_bits_to_float(__ldcg(e.residual + idx)), bf16_bits_to_float(b)));
        static_cast<uint16_t*>(e.y)[idx] = b;
    }
}

// z = relu2_mul(bf16(rescale(acc_gate)), bf16(rescale(acc_up))) of a gate/up pair.
__device__ __forceinline__ void store_gate_up(const EpiConsts& e, int64_t idx, int acc_g, int acc_u,
                                              const RecipDiv& s_x) {
    const uint16_t a = float_to_bf16_bits(recip_div(__fmul_rn(__int2float_rn(acc_g), e.beta), s_x));
    const uint16_t b = float_to_bf16_bits(recip_div(__fmul_rn(__int2float_rn(acc_u), e.beta2), s_x));
    static_cast<uint16_t*>(e.y)[idx] = relu2_mul_one(a, b);
}

// Sum 4 per-lane partials over the warp (reduce-scatter: 6 shuffles).  On
// return lane 8*i holds the total of a[i] (lanes 0, 8, 16, 24).
__device__ __forceinline__ int warp_reduce4(const int (&a)[4], int lane) {
    const bool hi16 = lane & 16, hi8 = lane & 8;
    int k0 = hi16 ? a[2] : a[0], k1 = hi16 ? a[3] : a[1];
    const int s0 = hi16 ? a[0] : a[2], s1 = hi16 ? a[1] : a[3];
    k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
    k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
    int k = hi8 ? k1 : k0;
    k += __shfl_xor_sync(0xffffffffu, hi8 ? k0 : k1, 8);
    k += __shfl_xor_sync(0xffffffffu, k, 4);
    k += __shfl_xor_sync(0xffffffffu, k, 2);
    k += __shfl_xor_sync(0xffffffffu, k, 1);
    return k;
}

// The same within each half-warp: on return lane 16h + 4i holds the total of
// a[i] over lanes 16h .. 16h+15 (5 shuffles for both halves at once).
__device__ __forceinline__ int half_reduce4(const int (&a)[4], int lane) {
    const bool hi8 = lane & 8, hi4 = lane & 4;
    int k0 = hi8 ? a[2] : a[0], k1 = hi8 ? a[3] : a[1];
    const int s0 = hi8 ? a[0] : a[2], s1 = hi8 ? a[1] : a[3];
    k0 += __shfl_xor_sync(0xffffffffu, s0, 8);
    k1 += __shfl_xor_sync(0xffffffffu, s1, 8);
    int k = hi4 ? k1 : k0;
    k += __shfl_xor_sync(0xffffffffu, hi4 ? k0 : k1, 4);
    k += __shfl_xor_sync(0xffffffffu, k, 2);
    k += __shfl_xor_sync(0xffffffffu, k, 1);
    return k;
}

template <int MT, int CAP>
__global__ void __launch_bounds__(kDecThreads, 1) decode_batch_kernel(
    const __grid_constant__ DecBatch<CAP> b) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    uint8_t* rings = smem + kDecBarBytes;
    int8_t* qs = reinterpret_cast<int8_t*>(smem + kDecBarBytes + kDecSlotBytes);
    float* sxs = reinterpret_cast<float*>(smem + kDecBarBytes + kDecSlotBytes + kDecQBudget);
    int* rss = reinterpret_cast<int*>(sxs + kDecMaxStaged * kDecMaxTokens);
    int* qoff = rss + kDecMaxStaged * kDecMaxTokens;
    ItemDesc* descs = reinterpret_cast<ItemDesc*>(
        smem + kDecBarBytes + kDecSlotBytes + kDecQBudget + kDecMetaBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* ring = rings + (size_t)warp * kDecRing;
    ItemDesc* my_descs = descs + warp * kDecSlots;
    const uint32_t bar0 = smem_addr(&bars[warp * kDecSlots]);  // this warp's barriers

    // this warp's (and this CTA's) share of the batch's packed bytes
    const int64_t W = (int64_t)gridDim.x * kDecWarps;
    const int64_t gw = (int64_t)blockIdx.x * kDecWarps + warp;
    const int64_t lo = gw * b.total / W, hi = (gw + 1) * b.total / W;
    const int64_t clo = (int64_t)blockIdx.x * kDecWarps * b.total / W;
    const int64_t chi = ((int64_t)blockIdx.x + 1) * kDecWarps * b.total / W;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kDecWarps * kDecSlots; ++i) mbar_init(smem_addr(&bars[i]), 1);
        mbar_init_fence();
    }
    __syncthreads();

    // The only walk over this warp's items is the issuing one; each issued
    // copy leaves its descriptor in the warp's queue for the consumer.
    const uint64_t policy = policy_evict_first();
    Walker<CAP> iw;
    iw.start(b, lo, hi);
    uint32_t issued = 0, done = 0;                      // items
    uint32_t ioff = 0, ring_free = kDecRing;            // ring bookkeeping (bytes)
    auto refill = [&]() {
        while (issued - done < (uint32_t)kDecSlots && iw.valid(b)) {
            const int bytes = iw.bytes();
            const RingSpot spot = ring_spot(ioff, bytes);
            if (spot.used > ring_free) break;
            const uint32_t bar = bar0 + 8u * (issued % kDecSlots);
            if (lane == 0) {
                my_descs[issued % kDecSlots] =
                    ItemDesc{iw.p, iw.r, iw.c, bytes, spot.at, spot.used, iw.rows(), 0};
                fence_proxy_async_smem();  // this warp's earlier reads of the ring come first
                mbar_arrive_expect_tx(bar, (uint32_t)bytes);
                bulk_g2s_stream(smem_addr(ring + spot.at), iw.src(), (uint32_t)bytes, bar, policy);
            }
            ring_free -= spot.used;
            ioff = spot.at + (uint32_t)bytes;
            ++issued;
            iw.advance(b, hi);
        }
        __syncwarp();  // descriptors written by lane 0 are visible to the warp
    };
    refill();

    // Everything above touches only the (constant) weights.  Dependents are
    // released only after this grid's own inputs are complete, so no kernel
    // runs more than one launch ahead of the data it reads.
    pdl_wait();
    pdl_launch_dependents();

    // Stage the codes, scales and row sums of the problems this CTA touches
    // (rows starting in [clo, chi)): they are reused by every row of a problem.
    Walker<CAP> cta;
    cta.start(b, clo, chi);
    const int pa = cta.p;
    const int pb = chi > 0 ? problem_at(b, chi - 1) : -1;
    int64_t need = 0;
    for (int p = pa; p <= pb; ++p) need += (int64_t)MT * b.p[p].K;
    const bool staged = cta.valid(b) && pb - pa + 1 <= kDecMaxStaged && need <= kDecQBudget;
    if (staged) {
        int off = 0;
        for (int p = pa; p <= pb; ++p) {
            const DecProblem& pr = b.p[p];
            const int nv = MT * pr.K / 16;
            const uint4* src = reinterpret_cast<const uint4*>(pr.q);
            uint4* dst = reinterpret_cast<uint4*>(qs + off);
            for (int v = threadIdx.x; v < nv; v += kDecThreads) dst[v] = __ldcg(src + v);
            if (threadIdx.x < MT) {
                sxs[(p - pa) * kDecMaxTokens + threadIdx.x] =
                    pr.epi == kEpiI32 ? 1.0f : __ldcg(pr.s_x + threadIdx.x);
                rss[(p - pa) * kDecMaxTokens + threadIdx.x] = __ldcg(pr.rowsum + threadIdx.x);
            }
            if (threadIdx.x == 0) qoff[p - pa] = off;
            off += MT * pr.K;
        }
    }
    __syncthreads();

    bool ok = true;
    int acc[MT][4];
    int cur_p = -1, K = 0;
    const int8_t* qbase = nullptr;
    RecipDiv sx[MT];
    int rsum[MT];
    EpiConsts ec{};
    int qoff_cur = 0;
    while (done < issued) {  // refill() keeps the queue non-empty until the walk ends
        const ItemDesc d = my_descs[done % kDecSlots];
        if (d.p != cur_p) {  // entering a problem: cache its activation and output data
            cur_p = d.p;
            const DecProblem& pr = b.p[cur_p];
            K = pr.K;
            ec.load(pr);
            if (staged) {
                qoff_cur = qoff[cur_p - pa];
                qbase = qs + qoff_cur;
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    sx[m] = recip_div_init(sxs[(cur_p - pa) * kDecMaxTokens + m]);
                    rsum[m] = rss[(cur_p - pa) * kDecMaxTokens + m];
                }
            } else {
                qbase = pr.q;
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    sx[m] = recip_div_init(pr.epi == kEpiI32 ? 1.0f : __ldcg(pr.s_x + m));
                    rsum[m] = __ldcg(pr.rowsum + m);
                }
            }
        }
        if (d.c == 0) {
#pragma unroll
            for (int m = 0; m < MT; ++m)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[m][i] = 0;
        }
        const bool got = mbar_wait(bar0 + 8u * (done % kDecSlots), (done / kDecSlots) & 1u);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        const uint8_t* wbase = ring + d.at;
        const int8_t* qrow = qbase + d.c * kDecChunk;
        // the staged codes addressed from the shared array itself, so that the
        // compiler emits shared-memory loads with 32-bit addresses
        const int8_t* qrow_s = qs + qoff_cur + d.c * kDecChunk;
        if (d.rows == 2) {
            // two rows: half-warp h takes row d.r + h
            const int h = lane >> 4, hl = lane & 15;
            const uint4* wp = reinterpret_cast<const uint4*>(wbase + h * K);
            const int nvec = K >> 4;
            if (staged) {
#pragma unroll 2
                for (int v = hl; v < nvec; v += 16) {
                    const uint4 w4 = wp[v];
#pragma unroll
                    for (int m = 0; m < MT; ++m)
                        dot16(w4, reinterpret_cast<const uint4*>(qrow_s + m * K)[v], acc[m]);
                }
            } else {
                for (int v = hl; v < nvec; v += 16) {
                    const uint4 w4 = wp[v];
#pragma unroll
                    for (int m = 0; m < MT; ++m)
                        dot16(w4, __ldcg(reinterpret_cast<const uint4*>(qrow + (int64_t)m * K) + v),
                              acc[m]);
                }
            }
        } else {
            const uint4* wp = reinterpret_cast<const uint4*>(wbase);
            const int nvec = d.bytes >> 4;
            if (staged) {
#pragma unroll 2
                for (int v = lane; v < nvec; v += 32) {
                    const uint4 w4 = wp[v];
#pragma unroll
                    for (int m = 0; m < MT; ++m)
                        dot16(w4, reinterpret_cast<const uint4*>(qrow_s + m * K)[v], acc[m]);
                }
            } else {
                for (int v = lane; v < nvec; v += 32) {
                    const uint4 w4 = wp[v];
#pragma unroll
                    for (int m = 0; m < MT; ++m)
                        dot16(w4, __ldcg(reinterpret_cast<const uint4*>(qrow + (int64_t)m * K) + v),
                              acc[m]);
                }
            }
        }
        __syncwarp();
        ring_free += d.used;
        ++done;
        refill();
        if ((d.c + 1) * kDecChunk >= K || d.rows == 2) {  // the item ends its row(s)
#pragma unroll
            for (int m = 0; m < MT; ++m) finish_acc(acc[m]);
            // a gate/up pair takes the up total (bit pair i + 2) from the lane
            // that holds it: 8 lanes up for half-warp rows, 16 for whole rows
            const bool gu = ec.epi == kEpiGateUp;  // the same in the whole warp
            if (d.rows == 2) {
                const int i = (lane >> 2) & 3;
                const int64_t o = (int64_t)i * ec.R + d.r + (lane >> 4);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const int tot = half_reduce4(acc[m], lane);
                    if (gu) {
                        const int up = __shfl_down_sync(0xffffffffu, tot, 8);
                        if ((lane & 3) == 0 && i < 2)
                            store_gate_up(ec, m * ec.N + o, (tot >> (2 * i)) - rsum[m],
                                          (up >> (2 * i + 4)) - rsum[m], sx[m]);
                    } else if ((lane & 3) == 0) {
                        store_output(ec, m * ec.N + o, (tot >> (2 * i)) - rsum[m], sx[m]);
                    }
                }
            } else {
                const int i = lane >> 3;
                const int64_t o = (int64_t)i * ec.R + d.r;
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const int tot = warp_reduce4(acc[m], lane);
                    if (gu) {
                        const int up = __shfl_down_sync(0xffffffffu, tot, 16);
                        if ((lane & 7) == 0 && i < 2)
                            store_gate_up(ec, m * ec.N + o, (tot >> (2 * i)) - rsum[m],
                                          (up >> (2 * i + 4)) - rsum[m], sx[m]);
                    } else if ((lane & 7) == 0) {
                        store_output(ec, m * ec.N + o, (tot >> (2 * i)) - rsum[m], sx[m]);
                    }
                }
            }
        }
    }

    if (!ok && lane == 0) {
        // Drain the copies still in flight into this warp's ring before exiting.
        for (uint32_t j = done; j < issued; ++j)
            mbar_wait(bar0 + 8u * (j % kDecSlots), (j / kDecSlots) & 1u);
    }
}

}  // namespace bl
