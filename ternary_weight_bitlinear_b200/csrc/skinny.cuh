// skinny.cuh -- BitLinear for 5..64 tokens (batched decode): a weight-streaming
// tensor-core GEMV over a batch of independent problems.
//
// acc[m,n] = sum_k q[m,k] t[n,k] ("Transformers 实战 BitNet 1.58 位量化"
// walkthrough, "推理侧 BitLinear": unpack_weights + F.linear) with the roles of
// the prefill GEMM swapped: the 2-bit weights are the wide operand and the few
// tokens the narrow one, and the weight bytes stream from HBM exactly once.
//
// Design (B200):
//  * Work unit ("item"): 32 packed rows (= 128 output rows, the MMA's M) x 512
//    bytes of K of one problem (16 KB of packed weights; the part of the last
//    item past the row end is neither loaded nor multiplied).  The batch's
//    items are laid end to end (problem, row tile, K stage) and each
//    persistent CTA owns an equal contiguous share, so all SMs stream the same
//    number of bytes whatever the mix of shapes.
//  * The tensor core costs max(44, N/2) cycles per tcgen05.mma.kind::i8 of
//    K = 32 on this GPU whatever M (64 or 128) or the source of A (measured).
//    With the weights as A (M = 128 rows) and the tokens as B (N <= 64), one
//    instruction takes 1 KB of packed weights per 44 cycles, about the HBM
//    rate of one SM; the swapped shape (weights as B, N = 256) would take 2 KB
//    per 128 cycles.  So the weights are A, and the pipeline below exists to
//    keep that one issuing thread fed.
//  * Warp 0 loads, per item, the packed tile and the token tile (int8 codes of
//    all M tokens for those K bytes) with TMA (128-byte swizzled boxes, no
//    multicast) into a shared-memory ring 4 to 8 items deep.  The packed tiles
//    of the first ring's worth of items are requested before the kernel waits
//    on the previous grid (programmatic dependent launch): weights are
//    constant, so their stream overlaps the quantisation kernel before.
//  * Two teams of four expansion warps (one per TMEM lane quadrant) alternate
//    items: each thread reads its packed row, selects its bit pair
//    (code = t + 1) and writes the codes of its weight row straight into
//    tensor memory with tcgen05.st (a ring of three 128-column slots), so the
//    expanded weights never use shared-memory bandwidth.
//  * One thread issues tcgen05.mma.cta_group::1.kind::i8 with A (weights) from
//    TMEM and B (tokens, N = M rounded up to 16) from shared memory into one
//    of two TMEM accumulators, and releases the ring slots with
//    tcgen05.commit (one commit per item frees its ring stage and its TMEM
//    slot).
//  * Four epilogue warps (one per TMEM lane quadrant) up to 16 tokens, eight
//    (two per quadrant, each half of the tokens) beyond, take a finished row
//    tile: tcgen05.ld, minus the row sums, rescale (exact division through
//    the token's reciprocal), store.
//  * A row tile whose items straddle several CTAs is finished by whichever of
//    them gets there last: each leaves its int32 partial sums in the caller's
//    workspace and counts itself in on the tile's counter (an atomic
//    compare-and-swap that carries this launch's epoch, so no counter needs
//    clearing); the one that completes the count adds the others' sums and
//    writes the outputs.  No CTA waits for another, so the kernel needs no
//    co-residency of its CTAs.  Without a workspace the CTA shares are cut at
//    row-tile boundaries.
//  * Every mbarrier wait is bounded (status word + unwind).
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "decode.cuh"
#include "gemm_tc.cuh"

namespace bl {

constexpr int kSkMinTokens = 5;
constexpr int kSkMaxTokens = 64;
constexpr int kSkRows = 32;                          // packed rows per tile
constexpr int kSkBK = 128;                           // K bytes per TMA box / swizzle atom
constexpr int kSkKB = 4;                             // boxes per item
constexpr int kSkItemK = kSkKB * kSkBK;              // 512 K bytes per item
constexpr int kSkMaxStages = 8;                      // shared-memory ring depth (for npad 16)
constexpr int kSkPBox = kSkRows * kSkBK;             // 4 KB packed box
constexpr int kSkPBytes = kSkKB * kSkPBox;           // 16 KB packed per item
constexpr int kSkRingBytes = 192 * 1024;             // ring: (16 KB + 4 * npad * 128) per stage
constexpr int kSkASlots = 3;                         // TMEM ring of expanded items (128 columns each)
constexpr int kSkTeams = 2;                          // expansion teams (4 warps each)
constexpr int kSkMmaWarp = 1;
constexpr int kSkExpWarp0 = 2;
constexpr int kSkEpiWarp0 = kSkExpWarp0 + 4 * kSkTeams;
// epilogue warps: 4 (one per lane quadrant, all tokens) up to 16 tokens, 8
// (two per lane quadrant, each half the tokens) beyond; the register budget
// of the 4-warp form is 128 per thread, of the 8-warp form 96 (below).  On
// this GPU the 4-warp form is ~3 % faster at 8 and 16 tokens and ~12 %
// slower at 32, where the epilogue's share of an item grows.
__host__ __device__ constexpr int sk_threads(int ew) { return 32 * (kSkEpiWarp0 + ew); }
__host__ __device__ constexpr int sk_epi_warps(int npad) { return npad <= 16 ? 4 : 8; }
constexpr int kSkCap = 64;                           // problems per launch
constexpr int kSkMaxGrid = 160;                      // CTAs per launch (>= SM count)
// TMEM columns: A ring [0, 384); accumulators [384, 512): two buffers of 64
constexpr uint32_t kSkTmemCols = 512;
constexpr uint32_t kSkACols = 32 * kSkKB;            // 128 columns (512 K bytes) per slot
constexpr uint32_t kSkDCol0 = kSkACols * kSkASlots;
constexpr uint32_t kSkDBuf = 64;
constexpr int kSkNumBars = 2 * kSkMaxStages + kSkASlots + 2 * 2 + 1;
constexpr int kSkOffBar = kSkRingBytes;
// tmem address | last-arriver flag | per-problem token constants (s_x,
// RN(1/s_x), row sums) for the epilogue
constexpr int kSkOffTmem = kSkOffBar + 8 * kSkNumBars;
constexpr int kSkOffTok = kSkOffTmem + 16;
constexpr int kSkSmemBytes = kSkOffTok + 12 * kSkMaxTokens + 1024;
static_assert(kSkSmemBytes <= 227 * 1024, "shared memory budget");
static_assert(kSkPBytes % 1024 == 0, "swizzle atoms stay 1024-aligned");
static_assert(kSkMaxStages * (kSkPBytes + kSkKB * 16 * kSkBK) <= kSkRingBytes, "ring holds 8 stages at npad 16");
// the ring's "item done" barriers also free the TMEM slots: an expansion team
// waits on item g - kSkASlots, which needs a ring of more than kSkASlots stages
static_assert(kSkRingBytes / (kSkPBytes + kSkKB * kSkMaxTokens * kSkBK) > kSkASlots, "ring depth");
static_assert(kSkDCol0 + 2 * kSkDBuf <= kSkTmemCols && kSkMaxTokens <= (int)kSkDBuf, "TMEM budget");
// each of the four schedulers of an SM holds 16384 registers: with 18 warps one
// scheduler holds 5, so at most 96 registers a thread; with 14, 4 and 128
// (launch bounds below)
static_assert((sk_threads(8) / 32 + 3) / 4 * 32 * 96 <= 16384, "register budget, 8 epilogue warps");
static_assert((sk_threads(4) / 32 + 3) / 4 * 32 * 128 <= 16384, "register budget, 4 epilogue warps");

struct SkProblem {
    const float* s_x;          // [M]
    const int32_t* rowsum;     // [M]
    void* y;                   // [M,N]
    const uint16_t* residual;  // bf16 [M,N] or nullptr
    int64_t N;
    int64_t item0;             // first item of this problem in the batch
    int R;                     // N/4
    int K;
    int tiles;                 // ceil(R / 32)
    int kst;                   // items per row tile: ceil(K / 512)
    float beta;
    float beta2;               // up projection's scale (kEpiGateUp)
    int epi;
    const float* beta_dev;     // when set: beta is read from device memory
};

struct alignas(64) SkBatch {
    CUtensorMap tmap_p[kSkCap];  // packed weights [R,K] u8, box 128 x 32, 128-byte swizzle
    CUtensorMap tmap_q[kSkCap];  // codes [M,K] i8, box 128 x npad, 128-byte swizzle
    SkProblem p[kSkCap];
    int count;
    int M;
    int npad;                    // MMA N: M rounded up to 16
    int split;                   // CTA shares may cut row tiles (workspace given)
    int64_t total;               // items in the batch
    unsigned long long epoch;    // nonzero, distinct per launch
    unsigned long long* ctr;     // [gridDim.x] split-tile counters (split only)
    int32_t* part;               // [gridDim.x][2][128][npad] partial sums (split only)
};

__device__ __forceinline__ int sk_problem_at(const SkBatch& b, int64_t item) {
    int lo = 0, hi = b.count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (b.p[mid].item0 <= item) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// First item of CTA c's share (c == G gives the end of the batch).
__device__ __forceinline__ int64_t sk_share_start(const SkBatch& b, int64_t c, int64_t G) {
    int64_t i = c * b.total / G;
    if (!b.split && i < b.total) {  // cut at the start of the row tile holding i
        const SkProblem& pr = b.p[sk_problem_at(b, i)];
        i = pr.item0 + (i - pr.item0) / pr.kst * pr.kst;
    }
    return i;
}

// The CTA whose share holds `item` (split schedule: shares floor(c T / G)).
__device__ __forceinline__ int64_t sk_owner(const SkBatch& b, int64_t item, int64_t G) {
    int64_t c = item * G / b.total;
    while (c + 1 < G && sk_share_start(b, c + 1, G) <= item) ++c;
    while (c > 0 && sk_share_start(b, c, G) > item) --c;
    return c;
}

// Walk over items: (problem, row tile, K stage).  The current problem's sizes
// stay in registers: the batch lives in the kernel's parameter block, and
// indexing it with a runtime problem number on every item costs a
// constant-cache miss each time.
struct SkCursor {
    int p, tile, ks, kst, tiles, K;
    __device__ __forceinline__ void load(const SkBatch& b) {
        if (p < b.count) {
            kst = b.p[p].kst;
            tiles = b.p[p].tiles;
            K = b.p[p].K;
        }
    }
    __device__ __forceinline__ void start(const SkBatch& b, int64_t item) {
        p = sk_problem_at(b, item);
        load(b);
        const int64_t rel = item - b.p[p].item0;
        tile = (int)(rel / kst);
        ks = (int)(rel - (int64_t)tile * kst);
    }
    __device__ __forceinline__ void next(const SkBatch& b) {
        if (++ks == kst) {
            ks = 0;
            if (++tile == tiles) {
                tile = 0;
                ++p;
                load(b);
            }
        }
    }
    // K bytes of this item inside the row (1..512)
    __device__ __forceinline__ int valid_k() const { return min(kSkItemK, K - ks * kSkItemK); }
};

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0],"
        " {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16,"
        " %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
          "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
          "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]),
          "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
          "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 8 consecutive 32-bit TMEM columns of this thread's lane (no wait).
__device__ __forceinline__ void tmem_ld8_nowait(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7])
                 : "r"(taddr));
}

// 16 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0],"
        " {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
          "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
          "r"(r[14]), "r"(r[15])
        : "memory");
}

// A (weights) from TMEM, B (tokens) from shared memory, D in TMEM.
__device__ __forceinline__ void sk_mma(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// int32 accumulate, signed 8-bit A and B, both K-major, M = 128, N = npad.
__device__ __forceinline__ uint32_t sk_idesc(int npad) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(npad >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// Named barrier among the EW epilogue warps.
template <int EW>
__device__ __forceinline__ void sk_epi_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(32 * EW) : "memory");
}

// The same barrier, returning whether `pred` held in all of them (so that they
// always take the same exits and never leave one another waiting).
template <int EW>
__device__ __forceinline__ bool sk_epi_all(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred a, b;\n\t"
        "setp.ne.u32 a, %1, 0;\n\t"
        "bar.red.and.pred b, 1, %2, a;\n\t"
        "selp.u32 %0, 1, 0, b;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "n"(32 * EW)
        : "memory");
    return r != 0;
}

// Count one participant in on a split tile's counter; true for the one that
// completes the count of n.  The counter's high word holds the launch epoch,
// so a counter left by an earlier launch (or never written) reads as zero.
// A compare-and-swap loop: some participant's swap succeeds on every round.
__device__ __forceinline__ bool sk_arrive_last(unsigned long long* ctr, uint32_t ep, uint32_t n,
                                               bool& ok) {
    unsigned long long old = atomicAdd(ctr, 0ull);
    for (uint32_t it = 0; it < (1u << 20); ++it) {
        const unsigned long long base =
            (uint32_t)(old >> 32) == ep ? old : ((unsigned long long)ep << 32);
        const unsigned long long nv = base + 1ull;
        const unsigned long long seen = atomicCAS(ctr, old, nv);
        if (seen == old) return (uint32_t)nv == n;
        old = seen;
    }
    atomicOr(&g_status, kStatusTimeout);
    ok = false;
    return false;
}

// One rescaled output: RN32(RN32(acc * beta) / s_x) through the token's reciprocal.
__device__ __forceinline__ float sk_scale(int acc, float beta, const PairDiv& d) {
    if (d.fast) {
        bool ok;
        const float q = scale_fast(acc, beta, d, ok);
        if (ok) return q;
    }
    return scale_slow(acc, beta, d.s, d.y);
}

__device__ __forceinline__ void sk_store(const SkProblem& pr, int m, int64_t n, int acc, float s_x,
                                         float s_rcp) {
    const int64_t idx = (int64_t)m * pr.N + n;
    if (pr.epi == kEpiI32) {
        static_cast<int32_t*>(pr.y)[idx] = acc;
        return;
    }
    const bool fast = s_x >= 0x1p-40f && s_x <= 0x1p40f && pr.beta >= 0x1p-40f && pr.beta <= 0x1p40f;
    const float y = sk_scale(acc, pr.beta, PairDiv{s_x, s_rcp, -s_x, fast});
    if (pr.epi == kEpiF32) {
        static_cast<float*>(pr.y)[idx] = y;
    } else {
        uint16_t bv = float_to_bf16_bits(y);
        if (pr.residual)
            bv = float_to_bf16_bits(
                __fadd_rn(bf16_bits_to_float(__ldcg(pr.residual + idx)), bf16_bits_to_float(bv)));
        static_cast<uint16_t*>(pr.y)[idx] = bv;
    }
}

template <int EW>
__global__ void __launch_bounds__(sk_threads(EW), 1) skinny_tc_kernel(const __grid_constant__ SkBatch b) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* sm = smem_raw + (base - raw);
    const uint32_t bars = base + kSkOffBar;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    // empty_bar(s): the MMAs of the item in ring stage s are done, which frees
    // the stage and the item's TMEM slot (one commit per item)
    auto empty_bar = [&](int s) { return bars + 8u * (kSkMaxStages + s); };
    auto afull_bar = [&](int a) { return bars + 8u * (2 * kSkMaxStages + a); };
    auto dfull_bar = [&](int d) { return bars + 8u * (2 * kSkMaxStages + kSkASlots + d); };
    auto dempty_bar = [&](int d) { return bars + 8u * (2 * kSkMaxStages + kSkASlots + 2 + d); };
    const uint32_t mma_done_bar = bars + 8u * (2 * kSkMaxStages + kSkASlots + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kSkOffTmem);
    volatile uint32_t* last_flag = reinterpret_cast<volatile uint32_t*>(sm + kSkOffTmem + 4);
    // ring stage: 4 packed boxes (4 KB each) | 4 token boxes (npad x 128 each)
    const uint32_t qbox = (uint32_t)(b.npad * kSkBK);
    const uint32_t stage_bytes = (uint32_t)kSkPBytes + kSkKB * qbox;
    const int nstages = min(kSkMaxStages, (int)(kSkRingBytes / stage_bytes));
    auto stage_p = [&](int s) { return base + (uint32_t)s * stage_bytes; };
    auto stage_q = [&](int s) { return base + (uint32_t)s * stage_bytes + (uint32_t)kSkPBytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kSkMaxStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < kSkASlots; ++a) mbar_init(afull_bar(a), 4);
        for (int d = 0; d < 2; ++d) {
            mbar_init(dfull_bar(d), 1);
            mbar_init(dempty_bar(d), EW);
        }
        mbar_init(mma_done_bar, 1);
        mbar_init_fence();
    }
    if (warp == kSkMmaWarp) tmem_alloc(smem_addr(tmem_slot), kSkTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int64_t G = gridDim.x, c = blockIdx.x;
    const int64_t i0 = sk_share_start(b, c, G), i1 = sk_share_start(b, c + 1, G);
    const uint32_t n_items = (uint32_t)(i1 - i0);
    bool ok = true;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            // the first ring's worth of packed tiles before the wait on the
            // previous grid (weights are constant), their token tiles after it
            const uint32_t pre = min(n_items, (uint32_t)nstages);
            SkCursor cur;
            if (n_items) cur.start(b, i0);
            for (uint32_t g = 0; g < pre; ++g) {
                const int nkb = (cur.valid_k() + kSkBK - 1) / kSkBK;
                mbar_arrive_expect_tx(full_bar((int)g), (uint32_t)nkb * ((uint32_t)kSkPBox + qbox));
                for (int kb = 0; kb < nkb; ++kb)
                    tma_load_2d(stage_p((int)g) + kb * kSkPBox, &b.tmap_p[cur.p],
                                cur.ks * kSkItemK + kb * kSkBK, cur.tile * kSkRows, full_bar((int)g));
                cur.next(b);
            }
            pdl_wait();
            pdl_launch_dependents();
            if (n_items) cur.start(b, i0);
            for (uint32_t g = 0; g < pre; ++g) {
                const int nkb = (cur.valid_k() + kSkBK - 1) / kSkBK;
                for (int kb = 0; kb < nkb; ++kb)
                    tma_load_2d(stage_q((int)g) + kb * qbox, &b.tmap_q[cur.p],
                                cur.ks * kSkItemK + kb * kSkBK, 0, full_bar((int)g));
                cur.next(b);
            }
            uint32_t g = pre, inflight_from = 0;
            for (; g < n_items && ok; ++g) {
                const int s = (int)(g % (uint32_t)nstages);
                if (!mbar_wait(empty_bar(s), ((g / nstages) & 1u) ^ 1u)) { ok = false; break; }
                inflight_from = g - nstages + 1;
                const int nkb = (cur.valid_k() + kSkBK - 1) / kSkBK;
                mbar_arrive_expect_tx(full_bar(s), (uint32_t)nkb * ((uint32_t)kSkPBox + qbox));
                for (int kb = 0; kb < nkb; ++kb) {
                    const int x = cur.ks * kSkItemK + kb * kSkBK;
                    tma_load_2d(stage_p(s) + kb * kSkPBox, &b.tmap_p[cur.p], x, cur.tile * kSkRows,
                                full_bar(s));
                    tma_load_2d(stage_q(s) + kb * qbox, &b.tmap_q[cur.p], x, 0, full_bar(s));
                }
                cur.next(b);
            }
            if (!ok)  // let the copies still in flight land before the CTA exits
                for (uint32_t j = inflight_from; j < g; ++j)
                    mbar_wait(full_bar((int)(j % (uint32_t)nstages)), (j / nstages) & 1u);
        } else {
            pdl_wait();
            pdl_launch_dependents();
        }
    } else if (warp == kSkMmaWarp) {
        pdl_wait();
        pdl_launch_dependents();
        // ---------------- MMA issuer ----------------
        // Kept small on purpose: ring positions and phases are counters, and
        // the MMAs of an item are one rolled loop, so that this thread's code
        // stays in the instruction cache next to the other roles' code.
        if (lane == 0) {
            SkCursor cur;
            if (n_items) cur.start(b, i0);
            const uint32_t idesc = sk_idesc(b.npad);
            const uint32_t qstep = qbox >> 4;  // descriptor address units between token boxes
            int s = 0, a = 0, d = 0;
            uint32_t sph = 0, aph = 0, dph = 0;
            bool first = true;
            for (uint32_t g = 0; g < n_items && ok; ++g) {
                if (first && !mbar_wait(dempty_bar(d), dph ^ 1u)) { ok = false; break; }
                if (!mbar_wait(afull_bar(a), aph) || !mbar_wait(full_bar(s), sph)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t dcol = tmem + kSkDCol0 + (uint32_t)d * kSkDBuf;
                uint32_t acol = tmem + kSkACols * (uint32_t)a;  // 32 K bytes = 8 TMEM columns of A
                const uint64_t bd = smem_desc_sw128(stage_q(s));
                const int nmma = (cur.valid_k() + 31) >> 5;
                uint32_t acc = first ? 0u : 1u;
#pragma unroll 1
                for (int t = 0; t < nmma; ++t) {
                    sk_mma(dcol, acol, bd + 2u * (uint32_t)(t & 3) + qstep * (uint32_t)(t >> 2), idesc, acc);
                    acc = 1u;
                    acol += 8u;
                }
                tc_commit(empty_bar(s));
                const bool last = g + 1 == n_items || cur.ks + 1 == cur.kst;
                first = last;
                if (last) {
                    tc_commit(dfull_bar(d));
                    if ((d ^= 1) == 0) dph ^= 1u;
                }
                if (++s == nstages) { s = 0; sph ^= 1u; }
                if (++a == kSkASlots) { a = 0; aph ^= 1u; }
                cur.next(b);
            }
            tc_commit(mma_done_bar);
            mbar_wait(mma_done_bar, 0);
        }
    } else if (warp < kSkEpiWarp0) {
        pdl_wait();
        pdl_launch_dependents();
        // ---------------- expansion teams ----------------
        const int team = (warp - kSkExpWarp0) >> 2, qd = warp & 3;
        const int bit = lane >> 3, j = lane & 7;  // this lane: bit pair, packed row 8*qd + j
        const int prow = 8 * qd + j;
        const uint32_t tlane = (uint32_t)(32 * qd) << 16;
        SkCursor cur;
        if (n_items > (uint32_t)team) {
            cur.start(b, i0);
            if (team) cur.next(b);
        }
        for (uint32_t g = (uint32_t)team; g < n_items && ok; g += kSkTeams) {
            const int s = (int)(g % (uint32_t)nstages), a = (int)(g % kSkASlots);
            // TMEM slot a is free once item g - kSkASlots (which used it) is done
            const uint32_t gp = g - kSkASlots;
            const bool got = mbar_wait(full_bar(s), (g / nstages) & 1u) &&
                             (g < (uint32_t)kSkASlots ||
                              mbar_wait(empty_bar((int)(gp % (uint32_t)nstages)), (gp / nstages) & 1u));
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            const int nkb = (cur.valid_k() + kSkBK - 1) / kSkBK;
            for (int kb = 0; kb < nkb; ++kb) {
                const uint8_t* pk = sm + (size_t)s * stage_bytes + kb * kSkPBox + prow * kSkBK;
                uint32_t w[32];
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {  // 128-byte swizzle: chunk ch sits at ch ^ (row & 7)
                    const uint4 v = *reinterpret_cast<const uint4*>(pk + ((ch ^ j) << 4));
                    w[4 * ch + 0] = (v.x >> (2 * bit)) & 0x03030303u;
                    w[4 * ch + 1] = (v.y >> (2 * bit)) & 0x03030303u;
                    w[4 * ch + 2] = (v.z >> (2 * bit)) & 0x03030303u;
                    w[4 * ch + 3] = (v.w >> (2 * bit)) & 0x03030303u;
                }
                tmem_st32(tmem + tlane + kSkACols * (uint32_t)a + 32u * (uint32_t)kb, w);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(afull_bar(a));
            cur.next(b);
            cur.next(b);
        }
    } else {
        pdl_wait();
        pdl_launch_dependents();
        // ---------------- epilogue: one weight row, half of the tokens per thread ----------------
        const int ew = warp - kSkEpiWarp0;
        const int qd = warp & 3, half = EW == 8 ? ew >> 2 : 0;
        const int bit = lane >> 3, j = lane & 7;
        const int row128 = 32 * qd + lane;  // D row (TMEM lane)
        float* tok_s = reinterpret_cast<float*>(sm + kSkOffTok);
        float* tok_y = tok_s + kSkMaxTokens;
        int* tok_rs = reinterpret_cast<int*>(tok_y + kSkMaxTokens);
        const int et = threadIdx.x - 32 * kSkEpiWarp0;  // 0..32 EW - 1
        // this thread's token columns [c0, c1): all of them (4 warps, npad =
        // 16), or halves of npad in 16-column steps (8 warps)
        const int hc = EW == 8 ? ((b.npad / 2) + 15) & ~15 : b.npad;
        const int c0 = half * hc, c1 = min(b.npad, c0 + hc);
        const uint32_t ep32 = (uint32_t)b.epoch;
        int staged = -1;
        SkCursor cur;
        if (n_items) cur.start(b, i0);
        int64_t item = i0;
        uint32_t tl = 0;
        while (item < i1 && ok) {
            // the part of (cur.p, cur.tile) inside this CTA's share; the
            // problem's constants are copied to registers once per part
            SkProblem pr = b.p[cur.p];
            if (pr.beta_dev) pr.beta = __ldcg(pr.beta_dev);
            if (staged != cur.p) {  // this problem's token scales and row sums, once
                sk_epi_sync<EW>();
                if (et < b.M) {
                    const float sx = pr.epi == kEpiI32 ? 1.0f : __ldcg(pr.s_x + et);
                    tok_s[et] = sx;
                    tok_y[et] = __frcp_rn(sx);
                    tok_rs[et] = __ldcg(pr.rowsum + et);
                }
                sk_epi_sync<EW>();
                staged = cur.p;
            }
            const int64_t tile_first = pr.item0 + (int64_t)cur.tile * pr.kst;
            const int64_t tile_end = tile_first + pr.kst;
            const int64_t part_end = min(tile_end, i1);
            const bool split = item > tile_first || part_end < tile_end;
            const int d = (int)(tl & 1);
            const bool got = mbar_wait(dfull_bar(d), (tl >> 1) & 1u);
            if (!sk_epi_all<EW>(got)) { ok = false; break; }
            tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(32 * qd) << 16) + kSkDCol0 + (uint32_t)d * kSkDBuf;
            bool write = true;
            if (split) {
                // leave this CTA's partial sums, count in; the last one to
                // arrive adds the others' sums into its accumulator and writes
                const int64_t cf = sk_owner(b, tile_first, G), cl = sk_owner(b, tile_end - 1, G);
                const int role = item > tile_first ? 0 : 1;
                uint32_t v[32];
                if (c0 < c1) {
                    tmem_ld16_nowait(taddr + (uint32_t)c0, v);
                    if (c1 - c0 > 16) tmem_ld16_nowait(taddr + (uint32_t)(c0 + 16), v + 16);
                    tmem_ld_wait();
                }
                int32_t* mine = b.part + ((size_t)(2 * c + role) * 128 + row128) * b.npad;
#pragma unroll
                for (int k = 0; k < 32; k += 4)
                    if (c0 + k < c1)
                        *reinterpret_cast<uint4*>(mine + c0 + k) = make_uint4(v[k], v[k + 1], v[k + 2], v[k + 3]);
                __threadfence();
                sk_epi_sync<EW>();
                if (et == 0) {
                    bool aok = true;
                    *last_flag = sk_arrive_last(b.ctr + cf, ep32, (uint32_t)(cl - cf + 1), aok) ? 1u : 0u;
                    if (!aok) *last_flag = 2u;
                }
                sk_epi_sync<EW>();
                const uint32_t lf = *last_flag;
                if (lf == 2u) ok = false;
                write = lf == 1u;
                if (write) {
                    __threadfence();
                    auto other_part = [&](int64_t c2) {
                        return b.part + ((size_t)(2 * c2 + (c2 == cf ? 1 : 0)) * 128 + row128) * b.npad;
                    };
                    if constexpr (EW == 4) {
                        // the others' partial sums, two participants' loads in flight
                        // at a time (a participant's sums are one L2 round trip)
                        int64_t c2 = cf == c ? cf + 1 : cf;
                        while (c2 <= cl) {
                            int64_t c3 = c2 + 1;
                            if (c3 == c) ++c3;
                            const int32_t* o2 = other_part(c2);
                            const int32_t* o3 = other_part(c3 <= cl ? c3 : c2);
                            // four epilogue warps serve npad 16: 16 columns a thread
                            uint4 w2[4], w3[4];
#pragma unroll
                            for (int k = 0; k < 16; k += 4) {
                                if (c0 + k < c1) {
                                    w2[k / 4] = __ldcg(reinterpret_cast<const uint4*>(o2 + c0 + k));
                                    w3[k / 4] = c3 <= cl ? __ldcg(reinterpret_cast<const uint4*>(o3 + c0 + k))
                                                         : make_uint4(0u, 0u, 0u, 0u);
                                }
                            }
#pragma unroll
                            for (int k = 0; k < 16; k += 4) {
                                if (c0 + k < c1) {
                                    v[k] += w2[k / 4].x + w3[k / 4].x;
                                    v[k + 1] += w2[k / 4].y + w3[k / 4].y;
                                    v[k + 2] += w2[k / 4].z + w3[k / 4].z;
                                    v[k + 3] += w2[k / 4].w + w3[k / 4].w;
                                }
                            }
                            c2 = c3 + 1;
                            if (c2 == c) ++c2;
                        }
                    } else {
                        for (int64_t c2 = cf; c2 <= cl; ++c2) {
                            if (c2 == c) continue;
                            const int32_t* other = other_part(c2);
#pragma unroll
                            for (int k = 0; k < 32; k += 4) {
                                if (c0 + k < c1) {
                                    const uint4 w4 = __ldcg(reinterpret_cast<const uint4*>(other + c0 + k));
                                    v[k] += w4.x;
                                    v[k + 1] += w4.y;
                                    v[k + 2] += w4.z;
                                    v[k + 3] += w4.w;
                                }
                            }
                        }
                    }
                    // the tile's sums back into the accumulator, read below like any other
                    if (c0 < c1) {
                        tmem_st16(taddr + (uint32_t)c0, v);
                        if (c1 - c0 > 16) tmem_st16(taddr + (uint32_t)(c0 + 16), v + 16);
                        tmem_st_wait();
                    }
                }
            }
            const int r = cur.tile * kSkRows + 8 * qd + j;  // packed row
            if (write) {  // warp-uniform: the TMEM loads are warp-wide, the stores per lane
                // eight tokens at a time from TMEM, in a rolled loop (small code)
                const int64_t n = (int64_t)bit * pr.R + r;
                const int cend = min(c1, b.M);
#pragma unroll 1
                for (int cg = c0; cg < cend; cg += 8) {
                    uint32_t v8[8];
                    tmem_ld8_nowait(taddr + (uint32_t)cg, v8);
                    tmem_ld_wait();
                    if (pr.epi == kEpiGateUp) {
                        // every lane rescales its own row (gate rows: bit pairs 0, 1
                        // with the gate's scale; up rows: 2, 3 with the up's), then
                        // the up value moves 16 lanes down to its gate row
                        const float bl = bit < 2 ? pr.beta : pr.beta2;
                        const bool bok = bl >= 0x1p-40f && bl <= 0x1p40f;
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const float sx = tok_s[cg + k];
                            const bool fast = bok && sx >= 0x1p-40f && sx <= 0x1p40f;
                            const uint16_t mine = float_to_bf16_bits(
                                sk_scale((int)v8[k] - tok_rs[cg + k], bl, PairDiv{sx, tok_y[cg + k], -sx, fast}));
                            const uint32_t up = __shfl_down_sync(0xffffffffu, (uint32_t)mine, 16);
                            if (bit < 2 && r < pr.R && cg + k < cend)
                                static_cast<uint16_t*>(pr.y)[(int64_t)(cg + k) * pr.N + n] =
                                    relu2_mul_one(mine, up);
                        }
                    } else if (r < pr.R) {
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            if (cg + k < cend)
                                sk_store(pr, cg + k, n, (int)v8[k] - tok_rs[cg + k], tok_s[cg + k], tok_y[cg + k]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dempty_bar(d));  // the accumulator is free again
            // next part
            for (int64_t k = item; k < part_end; ++k) cur.next(b);
            item = part_end;
            ++tl;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kSkMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kSkTmemCols);
    }
}

}  // namespace bl
