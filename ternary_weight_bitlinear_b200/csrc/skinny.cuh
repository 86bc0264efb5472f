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
//    bytes of K of one problem; every item moves the same 16 KB of packed
//    weights (K past the row end reads as zeros).  Items this large keep the
//    per-item barrier round trips of the single issuing thread off the
//    critical path.  The batch's items are laid end to end (problem, row tile, K
//    stage) and each persistent CTA owns an equal contiguous share, so all SMs
//    stream the same number of bytes whatever the mix of shapes.
//  * Warp 0 loads, per item, the packed tile and the token tile (int8 codes of
//    all M tokens for those 512 K bytes) with TMA (four 128-byte-swizzled
//    boxes each, no multicast) into a shared-memory ring, 4 to 8 items deep
//    depending on M.
//  * Two teams of four expansion warps (one per TMEM lane quadrant) alternate
//    items: each thread reads its packed row, selects its bit pair
//    (code = t + 1) and writes the 512 codes of its weight row straight into
//    tensor memory with tcgen05.st -- the expanded weights never touch shared
//    memory, whose bandwidth is what limits a shared-memory operand here.
//  * One thread issues tcgen05.mma.cta_group::1.kind::i8 with A (weights,
//    M=128) from TMEM and B (tokens, N = M rounded up to 16) from shared
//    memory.  An item's 16 MMAs rotate over 2-4 independent accumulator
//    chains (double-buffered per row tile) that the epilogue sums.  MMAs this
//    narrow are bound by their issue rate (~65 cycles each on this GPU,
//    measured), not by the tensor pipe, which caps this kernel near 0.7 of
//    the HBM roofline.
//  * Four epilogue warps take a finished row tile: tcgen05.ld, minus the row
//    sums, rescale (exact division through the token's reciprocal), store.
//    A row tile whose items straddle two or more CTAs is finished by the CTA
//    holding its first items (it reaches them last): the others leave int32
//    partial sums in the caller's workspace and raise a flag carrying this
//    launch's epoch; the finisher polls those flags side by side, adds the
//    sums (16-byte loads of each contributor's block) and clears the flags.
//    Without a workspace the CTA shares are cut at row-tile boundaries.
//  * Every wait is bounded (status word + unwind).
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
constexpr int kSkRingBytes = 196 * 1024;             // ring: (16 KB + 4 * npad * 128) per stage
constexpr int kSkAStages = 2;                        // TMEM ring of expanded items (128 columns each)
constexpr int kSkTeams = 2;                          // expansion teams (4 warps each)
constexpr int kSkMmaWarp = 1;
constexpr int kSkExpWarp0 = 2;
constexpr int kSkEpiWarp0 = kSkExpWarp0 + 4 * kSkTeams;
constexpr int kSkThreads = 32 * (kSkEpiWarp0 + 4);
constexpr int kSkCap = 64;                           // problems per launch
constexpr int kSkMaxGrid = 160;                      // CTAs per launch (>= SM count)
// TMEM columns: A ring [0, 256); accumulators [256, 512): two buffers of 128
// columns, each holding 128/stride chains of `stride` = max(32, npad rounded
// up to 32) columns
constexpr uint32_t kSkTmemCols = 512;
constexpr uint32_t kSkDCol0 = 32 * kSkKB * kSkAStages;
constexpr uint32_t kSkDBuf = 128;
constexpr int kSkNumBars = 2 * kSkMaxStages + 2 * kSkAStages + 2 * 2 + 1;
constexpr int kSkOffBar = kSkRingBytes;
// per-problem token constants for the epilogue: s_x, RN(1/s_x), row sums
constexpr int kSkOffTok = kSkOffBar + 8 * kSkNumBars + 16;
constexpr int kSkSmemBytes = kSkOffTok + 12 * kSkMaxTokens + 1024;
static_assert(kSkSmemBytes <= 227 * 1024, "shared memory budget");
static_assert(kSkPBytes % 1024 == 0, "swizzle atoms stay 1024-aligned");
static_assert(kSkMaxStages * (kSkPBytes + kSkKB * 16 * kSkBK) <= kSkRingBytes, "ring holds 8 stages at npad 16");
static_assert(kSkDCol0 + 2 * kSkDBuf <= kSkTmemCols && 2 * kSkMaxTokens <= kSkDBuf, "TMEM budget");

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
    int epi;
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
    unsigned long long* flags;   // [gridDim.x] partial-sum flags (split only)
    int32_t* part;               // [gridDim.x][128][npad] partial sums (split only)
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

// Walk over items: (problem, row tile, K stage).  The current problem's sizes
// stay in registers: the batch lives in the kernel's parameter block, and
// indexing it with a runtime problem number on every item costs a
// constant-cache miss each time.
struct SkCursor {
    int p, tile, ks, kst, tiles;
    __device__ __forceinline__ void load(const SkBatch& b) {
        if (p < b.count) {
            kst = b.p[p].kst;
            tiles = b.p[p].tiles;
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

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Named barrier among the four epilogue warps, and the same barrier returning
// whether `pred` held in all of them (so that they always take the same exits
// and never leave one another waiting at the barrier).
__device__ __forceinline__ void sk_epi_sync() {
    asm volatile("bar.sync 1, 128;" ::: "memory");
}

__device__ __forceinline__ bool sk_epi_all(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred a, b;\n\t"
        "setp.ne.u32 a, %1, 0;\n\t"
        "bar.red.and.pred b, 1, 128, a;\n\t"
        "selp.u32 %0, 1, 0, b;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred)
        : "memory");
    return r != 0;
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

__global__ void __launch_bounds__(kSkThreads, 1) skinny_tc_kernel(const __grid_constant__ SkBatch b) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* sm = smem_raw + (base - raw);
    const uint32_t bars = base + kSkOffBar;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (kSkMaxStages + s); };
    auto afull_bar = [&](int a) { return bars + 8u * (2 * kSkMaxStages + a); };
    auto aempty_bar = [&](int a) { return bars + 8u * (2 * kSkMaxStages + kSkAStages + a); };
    auto dfull_bar = [&](int d) { return bars + 8u * (2 * kSkMaxStages + 2 * kSkAStages + d); };
    auto dempty_bar = [&](int d) { return bars + 8u * (2 * kSkMaxStages + 2 * kSkAStages + 2 + d); };
    const uint32_t mma_done_bar = bars + 8u * (2 * kSkMaxStages + 2 * kSkAStages + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kSkOffBar + 8 * kSkNumBars);
    // ring stage: 4 packed boxes (4 KB each) | 4 token boxes (npad x 128 each)
    const uint32_t qbox = (uint32_t)(b.npad * kSkBK);
    const uint32_t stage_bytes = (uint32_t)kSkPBytes + kSkKB * qbox;
    const int nstages = min(kSkMaxStages, (int)(kSkRingBytes / stage_bytes));
    const int dstride = b.npad <= 32 ? 32 : 64;  // accumulator chain width (columns)
    const int chains = (int)kSkDBuf / dstride;   // 4 or 2
    auto stage_p = [&](int s) { return base + (uint32_t)s * stage_bytes; };
    auto stage_q = [&](int s) { return base + (uint32_t)s * stage_bytes + (uint32_t)kSkPBytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kSkMaxStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < kSkAStages; ++a) {
            mbar_init(afull_bar(a), 4);
            mbar_init(aempty_bar(a), 1);
        }
        for (int d = 0; d < 2; ++d) {
            mbar_init(dfull_bar(d), 1);
            mbar_init(dempty_bar(d), 4);
        }
        mbar_init(mma_done_bar, 1);
        mbar_init_fence();
    }
    if (warp == kSkMmaWarp) tmem_alloc(smem_addr(tmem_slot), kSkTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    pdl_wait();
    pdl_launch_dependents();

    const int64_t G = gridDim.x, c = blockIdx.x;
    const int64_t i0 = sk_share_start(b, c, G), i1 = sk_share_start(b, c + 1, G);
    const uint32_t n_items = (uint32_t)(i1 - i0);
    bool ok = true;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            SkCursor cur;
            if (n_items) cur.start(b, i0);
            const uint32_t tx = stage_bytes;  // out-of-range parts of a box are zero-filled, still counted
            uint32_t g = 0, inflight_from = 0;
            for (; g < n_items && ok; ++g) {
                const int s = (int)(g % (uint32_t)nstages);
                if (!mbar_wait(empty_bar(s), ((g / nstages) & 1u) ^ 1u)) { ok = false; break; }
                inflight_from = g >= (uint32_t)nstages ? g - nstages + 1 : 0;
                mbar_arrive_expect_tx(full_bar(s), tx);
#pragma unroll
                for (int kb = 0; kb < kSkKB; ++kb) {
                    const int x = cur.ks * kSkItemK + kb * kSkBK;
                    tma_load_2d(stage_p(s) + kb * kSkPBox, &b.tmap_p[cur.p], x, cur.tile * kSkRows,
                                full_bar(s));
                    tma_load_2d(stage_q(s) + kb * qbox, &b.tmap_q[cur.p], x, 0, full_bar(s));
                }
                cur.next(b);
            }
            if (!ok)
                for (uint32_t j = inflight_from; j < g; ++j)
                    mbar_wait(full_bar((int)(j % (uint32_t)nstages)), (j / nstages) & 1u);
        }
    } else if (warp == kSkMmaWarp) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            SkCursor cur;
            if (n_items) cur.start(b, i0);
            const uint32_t idesc = sk_idesc(b.npad);
            uint32_t tl = 0;
            bool first = true;
            for (uint32_t g = 0; g < n_items && ok; ++g) {
                const int s = (int)(g % (uint32_t)nstages), a = (int)(g % kSkAStages), d = (int)(tl & 1);
                if (first && !mbar_wait(dempty_bar(d), ((tl >> 1) & 1u) ^ 1u)) { ok = false; break; }
                if (!mbar_wait(full_bar(s), (g / nstages) & 1u) ||
                    !mbar_wait(afull_bar(a), (g / kSkAStages) & 1u)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t dcol = tmem + kSkDCol0 + (uint32_t)d * kSkDBuf;
#pragma unroll
                for (int kb = 0; kb < kSkKB; ++kb) {
                    const uint64_t bd = smem_desc_sw128(stage_q(s) + kb * qbox);
#pragma unroll
                    for (int kk = 0; kk < kSkBK / 32; ++kk) {  // 32 K bytes = 8 TMEM columns of A
                        const int t = kb * (kSkBK / 32) + kk;  // MMA number in the item
                        const int ch = t & (chains - 1);
                        sk_mma(dcol + (uint32_t)(ch * dstride), tmem + (uint32_t)(32 * kSkKB * a + 8 * t),
                               bd + 2u * kk, idesc, (first && t < chains) ? 0u : 1u);
                    }
                }
                tc_commit(empty_bar(s));
                tc_commit(aempty_bar(a));
                const bool last = g + 1 == n_items || cur.ks + 1 == cur.kst;
                first = last;
                if (last) {
                    tc_commit(dfull_bar(d));
                    ++tl;
                }
                cur.next(b);
            }
            tc_commit(mma_done_bar);
            mbar_wait(mma_done_bar, 0);
        }
    } else if (warp < kSkEpiWarp0) {
        // ---------------- expansion teams ----------------
        const int team = (warp - kSkExpWarp0) >> 2, qd = warp & 3;
        const int bit = lane >> 3, j = lane & 7;  // this lane: bit pair, packed row 8*qd + j
        const int prow = 8 * qd + j;
        const uint32_t tlane = (uint32_t)(32 * qd) << 16;
        for (uint32_t g = (uint32_t)team; g < n_items && ok; g += kSkTeams) {
            const int s = (int)(g % (uint32_t)nstages), a = (int)(g % kSkAStages);
            const bool got = mbar_wait(full_bar(s), (g / nstages) & 1u) &&
                             mbar_wait(aempty_bar(a), ((g / kSkAStages) & 1u) ^ 1u);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int kb = 0; kb < kSkKB; ++kb) {
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
                tmem_st32(tmem + tlane + (uint32_t)(32 * kSkKB * a + 32 * kb), w);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(afull_bar(a));
        }
    } else {
        // ---------------- epilogue: one weight row per thread ----------------
        const int qd = warp & 3;
        const int bit = lane >> 3, j = lane & 7;
        const int row128 = 32 * qd + lane;  // D row (TMEM lane)
        float* tok_s = reinterpret_cast<float*>(sm + kSkOffTok);
        float* tok_y = tok_s + kSkMaxTokens;
        int* tok_rs = reinterpret_cast<int*>(tok_y + kSkMaxTokens);
        const int et = threadIdx.x - 32 * kSkEpiWarp0;  // 0..127
        int staged = -1;
        SkCursor cur;
        if (n_items) cur.start(b, i0);
        int64_t item = i0;
        uint32_t tl = 0;
        while (item < i1 && ok) {
            // the part of (cur.p, cur.tile) inside this CTA's share; the
            // problem's constants are copied to registers once per part
            const SkProblem pr = b.p[cur.p];
            if (staged != cur.p) {  // this problem's token scales and row sums, once
                sk_epi_sync();
                if (et < b.M) {
                    const float sx = pr.epi == kEpiI32 ? 1.0f : __ldcg(pr.s_x + et);
                    tok_s[et] = sx;
                    tok_y[et] = __frcp_rn(sx);
                    tok_rs[et] = __ldcg(pr.rowsum + et);
                }
                sk_epi_sync();
                staged = cur.p;
            }
            const int64_t tile_first = pr.item0 + (int64_t)cur.tile * pr.kst;
            const int64_t tile_end = tile_first + pr.kst;
            const int64_t part_end = min(tile_end, i1);
            const bool started_before = item > tile_first;
            const bool continues = part_end < tile_end;
            const int d = (int)(tl & 1);
            const bool got = mbar_wait(dfull_bar(d), (tl >> 1) & 1u);
            if (!sk_epi_all(got)) { ok = false; break; }
            tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(32 * qd) << 16) + kSkDCol0 + (uint32_t)d * kSkDBuf;
            // a finisher first waits for the partial sums of every later CTA
            // whose share starts inside this tile (CTAs c+1 .. c_end-1); the
            // lanes of the first epilogue warp poll those flags side by side
            int64_t c_end = c + 1;
            bool waited = true;
            if (!started_before && continues) {
                while (c_end < G && sk_share_start(b, c_end, G) < tile_end) ++c_end;
                if (warp == kSkEpiWarp0) {
                    const unsigned long long t0 = globaltimer_ns();
                    for (int64_t c2 = c + 1 + lane; c2 < c_end && waited; c2 += 32) {
                        while (ld_acquire_u64(b.flags + c2) != b.epoch) {
                            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                                atomicOr(&g_status, kStatusTimeout);
                                waited = false;
                                break;
                            }
                        }
                    }
                }
                waited = sk_epi_all(waited);  // also orders the flags before the reads
            }
            const int r = cur.tile * kSkRows + 8 * qd + j;  // packed row
            const int64_t n = (int64_t)bit * pr.R + r;
            const int halves = (b.npad + 31) >> 5;
            for (int h = 0; h < halves; ++h) {  // 32 tokens at a time
                uint32_t v[32];
                tmem_ld32(taddr + (uint32_t)(32 * h), v);
                for (int ch = 1; ch < chains; ++ch) {  // sum the accumulator chains
                    uint32_t u[32];
                    tmem_ld32(taddr + (uint32_t)(ch * dstride + 32 * h), u);
#pragma unroll
                    for (int m = 0; m < 32; ++m) v[m] += u[m];
                }
                if (started_before) {
                    // contributor: leave the partial sums for the tile's finisher,
                    // each weight row's npad sums contiguous (16-byte stores)
                    uint4* dst = reinterpret_cast<uint4*>(b.part + ((size_t)c * 128 + row128) * b.npad + 32 * h);
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        if (32 * h + 4 * k < b.npad)
                            dst[k] = make_uint4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
                } else if (waited) {
                    // one contributor at a time, all of its 16-byte loads in flight
                    for (int64_t c2 = c + 1; c2 < c_end; ++c2) {
                        const uint4* src =
                            reinterpret_cast<const uint4*>(b.part + ((size_t)c2 * 128 + row128) * b.npad + 32 * h);
                        uint4 w[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            w[k] = 32 * h + 4 * k < b.npad ? __ldcg(src + k) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            v[4 * k] += w[k].x;
                            v[4 * k + 1] += w[k].y;
                            v[4 * k + 2] += w[k].z;
                            v[4 * k + 3] += w[k].w;
                        }
                    }
                    if (r < pr.R) {
#pragma unroll
                        for (int m = 0; m < 32; ++m) {
                            const int mm = 32 * h + m;
                            if (mm < b.M) sk_store(pr, mm, n, (int)v[m] - tok_rs[mm], tok_s[mm], tok_y[mm]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dempty_bar(d));
            if (started_before) {  // raise this CTA's flag once all four warps wrote
                __threadfence();
                sk_epi_sync();
                if (warp == kSkEpiWarp0 && lane == 0) st_release_u64(b.flags + c, b.epoch);
            } else if (continues) {
                sk_epi_sync();  // every warp has read before the flags are cleared
                if (threadIdx.x == kSkEpiWarp0 * 32)
                    for (int64_t c2 = c + 1; c2 < c_end; ++c2) b.flags[c2] = 0ull;
                if (!waited) ok = false;
            }
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
