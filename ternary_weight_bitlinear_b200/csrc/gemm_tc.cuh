// gemm_tc.cuh -- BitLinear matmul on the 5th-generation tensor cores (tcgen05),
// for token counts beyond the decode kernel (prefill, batched decode).
//
// acc[m,n] = sum_k q[m,k] t[n,k] ("Transformers 实战 BitNet 1.58 位量化"
// walkthrough, "推理侧 BitLinear": unpack_weights + F.linear) as a dense int8
// contraction: D[m, n] = sum_k q[m,k] * code[n,k] with code = t + 1 in {0,1,2},
// then acc = D - rowsum_q[m] (exact), rescaled like the decode kernel.
//
// Tile: 128 tokens x 256 output rows (= 64 packed rows x 4 bit pairs), K in
// stages of 128 bytes.  Persistent CTAs, one per SM, walk the tiles
// round-robin; when the last wave would fill at most half the SMs its tiles
// run as two halves in N each (32 packed rows, MMA N=128), on twice as many
// SMs.
// Warp roles:
//   warp 0      TMA producer: per stage, the 128x128-byte int8 activation tile
//               (A operand, 128-byte swizzle, rows past M zero-filled) and the
//               64x128-byte packed weight tile; no multicast.
//   warps 1-8   expansion: 2-bit codes -> int8 codes written straight into the
//               128-byte-swizzled K-major B operand (256 rows) in shared memory.
//   warp 9      one thread issues tcgen05.mma.cta_group::1.kind::i8
//               (M=128, N=256, K=32) into a TMEM accumulator (2 buffers).
//   warps 10-17 epilogue: each thread owns one token (a TMEM lane of its
//               warp's quadrant) and half of the 256 output rows: tcgen05.ld,
//               minus the token's row sum, rescale (division by the token's
//               scale through its reciprocal, exactness checked per output),
//               16-byte stores of contiguous outputs.
// Loads run up to kTcStages stages ahead; expanded operands are double-buffered.
// Every mbarrier wait is bounded (records BL_ERR_TIMEOUT and unwinds).
#pragma once

#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "decode.cuh"

namespace bl {

constexpr int kTcBM = 128;        // tokens per tile (MMA M)
constexpr int kTcBN = 256;        // output rows per tile (MMA N)
constexpr int kTcBK = 128;        // K bytes per stage (one 128-byte swizzle atom)
constexpr int kTcPackRows = 64;   // packed rows per tile (x 4 bit pairs = kTcBN)
constexpr int kTcStages = 5;      // load stages (A + packed weights)
constexpr int kTcExp = 2;         // expanded-B buffers
constexpr int kTcExpWarps = 8;    // expansion warps (1 .. 8)
constexpr int kTcMmaWarp = 1 + kTcExpWarps;
constexpr int kTcEpiWarp0 = kTcMmaWarp + 1;
constexpr int kTcEpiWarps = 8;    // two per TMEM lane quadrant, each half the columns
constexpr int kTcThreads = 32 * (kTcEpiWarp0 + kTcEpiWarps);
constexpr int kTcABytes = kTcBM * kTcBK;          // 16 KB activations
constexpr int kTcBBytes = kTcBN * kTcBK;          // 32 KB expanded codes
constexpr int kTcPBytes = kTcPackRows * kTcBK;    // 8 KB packed codes
constexpr int kTcStageTx = kTcABytes + kTcPBytes;
// layout from a 1024-aligned base: A[5] | B[2] | P[5] | barriers | tmem addr
constexpr int kTcOffB = kTcStages * kTcABytes;
constexpr int kTcOffP = kTcOffB + kTcExp * kTcBBytes;
// per epilogue warp two 32 x 32 bf16 staging buffers for the TMA stores of y
constexpr int kTcStageOut = 32 * 32 * 2;
constexpr int kTcOffOut = kTcOffP + kTcStages * kTcPBytes;
constexpr int kTcOffBar = kTcOffOut + 2 * 8 * kTcStageOut;
constexpr int kTcNumBars = 2 * kTcStages + 2 * kTcExp + 5;
constexpr int kTcOffTmem = kTcOffBar + 8 * kTcNumBars;
constexpr int kTcSmemBytes = kTcOffTmem + 16 + 1024;   // + alignment slack
constexpr uint32_t kTcTmemCols = 2 * kTcBN;           // two accumulators
static_assert(kTcSmemBytes <= 227 * 1024, "shared memory budget");
static_assert((kTcPackRows * 8) % (32 * kTcExpWarps) == 0, "expansion items per thread");
static_assert(kTcEpiWarps == 8 && (kTcEpiWarp0 + kTcEpiWarps) * 32 <= 1024, "epilogue warps");

struct TcArgs {
    const uint8_t* P;          // [R,K] (through tmap_p)
    const float* s_x;          // [M]
    const int32_t* rowsum;     // [M]
    void* y;                   // [M,N]
    const uint16_t* residual;  // bf16 [M,N] or nullptr
    float beta;
    int epi;
    int M;
    int K;
    int R;
    int64_t N;
    int tiles_n;               // ceil(R / 64)
    int tiles_m;               // ceil(M / 128)
    int vec_ok;                // outputs of 32 consecutive rows can use 16-byte accesses
    int tma_store;             // bf16 y without residual: full 32 x 32 chunks leave by TMA store
    float beta2;               // up projection's scale (kEpiGateUp)
    const float* beta_dev;     // when set: beta is read from device memory
    int64_t full_units;        // tiles processed whole; the rest as two N-halves each
    int64_t units;             // full_units + 2 * (tiles - full_units)
};

// Work unit u of the round-robin schedule: a whole 128 x 256 tile, or (past
// full_units) one half in N of a tile of the last partial wave -- 32 of its
// 64 packed rows, 128 output rows -- so that wave's tiles spread over twice
// as many SMs.
struct TcUnit {
    int tn, tm;
    int nh;    // -1: whole tile; 0 / 1: packed rows 0-31 / 32-63 of it
    __device__ __forceinline__ TcUnit(const TcArgs& a, int64_t u) {
        int64_t t = u;
        nh = -1;
        if (u >= a.full_units) {
            t = a.full_units + (u - a.full_units) / 2;
            nh = (int)((u - a.full_units) & 1);
        }
        tn = (int)(t / a.tiles_m);
        tm = (int)(t % a.tiles_m);
    }
};

// ---- tcgen05 / TMA wrappers ------------------------------------------------
// Shared -> global tile store (TMA, bulk-group completion); rows or columns
// outside the tensor are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(src), "r"(x), "r"(y)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most one of this thread's bulk stores still reads shared memory.
__device__ __forceinline__ void bulk_wait_read_1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// Wait until this thread's bulk stores are complete.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(dst_smem), "r"(cols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, int8 x int8 -> int32.
__device__ __forceinline__ void tc_mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05 op this thread issued so far completes.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(bar) : "memory");
}

// 32 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32"
        " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
        " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31},"
        " [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 16 consecutive 32-bit TMEM columns of this thread's lane (no wait).
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32"
        " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (stride byte offset), descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: int32 accumulate, signed 8-bit A and B, both
// K-major, M = kTcBM, N = kTcBN (or half of it for a half unit).
constexpr uint32_t kTcIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kTcBN >> 3) << 17) |
                              ((uint32_t)(kTcBM >> 4) << 24);
constexpr uint32_t kTcIdescHalf = (2u << 4) | (1u << 7) | (1u << 10) |
                                  ((uint32_t)(kTcBN / 2 >> 3) << 17) | ((uint32_t)(kTcBM >> 4) << 24);

// Byte offset of the 16-byte chunk `chunk16` of `row` in a 128-byte-wide,
// 128-byte-swizzled K-major tile (8-row groups of 1024 bytes).
__device__ __forceinline__ uint32_t sw128_offset(int row, int chunk16) {
    return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((chunk16 ^ (row & 7)) << 4));
}

// scale_fast for two outputs at once on the paired fp32 pipe (f32x2).
__device__ __forceinline__ void scale_fast2(int a0, int a1, float beta, const PairDiv& d, float& y0,
                                            float& y1, bool& ok0, bool& ok1) {
    float r0, r1;
    asm("{\n\t.reg .b64 A, Q, R, B, Y, N;\n\t"
        "mov.b64 A, {%4, %5};\n\t"
        "mov.b64 B, {%6, %6};\n\t"
        "mov.b64 Y, {%7, %7};\n\t"
        "mov.b64 N, {%8, %8};\n\t"
        "mul.rn.f32x2 A, A, B;\n\t"     // a = RN(acc * beta)
        "mul.rn.f32x2 Q, A, Y;\n\t"     // q = RN(a * y)
        "fma.rn.f32x2 R, Q, N, A;\n\t"  // a - q*s
        "fma.rn.f32x2 Q, R, Y, Q;\n\t"  // q + (a - q*s)*y
        "fma.rn.f32x2 R, Q, N, A;\n\t"  // exact remainder of the refined q
        "mov.b64 {%0, %1}, Q;\n\t"
        "mov.b64 {%2, %3}, R;\n\t}"
        : "=f"(y0), "=f"(y1), "=f"(r0), "=f"(r1)
        : "f"(__int2float_rn(a0)), "f"(__int2float_rn(a1)), "f"(beta), "f"(d.y), "f"(d.ns));
    const uint32_t qb0 = __float_as_uint(y0), qb1 = __float_as_uint(y1);
    const float h0 = __fmul_rn(__uint_as_float((qb0 & 0x7F800000u) - 0x0C000000u), d.s);
    const float h1 = __fmul_rn(__uint_as_float((qb1 & 0x7F800000u) - 0x0C000000u), d.s);
    ok0 = a0 == 0 || ((qb0 & 0x007FFFFFu) != 0u && fabsf(r0) < h0);
    ok1 = a1 == 0 || ((qb1 & 0x007FFFFFu) != 0u && fabsf(r1) < h1);
}

// y[j] = RN32(RN32((v[j] - rsum) * beta) / s) for 16 outputs.
__device__ __forceinline__ void scale16(const uint32_t* v, int rsum, float beta, const PairDiv& d,
                                        float (&y)[16]) {
    uint32_t bad = 0;
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
        bool ok0, ok1;
        scale_fast2((int)v[j] - rsum, (int)v[j + 1] - rsum, beta, d, y[j], y[j + 1], ok0, ok1);
        bad |= ((ok0 ? 0u : 1u) | (ok1 ? 0u : 2u)) << j;
    }
    if (!d.fast) bad = 0xFFFFu;
    if (bad) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (bad & (1u << j)) y[j] = scale_slow((int)v[j] - rsum, beta, d.s, d.y);
    }
}

// y = RN32(RN32(acc * beta) / s_x)
__device__ __forceinline__ float tc_scale(int acc, float beta, const PairDiv& s_x) {
    return recip_div(__fmul_rn(__int2float_rn(acc), beta), RecipDiv{s_x.s, s_x.y});
}

// Store 32 consecutive outputs y[m, n0 .. n0+31] of one token (scalar path:
// only rows < R, i.e. n0 + j with j < valid).
__device__ __forceinline__ void tc_store_row32(const TcArgs& a, float beta, int64_t base,
                                               const uint32_t (&v)[32], int rsum, const PairDiv& s_x,
                                               int valid) {
    if (a.vec_ok && valid == 32) {
        if (a.epi == kEpiBF16) {
            uint32_t w[16];
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                float y[16];
                scale16(v + 16 * g, rsum, beta, s_x, y);
#pragma unroll
                for (int j = 0; j < 8; ++j) w[8 * g + j] = pack_bf16x2(y[2 * j], y[2 * j + 1]);
            }
            if (a.residual) {
                const uint4* rp = reinterpret_cast<const uint4*>(a.residual + base);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint4 r = __ldcg(rp + c);
                    const uint32_t rr[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const uint32_t x = w[4 * c + h];
                        w[4 * c + h] = pack_bf16x2(
                            __fadd_rn(bf16_bits_to_float(rr[h] & 0xFFFFu), bf16_bits_to_float(x & 0xFFFFu)),
                            __fadd_rn(bf16_bits_to_float(rr[h] >> 16), bf16_bits_to_float(x >> 16)));
                    }
                }
            }
            uint4* yp = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.y) + base);
#pragma unroll
            for (int c = 0; c < 4; ++c) yp[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
        } else if (a.epi == kEpiF32) {
            uint4* yp = reinterpret_cast<uint4*>(static_cast<uint32_t*>(a.y) + base);
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                float y[16];
                scale16(v + 16 * g, rsum, beta, s_x, y);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    yp[4 * g + c] = make_uint4(__float_as_uint(y[4 * c]), __float_as_uint(y[4 * c + 1]),
                                               __float_as_uint(y[4 * c + 2]), __float_as_uint(y[4 * c + 3]));
            }
        } else {
            uint4* yp = reinterpret_cast<uint4*>(static_cast<uint32_t*>(a.y) + base);
#pragma unroll
            for (int c = 0; c < 8; ++c)
                yp[c] = make_uint4(v[4 * c] - rsum, v[4 * c + 1] - rsum, v[4 * c + 2] - rsum,
                                   v[4 * c + 3] - rsum);
        }
        return;
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        if (j >= valid) break;
        const int acc = (int)v[j] - rsum;
        const int64_t idx = base + j;
        if (a.epi == kEpiI32) {
            static_cast<int32_t*>(a.y)[idx] = acc;
        } else if (a.epi == kEpiF32) {
            static_cast<float*>(a.y)[idx] = tc_scale(acc, beta, s_x);
        } else {
            uint16_t b = float_to_bf16_bits(tc_scale(acc, beta, s_x));
            if (a.residual)
                b = float_to_bf16_bits(
                    __fadd_rn(bf16_bits_to_float(__ldcg(a.residual + idx)), bf16_bits_to_float(b)));
            static_cast<uint16_t*>(a.y)[idx] = b;
        }
    }
}

// Expand one stage of packed codes into the B operand: packed row rr, bit
// pair i -> B row i * rows + rr (rows = 64 packed rows, or the 32 of a half
// unit starting at pk), codes t + 1 as int8 in the 128-byte swizzle.
template <bool kHalf>
__device__ __forceinline__ void tc_expand(const uint8_t* pk, uint8_t* bt, int e0) {
    constexpr int rows = kHalf ? kTcPackRows / 2 : kTcPackRows;
#pragma unroll
    for (int it = 0; it < rows * 8 / (32 * kTcExpWarps); ++it) {
        const int item = e0 + it * 32 * kTcExpWarps;  // (packed row, 16-byte chunk)
        const int rr = item >> 3, ch = item & 7;
        const uint4 w = *reinterpret_cast<const uint4*>(pk + rr * kTcBK + ch * 16);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 c = make_uint4((w.x >> (2 * i)) & 0x03030303u, (w.y >> (2 * i)) & 0x03030303u,
                                       (w.z >> (2 * i)) & 0x03030303u, (w.w >> (2 * i)) & 0x03030303u);
            *reinterpret_cast<uint4*>(bt + sw128_offset(i * rows + rr, ch)) = c;
        }
    }
}

__global__ void __launch_bounds__(kTcThreads, 1) gemm_tc_kernel(
    const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_p,
    const __grid_constant__ CUtensorMap tmap_y, const TcArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;  // 1024-aligned for the 128-byte swizzle
    uint8_t* sm = smem_raw + (base - raw);
    const uint32_t sA = base, sB = base + kTcOffB, sP = base + kTcOffP;
    const uint32_t bars = base + kTcOffBar;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (kTcStages + s); };
    auto bready_bar = [&](int e) { return bars + 8u * (2 * kTcStages + e); };
    auto bfree_bar = [&](int e) { return bars + 8u * (2 * kTcStages + kTcExp + e); };
    auto accfull_bar = [&](int b) { return bars + 8u * (2 * kTcStages + 2 * kTcExp + b); };
    auto accempty_bar = [&](int b) { return bars + 8u * (2 * kTcStages + 2 * kTcExp + 2 + b); };
    const uint32_t mma_done_bar = bars + 8u * (2 * kTcStages + 2 * kTcExp + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kTcOffTmem);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int e = 0; e < kTcExp; ++e) {
            mbar_init(bready_bar(e), kTcExpWarps);
            mbar_init(bfree_bar(e), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(accfull_bar(b), 1);
            mbar_init(accempty_bar(b), kTcEpiWarps);
        }
        mbar_init(mma_done_bar, 1);
        mbar_init_fence();
    }
    if (warp == kTcMmaWarp) tmem_alloc(smem_addr(tmem_slot), kTcTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    pdl_wait();
    pdl_launch_dependents();

    const int kstages = (a.K + kTcBK - 1) / kTcBK;
    bool ok = true;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            uint32_t g = 0;
            uint32_t inflight_from = 0;  // stages [inflight_from, g) may still be landing
            for (int64_t u = blockIdx.x; u < a.units && ok; u += gridDim.x) {
                const TcUnit un(a, u);
                const int tn = un.tn, tm = un.tm;
                for (int ks = 0; ks < kstages; ++ks, ++g) {
                    const int s = (int)(g % kTcStages);
                    if (!mbar_wait(empty_bar(s), ((g / kTcStages) & 1u) ^ 1u)) { ok = false; break; }
                    inflight_from = g >= kTcStages ? g - kTcStages + 1 : 0;
                    mbar_arrive_expect_tx(full_bar(s), kTcStageTx);
                    tma_load_2d(sA + s * kTcABytes, &tmap_q, ks * kTcBK, tm * kTcBM, full_bar(s));
                    tma_load_2d(sP + s * kTcPBytes, &tmap_p, ks * kTcBK, tn * kTcPackRows, full_bar(s));
                }
            }
            // after a failed wait, let the copies still in flight land first
            if (!ok)
                for (uint32_t j = inflight_from; j < g; ++j)
                    mbar_wait(full_bar((int)(j % kTcStages)), (j / kTcStages) & 1u);
        }
    } else if (warp >= 1 && warp <= kTcExpWarps) {
        // ---------------- expansion: 2-bit codes -> int8 B tile ----------------
        const int e0 = threadIdx.x - 32;  // 0 .. 32*kTcExpWarps-1
        uint32_t g = 0;
        // one instantiation of the stage loop per unit kind keeps the whole-tile loop branch-free
        auto expand_unit = [&](auto half_tag, const int rr0) {
            constexpr bool kHalf = decltype(half_tag)::value;
            for (int ks = 0; ks < kstages; ++ks, ++g) {
                const int s = (int)(g % kTcStages), e = (int)(g % kTcExp);
                const bool got = mbar_wait(full_bar(s), (g / kTcStages) & 1u) &&
                                 mbar_wait(bfree_bar(e), ((g / kTcExp) & 1u) ^ 1u);
                if (!__all_sync(0xffffffffu, got)) return false;
                tc_expand<kHalf>(sm + kTcOffP + s * kTcPBytes + rr0 * kTcBK, sm + kTcOffB + e * kTcBBytes, e0);
                fence_proxy_async_smem();  // generic writes -> visible to the tensor core
                __syncwarp();
                if (lane == 0) mbar_arrive(bready_bar(e));
            }
            return true;
        };
        for (int64_t u = blockIdx.x; u < a.units && ok; u += gridDim.x) {
            const TcUnit un(a, u);
            ok = un.nh < 0 ? expand_unit(std::false_type{}, 0)
                           : expand_unit(std::true_type{}, un.nh * (kTcPackRows / 2));
        }
    } else if (warp == kTcMmaWarp) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            uint32_t g = 0, tl = 0;
            for (int64_t u = blockIdx.x; u < a.units && ok; u += gridDim.x, ++tl) {
                const uint32_t idesc = u >= a.full_units ? kTcIdescHalf : kTcIdesc;
                const int buf = (int)(tl & 1);
                if (!mbar_wait(accempty_bar(buf), ((tl >> 1) & 1u) ^ 1u)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(buf * kTcBN);
                for (int ks = 0; ks < kstages; ++ks, ++g) {
                    const int s = (int)(g % kTcStages), e = (int)(g % kTcExp);
                    if (!mbar_wait(full_bar(s), (g / kTcStages) & 1u) ||
                        !mbar_wait(bready_bar(e), (g / kTcExp) & 1u)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = smem_desc_sw128(sA + s * kTcABytes);
                    const uint64_t bd = smem_desc_sw128(sB + e * kTcBBytes);
#pragma unroll
                    for (int kk = 0; kk < kTcBK / 32; ++kk)  // +32 bytes = +2 in the address field
                        tc_mma_i8(d, ad + 2u * kk, bd + 2u * kk, idesc, (ks | kk) != 0);
                    tc_commit(empty_bar(s));  // activation + packed stage reusable
                    tc_commit(bfree_bar(e));  // expanded operand reusable
                }
                if (!ok) break;
                tc_commit(accfull_bar(buf));  // accumulator ready for the epilogue
            }
            // every MMA this thread issued has finished before TMEM is freed
            tc_commit(mma_done_bar);
            mbar_wait(mma_done_bar, 0);
        }
    } else {
        // ---------------- epilogue: one token per thread ----------------
        const float beta = a.beta_dev ? __ldcg(a.beta_dev) : a.beta;
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        const int half = (warp - kTcEpiWarp0) >> 2;  // which 128 of the 256 columns
        // this warp's two staging buffers (64-byte rows, 64-byte swizzle: chunk c
        // of row r sits at chunk c ^ ((r >> 1) & 3))
        uint8_t* stage = sm + kTcOffOut + (warp - kTcEpiWarp0) * 2 * kTcStageOut;
        uint32_t nstore = 0;
        uint32_t tl = 0;
        for (int64_t u = blockIdx.x; u < a.units && ok; u += gridDim.x, ++tl) {
            const TcUnit un(a, u);
            const int tn = un.tn, tm = un.tm;
            // columns of this warp: [cb, ce) of the unit's 256 (whole) or 128 (half);
            // column c is bit pair c >> lg of packed row tn * 64 + rr0 + (c & (2^lg - 1))
            const int ucols = un.nh < 0 ? kTcBN : kTcBN / 2;
            const int cb = half * (ucols / 2), ce = cb + ucols / 2;
            const int lg = un.nh < 0 ? 6 : 5;
            const int rr0 = un.nh < 0 ? 0 : un.nh * (kTcPackRows / 2);
            const int buf = (int)(tl & 1);
            const int m = tm * kTcBM + q * 32 + lane;  // this thread's token
            const bool live = m < a.M;
            const PairDiv sx = pair_div_init((live && a.epi != kEpiI32) ? __ldcg(a.s_x + m) : 1.0f, beta);
            const int rsum = live ? __ldcg(a.rowsum + m) : 0;
            const bool got = mbar_wait(accfull_bar(buf), (tl >> 1) & 1u);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * kTcBN);
            if (a.epi == kEpiGateUp) {
                // gate columns [0, ucols/2) (bit pairs 0, 1), their up rows
                // ucols/2 further on; this warp takes a quarter of the columns
                const PairDiv sx2 = pair_div_init(sx.s, a.beta2);
                const int gcb = half * (ucols / 4), gce = gcb + ucols / 4;
#pragma unroll 1
                for (int c0 = gcb; c0 < gce; c0 += 32) {
                    uint32_t w[16];  // 32 bf16 outputs, two per word
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        uint32_t gv[16], uv[16];
                        tmem_ld16_nowait(taddr + (uint32_t)(c0 + 16 * h2), gv);
                        tmem_ld16_nowait(taddr + (uint32_t)(c0 + 16 * h2 + ucols / 2), uv);
                        tmem_ld_wait();
                        float yg[16], yu[16];
                        scale16(gv, rsum, beta, sx, yg);
                        scale16(uv, rsum, a.beta2, sx2, yu);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            w[8 * h2 + j] =
                                (uint32_t)relu2_mul_one(float_to_bf16_bits(yg[2 * j]), float_to_bf16_bits(yu[2 * j])) |
                                ((uint32_t)relu2_mul_one(float_to_bf16_bits(yg[2 * j + 1]),
                                                         float_to_bf16_bits(yu[2 * j + 1])) << 16);
                    }
                    const int i = c0 >> lg;                                          // bit pair 0 or 1
                    const int r = tn * kTcPackRows + rr0 + (c0 & ((1 << lg) - 1));  // first packed row
                    const int valid = min(32, a.R - r);
                    if (a.tma_store && valid == 32) {
                        uint8_t* buf_out = stage + (nstore & 1) * kTcStageOut;
                        if (lane == 0) bulk_wait_read_1();
                        __syncwarp();
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            *reinterpret_cast<uint4*>(buf_out + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)) =
                                make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0)
                            tma_store_2d(&tmap_y, smem_addr(buf_out), i * a.R + r, tm * kTcBM + q * 32);
                        ++nstore;
                    } else if (live && valid > 0) {
                        uint16_t* zp = static_cast<uint16_t*>(a.y) + (int64_t)m * a.N + (int64_t)i * a.R + r;
                        if (a.vec_ok && valid == 32) {
#pragma unroll
                            for (int c = 0; c < 4; ++c)
                                reinterpret_cast<uint4*>(zp)[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (j < valid) zp[j] = (uint16_t)(w[j >> 1] >> (16 * (j & 1)));
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(accempty_bar(buf));
                continue;
            }
#pragma unroll 1
            for (int c0 = cb; c0 < ce; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(taddr + (uint32_t)c0, v);
                const int i = c0 >> lg;                                          // bit pair
                const int r = tn * kTcPackRows + rr0 + (c0 & ((1 << lg) - 1));  // first packed row
                const int valid = min(32, a.R - r);
                if (a.tma_store && valid == 32) {
                    // 32 tokens x 32 outputs: pack, stage, one TMA store (rows past M are dropped)
                    uint32_t w[16];
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        float y[16];
                        scale16(v + 16 * g, rsum, beta, sx, y);
#pragma unroll
                        for (int j = 0; j < 8; ++j) w[8 * g + j] = pack_bf16x2(y[2 * j], y[2 * j + 1]);
                    }
                    uint8_t* buf_out = stage + (nstore & 1) * kTcStageOut;
                    if (lane == 0) bulk_wait_read_1();  // the store that used this buffer has read it
                    __syncwarp();
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        *reinterpret_cast<uint4*>(buf_out + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)) =
                            make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0)
                        tma_store_2d(&tmap_y, smem_addr(buf_out), i * a.R + r, tm * kTcBM + q * 32);
                    ++nstore;
                } else if (live && valid > 0) {
                    tc_store_row32(a, beta, (int64_t)m * a.N + (int64_t)i * a.R + r, v, rsum, sx, valid);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(accempty_bar(buf));
        }
        if (lane == 0) bulk_wait_all();  // the stores are complete before the CTA's memory goes
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kTcMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTcTmemCols);
    }
}

}  // namespace bl
