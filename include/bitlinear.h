/*
 * bitlinear.h -- C ABI of libbitlinear.so, the B200 (sm_100a) implementation of
 * the inference-time BitLinear forward of BitNet b1.58 (ternary weights, int8
 * activations: W1.58A8).
 *
 * Sources (web pages, cited by title and section):
 *   [QG] "BitNet" -- transformers quantization guide, steps 1-3 of the recipe.
 *   [BG] "Transformers 实战 BitNet 1.58 位量化：BitLinear 原理、量化流程与推理加载全指南",
 *        sections "BitLinear 的三步量化" (weight / activation quantisation) and
 *        "推理侧 BitLinear：打包权重、解包与缩放" (pack_weights, unpack_weights,
 *        BitLinear.forward, post_quant_process).
 *   [MD] "BitNet" -- transformers model doc, model details (W1.58A8, ReLU^2,
 *        subln) and BitNetConfig (rms_norm_eps = 1e-5).
 *
 * Conventions for every entry point
 *   - Pointers marked "device" must point to memory the current CUDA device can
 *     read/write (cudaMalloc, torch CUDA tensors).  The caller owns all memory;
 *     the library allocates nothing and keeps no pointer after returning.
 *   - Row-major, contiguous tensors.  bf16 tensors are passed as uint16_t bit
 *     patterns.  Sizes are element counts.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous on that stream; results are ready when the stream is.
 *   - Arguments are checked on the host before anything is launched; a failed
 *     check returns its status and launches nothing.  A launch failure returns
 *     BL_ERR_CUDA.  A kernel that stops waiting on an internal barrier after its
 *     time limit records BL_ERR_TIMEOUT in a device status word, read back with
 *     bitlinear_device_status().
 *   - Shapes: M >= 0 tokens (M == 0 is a no-op returning BL_OK), K > 0 input
 *     features with K % 16 == 0 and K <= BL_MAX_K, N > 0 output features with
 *     N % 4 == 0.  Tensor pointers must be 16-byte aligned.
 *   - Numerics: every floating-point step is a single IEEE operation rounded to
 *     nearest-even, in the order written below; sums named "exact" are taken
 *     exactly up to one final rounding to binary64 (computed in binary64 with
 *     error-free transformations).  Codes, packed bytes and int32 accumulators
 *     are therefore reproducible bit for bit.
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BL_ABI_VERSION 1
#define BL_MAX_K 65536
#define BL_MAX_BATCH 256

typedef enum {
    BL_OK = 0,
    BL_ERR_NULL = 1,      /* a required pointer is NULL */
    BL_ERR_SHAPE = 2,     /* M/K/N outside the rules above */
    BL_ERR_ALIGN = 3,     /* a tensor pointer is not 16-byte aligned */
    BL_ERR_DTYPE = 4,     /* unknown output dtype, or a dtype/option mismatch */
    BL_ERR_WORKSPACE = 5, /* workspace missing or smaller than required */
    BL_ERR_CUDA = 6,      /* a CUDA launch or runtime call failed */
    BL_ERR_TIMEOUT = 7,   /* a device-side bounded wait expired */
    BL_ERR_DEVICE = 8     /* no usable sm_100 device is current */
} bl_status;

typedef enum { BL_OUT_BF16 = 0, BL_OUT_F32 = 1 } bl_out_dtype;

/* Version of this ABI (BL_ABI_VERSION). */
int bitlinear_abi_version(void);

/* Static description of a status code. */
const char* bitlinear_status_string(bl_status status);

/* Text of the CUDA error behind the most recent BL_ERR_CUDA returned on the
 * calling thread (empty if none).  Owned by the library; valid until the next
 * call on this thread. */
const char* bitlinear_last_error(void);

/* ---- weight preparation (offline, load time) ---------------------------- */

/* Workspace needed by bitlinear_pack for an [N,K] master weight. */
bl_status bitlinear_pack_workspace_size(int64_t N, int64_t K, size_t* bytes);

/* Absmean ternarisation and 2-bit packing of a master weight ([BG] "BitLinear
 * 的三步量化" steps 1-2, [QG] steps 1-2; packing: [BG] "推理侧 BitLinear",
 * pack_weights).
 *   W         device fp32 [N,K] master weight (nn.Linear layout: out x in).
 *   P         device uint8 [N/4,K] output.  Bits 2i..2i+1 of P[r,k] hold
 *             t[i*N/4 + r, k] + 1 in {0,1,2} ("block" layout: bit pair i is the
 *             i-th quarter of the output rows).
 *   beta_out  device float[1] output: beta = max(RN32(exact sum|W| / (N*K)),
 *             1e-5), the absmean weight scale later passed to the forward.
 *   t[n,k] = clamp(round_half_even(RN32(W[n,k] * RN32(1/beta))), -1, 1).
 *   workspace device, >= bitlinear_pack_workspace_size(N, K) bytes. */
bl_status bitlinear_pack(const float* W, int64_t N, int64_t K, uint8_t* P, float* beta_out,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Pack already-ternary weights t[N,K] (values in {-1,0,1}, device int8) into P
 * [N/4,K] with the layout above ([BG] pack_weights).  Values outside {-1,0,1}
 * are not checked on the device; they produce unspecified codes. */
bl_status bitlinear_pack_ternary(const int8_t* t, int64_t N, int64_t K, uint8_t* P,
                                 void* stream);

/* Inverse of the packing ([BG] unpack_weights: bit pair i, masked by 3 << 2i,
 * shifted down, minus one): t[i*N/4 + r, k] = ((P[r,k] >> 2i) & 3) - 1, into
 * device int8 t[N,K].  A bit pair 11 (never written by the packers) gives +2. */
bl_status bitlinear_unpack(const uint8_t* P, int64_t N, int64_t K, int8_t* t, void* stream);

/* ---- activation quantisation --------------------------------------------- */

/* Optional RMSNorm, then per-token absmax int8 quantisation ([BG] "BitLinear
 * 的三步量化" step 3, [QG] step 3; the norm is the optional first step of
 * BitLinear.forward in [BG] "推理侧 BitLinear", eps from [MD] BitNetConfig).
 *   x       device bf16 [M,K].
 *   gain    device bf16 [K] RMSNorm weight, or NULL for no norm.
 *   eps     RMSNorm epsilon (ignored when gain is NULL).
 *   q       device int8 [M,K] output codes.
 *   s_x     device fp32 [M] output multipliers.
 *   rowsum  device int32 [M] output sum_k q[m,k], or NULL.
 * With the norm:  r = RN32(1/sqrt(exact sum_k x^2 / K + eps)) (binary64 ops),
 *                 h = RN32(RN32(x*r)*gain);  without it: h = x.
 * Then s_x = RN32(127 / max(max_k |h|, 1e-5)), q = clamp(rint(RN32(h*s_x)),
 * -128, 127).  No workspace. */
bl_status bitlinear_act_quant(const uint16_t* x, const uint16_t* gain, float eps, int64_t M,
                              int64_t K, int8_t* q, float* s_x, int32_t* rowsum, void* stream);

/* ---- forward -------------------------------------------------------------- */

/* Workspace bitlinear_forward needs for this shape: the int8 codes, s_x and
 * row sums of the quantised activations (0 when M == 0). */
bl_status bitlinear_forward_workspace_size(int64_t M, int64_t K, int64_t N, size_t* bytes);

/* The whole BitLinear forward ([BG] "推理侧 BitLinear": optional RMSNorm,
 * unpack, activation_quant, F.linear, post_quant_process):
 *   x      device bf16 [M,K];  gain: device bf16 [K] or NULL (no norm);  eps.
 *   P      device uint8 [N/4,K] packed weights (bitlinear_pack layout).
 *   beta   host float: the absmean weight scale of P.
 *   y      device [M,N], bf16 or fp32 per y_dtype:
 *          y = RN32(RN32(float(acc) * beta) / s_x[m]), acc = sum_k q[m,k] t[n,k]
 *          exact in int32; rounded once more to bf16 when y_dtype is BL_OUT_BF16.
 *   workspace  device, >= bitlinear_forward_workspace_size(M,K,N) bytes (may be
 *          NULL when that size is 0).  Holds the int8 codes between kernels. */
bl_status bitlinear_forward(const uint16_t* x, const uint16_t* gain, float eps,
                            const uint8_t* P, float beta, int64_t M, int64_t K, int64_t N,
                            void* y, bl_out_dtype y_dtype, void* workspace,
                            size_t workspace_bytes, void* stream);

/* One independent BitLinear problem of a batch (all pointers device). */
typedef struct {
    const uint16_t* x;        /* bf16 [M,K] input */
    const uint16_t* gain;     /* bf16 [K] RMSNorm weight, or NULL for no norm */
    const uint8_t* P;         /* uint8 [N/4,K] packed weights */
    void* y;                  /* [M,N] output, bf16 or fp32 per y_dtype */
    const uint16_t* residual; /* bf16 [M,N] added after the bf16 rounding, or NULL */
    int64_t K;
    int64_t N;
    float beta;               /* absmean weight scale of P */
    bl_out_dtype y_dtype;     /* BL_OUT_BF16 is required with a residual */
} bl_problem;

/* Workspace bitlinear_forward_batch needs: the sum over problems of
 * bitlinear_forward_workspace_size(M, K, N). */
bl_status bitlinear_forward_batch_workspace_size(const bl_problem* problems, int count, int64_t M,
                                                 size_t* bytes);

/* `count` (1..BL_MAX_BATCH) independent BitLinear forwards with the same
 * token count M and RMSNorm eps, each exactly as bitlinear_forward computes it
 * (plus the optional residual of bitlinear_forward_quantized; y may alias the
 * residual).  For M <= 4 (decode) all problems' activations are quantised by
 * one launch and all weights are streamed by one more, so a whole layer's
 * projections cost two launches.  `problems` is a host array read during the
 * call only.  workspace: device, >= bitlinear_forward_batch_workspace_size. */
bl_status bitlinear_forward_batch(const bl_problem* problems, int count, int64_t M, float eps,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* One matmul problem on already-quantised activations (all pointers device;
 * q, s_x, rowsum as produced by bitlinear_act_quant with a non-NULL rowsum). */
typedef struct {
    const int8_t* q;          /* int8 [M,K] codes */
    const float* s_x;         /* fp32 [M] */
    const int32_t* rowsum;    /* int32 [M] */
    const uint8_t* P;         /* uint8 [N/4,K] packed weights */
    void* y;                  /* [M,N] output, bf16 or fp32 per y_dtype */
    const uint16_t* residual; /* bf16 [M,N] or NULL (BL_OUT_BF16 only) */
    int64_t K;
    int64_t N;
    float beta;
    bl_out_dtype y_dtype;
} bl_quantized_problem;

/* Workspace that lets bitlinear_forward_quantized_batch split row tiles between
 * CTAs for 5 <= M <= 64 (0 for other M): one flag and one block of int32
 * partial sums per CTA. */
bl_status bitlinear_quantized_batch_workspace_size(int64_t M, size_t* bytes);

/* `count` (1..BL_MAX_BATCH) independent bitlinear_forward_quantized problems
 * with the same M.  Problems may share q (projections of one input, e.g. the
 * q|k|v or gate|up projections of a decoder layer).  For M <= 4 one launch
 * streams every problem's weights once; for 5 <= M <= 64 one launch per 64
 * problems does (tensor cores, weights expanded into tensor memory).
 *   workspace  device or NULL.  With at least
 *          bitlinear_quantized_batch_workspace_size(M) bytes every CTA streams
 *          an equal share of the weights; without it (NULL or smaller) shares
 *          are cut at 128-row tile boundaries, with the same results.  A
 *          workspace serves one call at a time; its contents need no
 *          initialisation and are left for the next call. */
bl_status bitlinear_forward_quantized_batch(const bl_quantized_problem* problems, int count,
                                            int64_t M, void* workspace, size_t workspace_bytes,
                                            void* stream);

/* Matmul and rescale on activations already quantised by bitlinear_act_quant
 * (so several projections can share one quantisation):
 *   q [M,K] int8, s_x [M] fp32, rowsum [M] int32 (all device, as produced by
 *   bitlinear_act_quant with a non-NULL rowsum);  P, beta, y, y_dtype as in
 *   bitlinear_forward.
 *   residual  device bf16 [M,N] or NULL.  When given, y_dtype must be
 *             BL_OUT_BF16 and y = bf16(float(residual) + float(bf16(y))) (the
 *             residual add of a decoder block); y may alias residual. */
bl_status bitlinear_forward_quantized(const int8_t* q, const float* s_x, const int32_t* rowsum,
                                      const uint8_t* P, float beta, int64_t M, int64_t K,
                                      int64_t N, void* y, bl_out_dtype y_dtype,
                                      const uint16_t* residual, void* stream);

/* The exact int32 accumulator acc[m,n] = sum_k q[m,k] t[n,k] of the same
 * kernels, without the rescale (for bit-exact verification).  Arguments as in
 * bitlinear_forward_quantized; acc is device int32 [M,N]. */
bl_status bitlinear_accumulate(const int8_t* q, const int32_t* rowsum, const uint8_t* P,
                               int64_t M, int64_t K, int64_t N, int32_t* acc, void* stream);

/* ---- the FFN block's gate/up pair in one pass ---------------------------- */

/* Workspace bitlinear_pack_gate_up needs for two [I,K] master weights. */
bl_status bitlinear_pack_gate_up_workspace_size(int64_t I, int64_t K, size_t* bytes);

/* The gate and up projections of an FFN block ([MD] model details: gated
 * ReLU^2 FFN) packed as one matrix: each ternarised with its own absmean
 * scale exactly as bitlinear_pack does, then packed as the concatenation
 * [gate; up] ([2I, K], the layout of bitlinear_pack).  With the block layout
 * ([BG] pack_weights, "推理侧 BitLinear") bit pairs 0 and 1 of packed row r
 * hold gate rows r and I/2 + r and bit pairs 2 and 3 the up rows with the
 * same indices, so one byte carries both operands of two outputs of
 * relu(gate)^2 * up.
 *   W_gate, W_up  device fp32 [I,K] master weights; I even.
 *   P2            device uint8 [I/2, K] output (bitlinear_pack_ternary of the
 *                 concatenated ternary matrices gives the same bytes).
 *   beta_out      device float[2] output: {beta_gate, beta_up}.
 *   workspace     device, >= bitlinear_pack_gate_up_workspace_size bytes. */
bl_status bitlinear_pack_gate_up(const float* W_gate, const float* W_up, int64_t I, int64_t K,
                                 uint8_t* P2, float* beta_out, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* The gate and up BitLinear projections of one quantised input and the gated
 * squared ReLU of the FFN block, in one pass over the pair's packed weights
 * ([BG] "推理侧 BitLinear" for each projection, [MD] model details for the
 * relu^2 gating):
 *   g = bf16(RN32(RN32(acc_gate * beta_gate) / s_x)),
 *   u = bf16(RN32(RN32(acc_up * beta_up) / s_x)),
 *   z[m, n] = bf16(RN32(RN32(relu(g) * relu(g)) * u)),  n < I,
 * bit for bit what bitlinear_forward_quantized of each projection followed by
 * bitlinear_relu2_mul gives, without writing g and u to memory.
 *   q, s_x, rowsum  as for bitlinear_forward_quantized (device).
 *   P2              device uint8 [I/2, K] from bitlinear_pack_gate_up.
 *   z               device bf16 [M, I] output.
 *   workspace       device or NULL: for 5 <= M <= 64, at least
 *                   bitlinear_quantized_batch_workspace_size(M) bytes give
 *                   every CTA an equal share of the weights (as for the
 *                   quantized batch); NULL cuts shares at row tiles. */
bl_status bitlinear_forward_gate_up(const int8_t* q, const float* s_x, const int32_t* rowsum,
                                    const uint8_t* P2, float beta_gate, float beta_up, int64_t M,
                                    int64_t K, int64_t I, uint16_t* z, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* ---- quantisation-aware training (online quantisation, STE backward) ---- */

/* Workspace bitlinear_forward_online needs: the absmean partial sums and, for
 * 5 <= M <= 64, the split-tile area of the 5..64-token kernel. */
bl_status bitlinear_forward_online_workspace_size(int64_t M, int64_t K, int64_t N,
                                                  size_t* bytes);

/* The training-time forward of a BitLinear whose weights are quantised on
 * every call ([BG] "量化器参数：BitNetQuantConfig 详解": AutoBitLinear with
 * quantization_mode "online"; [BG] "BitLinear 的三步量化" steps 1-3): the
 * absmean scale and the ternary weights come from the fp32 master weights on
 * this call, exactly as bitlinear_pack computes them, and the forward is the
 * inference forward on them (bit for bit bitlinear_pack followed by
 * bitlinear_forward).  All asynchronous: the scale stays on the device.
 *   x, gain, eps, y, y_dtype  as for bitlinear_forward (x may be NULL when M == 0).
 *   W        device fp32 [N,K] master weights.
 *   P        device uint8 [N/4,K] output: the packed ternary weights.
 *   beta     device float[1] output: the absmean scale (input of the backward).
 *   q, s_x, rowsum  device outputs [M,K] int8, [M] fp32, [M] int32: the
 *            quantised activations (inputs of the backward).
 *   workspace  device, >= bitlinear_forward_online_workspace_size bytes. */
bl_status bitlinear_forward_online(const uint16_t* x, const uint16_t* gain, float eps,
                                   const float* W, int64_t M, int64_t K, int64_t N, void* y,
                                   bl_out_dtype y_dtype, uint8_t* P, float* beta, int8_t* q,
                                   float* s_x, int32_t* rowsum, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* The backward of that layer under the straight-through estimator ([BG]
 * "BitLinear 的三步量化": both quantisers pass the gradient through unchanged),
 * i.e. the linear layer's backward on the dequantised operands:
 *   W_q[n,k] = RN32(t[n,k] / RN32(1/beta)),  x_q[m,k] = RN32(q[m,k] / s_x[m]),
 *   grad_x[m,k] = sum_n grad_y[m,n] W_q[n,k],
 *   grad_w[n,k] = sum_m grad_y[m,n] x_q[m,k]   (the master weights' gradient).
 * Sums in binary32, each product added with one fused multiply-add; the order
 * of the additions is not specified, so results agree with the exact sums to
 * within n * 2^-24 * sum |terms| (n = N for grad_x, M for grad_w).
 *   grad_y  device fp32 [M,N].
 *   q, s_x  device, from bitlinear_forward_online (needed for grad_w).
 *   P, beta device, from bitlinear_forward_online (needed for grad_x).
 *   grad_x  device fp32 [M,K] output, or NULL to skip it.
 *   grad_w  device fp32 [N,K] output, or NULL to skip it (not both NULL). */
bl_status bitlinear_backward_ste(const float* grad_y, const int8_t* q, const float* s_x,
                                 const uint8_t* P, const float* beta, int64_t M, int64_t K,
                                 int64_t N, float* grad_x, float* grad_w, void* stream);

/* ---- one token through a chain of dependent steps, in one launch -------- */

#define BL_MAX_CHAIN_STEPS 4096
#define BL_CHAIN_MAX_PROBLEMS 4

typedef enum { BL_CHAIN_BF16 = 0, BL_CHAIN_F32 = 1, BL_CHAIN_GATE_UP = 2 } bl_chain_kind;

/* One projection of a chain step (all pointers device; one token, M = 1). */
typedef struct {
    const uint8_t* P;          /* packed weights: [N/4, K], or [N/2, K] for a gate/up pair */
    void* y;                   /* [N] output: bf16 or fp32 per kind; bf16 z for a pair */
    const uint16_t* residual;  /* bf16 [N] added after the bf16 rounding, or NULL (bf16 only) */
    int64_t N;                 /* outputs (I for a gate/up pair from bitlinear_pack_gate_up) */
    float beta;                /* absmean scale (the gate's for a pair) */
    float beta_up;             /* the up projection's scale of a pair (else unused) */
    bl_chain_kind kind;
} bl_chain_problem;

/* One step: up to BL_CHAIN_MAX_PROBLEMS projections of one input row, each
 * exactly what bitlinear_forward (M = 1, with its RMSNorm), plus the residual
 * of bitlinear_forward_quantized or the relu^2 gating of
 * bitlinear_forward_gate_up, would compute. */
typedef struct {
    const uint16_t* x;         /* bf16 [K] input row (16-byte aligned) */
    const uint16_t* gain;      /* bf16 [K] RMSNorm weight or NULL */
    float eps;
    int64_t K;                 /* K % 16 == 0, K <= 8192 */
    int count;                 /* 1 .. BL_CHAIN_MAX_PROBLEMS */
    bl_chain_problem p[BL_CHAIN_MAX_PROBLEMS];
} bl_chain_step;

/* Workspace of a chain of nsteps steps (1 .. BL_MAX_CHAIN_STEPS). */
bl_status bitlinear_decode_chain_workspace_size(int nsteps, size_t* bytes);

/* Checks the steps and copies their description into the workspace (a
 * synchronous host-to-device copy; call it once, outside any stream capture).
 * The buffers the steps name must stay valid while the chain is run. */
bl_status bitlinear_decode_chain_prepare(const bl_chain_step* steps, int nsteps, void* workspace,
                                         size_t workspace_bytes);

/* Runs the prepared steps in order, for one token, in one persistent launch
 * ([BG] "推理侧 BitLinear" for each projection; [MD] model details for the
 * decoder layer's residual adds and gated relu^2 FFN): step s + 1 sees every
 * output of step s (a grid-wide barrier separates them), so a step may read
 * the previous steps' outputs as its input row or residual.  A step's input
 * row must not be written by that same step (use two residual buffers in
 * turn: the step that adds o to the residual stream reads x and writes a
 * second buffer).  Results are bit for bit those of the separate entry points.
 * Each CTA quantises a step's input itself and the weights of later steps
 * stream in while it waits at the barrier.  Needs every SM's CTA resident at
 * once (cooperative launch: BL_ERR_CUDA if the device cannot host it); the
 * barrier waits are bounded like every other wait (BL_ERR_TIMEOUT through
 * bitlinear_device_status).  Asynchronous on `stream`. */
bl_status bitlinear_decode_chain_run(void* workspace, size_t workspace_bytes, int nsteps,
                                     void* stream);

/* ---- forward without any caller-provided memory besides inputs and outputs -- */

/* Size of the library's fixed device scratch used by bitlinear_forward_noalloc. */
#define BL_NOALLOC_SCRATCH_BYTES (2u << 20)

/* Same computation and result as bitlinear_forward, for callers that cannot
 * allocate device memory: latency-critical loops that must not pay
 * cudaMalloc/cudaFree's implicit device synchronisation, and plugins embedded
 * in an engine that owns every allocation itself and hands them only their
 * inputs and outputs.  (The method's own pages have no counterpart; this is an
 * interface convenience.)
 *   Arguments as in bitlinear_forward, without the workspace.
 *   Scratch: instead of a caller workspace it uses one file-scope device array
 *   of BL_NOALLOC_SCRATCH_BYTES that every GPU which loads the library keeps
 *   until the process exits.  The first call on a device looks up that array's
 *   device address with a host-side runtime query.
 *   The array must hold the int8 codes, scales and row sums of the input
 *   (M*K bytes plus 8*M, each part rounded up to 256 bytes); larger shapes are
 *   rejected with BL_ERR_WORKSPACE before anything is launched, and
 *   bitlinear_last_error() names both sizes.  For 5 <= M <= 64, when the
 *   split-tile tail of bitlinear_forward_workspace_size does not fit beside
 *   the codes, the CTA shares are cut at row-tile boundaries instead (same
 *   results).
 *   All calls share the one array: calls that can overlap on the GPU (other
 *   streams, other host threads) race on it and must be serialised by the
 *   caller.  Nothing in it needs to start at zero: every byte a call reads was
 *   written earlier in the same call.
 *   Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
bl_status bitlinear_forward_noalloc(const uint16_t* x, const uint16_t* gain, float eps,
                                    const uint8_t* P, float beta, int64_t M, int64_t K,
                                    int64_t N, void* y, bl_out_dtype y_dtype, void* stream);

/* ---- FFN glue ([MD] model details: ReLU^2 FFN; [BG] ffn_sub_norm) ---------- */

/* z = bf16(RN32(RN32(relu(a) * relu(a)) * b)) elementwise over n values;
 * a = gate output, b = up output, all device bf16.  z may alias a or b. */
bl_status bitlinear_relu2_mul(const uint16_t* a, const uint16_t* b, int64_t n, uint16_t* z,
                              void* stream);

/* ---- attention block of the decoder layer (RoPE, GQA decode attention) ---- */

/* Rotary position embeddings ([MD] model details: the decoder uses RoPE;
 * BitNetConfig: 20 heads of 128 dimensions for q, 5 for k, 2048 positions).
 * The pages give no formula; the rotate-half form is used: for every head and
 * i < head_dim/2 the pair (x[i], x[i + head_dim/2]) is turned by the angle
 * a = pos[m] * theta^(-2i/head_dim):
 *   y[i]              = x[i] cos a - x[i + head_dim/2] sin a,
 *   y[i + head_dim/2] = x[i + head_dim/2] cos a + x[i] sin a,
 * each evaluated in binary64 and rounded once to bf16.
 *   x, y      device bf16 [M, heads * head_dim] (y may equal x: in place).
 *   pos       device int32 [M] token positions.
 *   theta     base of the frequencies (> 0, finite; rope_theta).
 * head_dim even and <= 1024; heads, M <= 65535. */
bl_status bitlinear_rope(const uint16_t* x, const int32_t* pos, int64_t M, int64_t heads,
                         int64_t head_dim, float theta, uint16_t* y, void* stream);

/* Workspace bitlinear_attn_decode needs for this shape (depends on the
 * current device's SM count). */
bl_status bitlinear_attn_decode_workspace_size(int64_t L, int64_t q_heads, int64_t kv_heads,
                                               int64_t head_dim, size_t* bytes);

/* Grouped-query attention of one decode token over its key/value cache ([MD]
 * BitNetConfig: num_attention_heads 20, num_key_value_heads 5 -- each
 * key/value head serves a group of query heads; model details: the layer
 * order q, k, v -> RoPE + attention -> attn_sub_norm -> o).  The pages give
 * no formula; the textbook one is used: query head h reads key/value head
 * g = h / (q_heads / kv_heads) and
 *   out[h] = sum_j p_j v[j, g],  p = softmax_j((q[h] . k[j, g]) * scale),
 * over the L cached positions (the current token's key and value included).
 * Arithmetic in binary32 (exp2 of log2-scaled scores, split over the cache
 * and merged), output rounded to bf16; it matches the exact value within a
 * stated tolerance, not bit for bit.
 *   q         device bf16 [q_heads * head_dim] (after RoPE).
 *   k_cache   device bf16 [>= L, kv_heads, head_dim], 16-byte aligned
 *             (positions past L are not read).
 *   v_cache   device bf16 [>= L, kv_heads, head_dim], 16-byte aligned.
 *   scale     score multiplier (1/sqrt(head_dim) in the model).
 *   out       device bf16 [q_heads * head_dim].
 *   workspace device, 16-byte aligned, at least
 *             bitlinear_attn_decode_workspace_size bytes.
 * head_dim 64 or 128; q_heads / kv_heads in {1, 2, 4, 8}; L >= 1. */
bl_status bitlinear_attn_decode(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                                int64_t L, int64_t q_heads, int64_t kv_heads, int64_t head_dim,
                                float scale, uint16_t* out, void* workspace, size_t workspace_bytes,
                                void* stream);

/* ---- device status -------------------------------------------------------- */

/* Synchronises `stream`, then returns and clears the library's device status
 * word on the current device: BL_OK, or BL_ERR_TIMEOUT if a kernel gave up on a
 * bounded wait since the last call. */
bl_status bitlinear_device_status(void* stream);

/* Failure-detection self-test (diagnostics; the pages have no counterpart).
 * Launches one CTA that waits on a shared-memory barrier nothing arrives on,
 * with a wait limit of limit_ns (clamped to 1 us .. 10 s) instead of the
 * kernels' 2 s: the wait runs out, records the timeout in the device status
 * word and the kernel returns, as every bounded wait of the library does.  The
 * next bitlinear_device_status() returns BL_ERR_TIMEOUT and clears the word;
 * the context stays usable.  Asynchronous on `stream`. */
bl_status bitlinear_selftest_wait_timeout(int64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H */
