/*
 * qgemv.h -- C ABI of libqgemv: weight-only quantized GEMV for LLM decode on
 * NVIDIA B200 (sm_100a).
 *
 * The operation, as the pages describe it: single-token decode reads every
 * decoder weight once per token and is bound by memory bandwidth ("Qwen3-VL 4B
 * -- Core AI (.aimodel)", section Measured: the int8hu decoder reads its whole
 * size per token).  The shipped format is an int8 per-block-32 symmetric body
 * and an absmax int8 LM head ("Qwen3-VL (2B / 4B / 8B, vision-language) --
 * Core AI", Measured table), with an INT4 group-64 variant ("Qwen3-VL 4B & 8B
 * -- Core ML stateful", Architecture) and a 16-token chunked-prefill function
 * beside the one-token step ("Qwen3.8-27B ... -- Core AI", The vision path).
 *
 * Conventions for every call below
 *   - Weights are row-major [n, k] (rows = outputs, k = the reduction axis,
 *     Linear.weight order); quantization blocks run along k.
 *   - fp16 values travel as their IEEE binary16 bit patterns (uint16_t).
 *   - Every pointer argument except `W` / `Wg` / `Wu` (host pointers to a
 *     qg_weight the call reads before returning) is DEVICE memory owned by the
 *     caller.  The library allocates nothing.
 *   - Calls validate their arguments synchronously, on the host, before any
 *     launch; on an error nothing is enqueued.  On success the work is
 *     enqueued on `stream` and the call returns at once (asynchronous).
 *   - Buffer rows are contiguous: row r of codes starts at r*k bytes (int8) or
 *     r*k/2 bytes (int4), row r of scales/biases at r*(k/32) or r*(k/64)
 *     elements.  A row range of a larger matrix is a valid weight on its own.
 *   - Outputs are unspecified after an error.  Non-finite inputs (NaN/Inf in
 *     weights or activations) give unspecified results.
 */
#ifndef QGEMV_H
#define QGEMV_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define QG_API __attribute__((visibility("default")))
#else
#define QG_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QG_OK = 0,
    QG_ERR_NULL = 1,      /* a required pointer is NULL */
    QG_ERR_SHAPE = 2,     /* n < 1, k < 1, k not a multiple of the block, S out of range */
    QG_ERR_ALIGN = 3,     /* a pointer is not aligned as documented */
    QG_ERR_FORMAT = 4,    /* unknown format, or gate/up weights that disagree */
    QG_ERR_WORKSPACE = 5, /* workspace NULL or smaller than required */
    QG_ERR_CUDA = 6,      /* a CUDA runtime call or launch failed */
    QG_ERR_TIMEOUT = 7,   /* a device-side bounded wait expired (see qg_stream_check) */
    QG_ERR_PLAN = 8       /* qg_sweep_run found no plan of that many stages in its
                             workspace (reported by qg_stream_check) */
} qg_status;

typedef enum {
    /* int8 codes, one fp16 scale per 32 consecutive k:  w ~= q * s */
    QG_FMT_I8_B32 = 0,
    /* int4 codes (two per byte, even k in the low nibble), one fp16 scale and
     * one fp16 bias per 64 consecutive k:  w ~= q * s + b */
    QG_FMT_I4_G64 = 1,
    /* plain fp16 weights, no scales: the tied fp16 LM head of the pages'
     * "int8lin" bundle ("Qwen3-VL (2B / 4B / 8B, vision-language) -- Core AI",
     * Measured table: 2B int8lin, tied fp16 head, 2.0 GB), where the head is
     * the fp16 embedding table itself.  Accepted by qg_gemv_s1 (and
     * qg_gemm_s16 with S == 1) and qg_head_argmax; QG_ERR_FORMAT elsewhere. */
    QG_FMT_F16 = 2
} qg_format;

/* A quantized weight matrix [n, k].
 *   fmt    : a qg_format value.
 *   codes  : QG_FMT_I8_B32: int8 [n, k]; QG_FMT_I4_G64: uint8 [n, k/2];
 *            QG_FMT_F16: fp16 [n, k].  16-byte aligned.  k % 32 == 0
 *            (int8), k % 64 == 0 (int4) or k % 8 == 0 (fp16).
 *   scales : fp16 [n, k/32] (int8) or [n, k/64] (int4); 16-byte aligned;
 *            ignored for fp16 weights.
 *   biases : fp16 [n, k/64] for int4, 16-byte aligned; ignored otherwise. */
typedef struct {
    int32_t fmt;
    int32_t reserved;
    int64_t n;
    int64_t k;
    const void* codes;
    const uint16_t* scales;
    const uint16_t* biases;
} qg_weight;

/* ---------------------------------------------------------------------------
 * qg_quantize_block32 -- int8 per-block-32 symmetric absmax quantization
 * ("Qwen3-VL 4B -- Core AI (.aimodel)", Files: int8 per-block-32 body +
 * absmax int8 head; "Qwen3.8-27B ... -- Core AI", Verified: the absmax
 * symmetric per-block-32 rule, no clipping).
 * For each row and each block of 32 consecutive k:
 *   s = fp16_rne( absmax_fp32 / 127 )          (IEEE fp32 division)
 *   q = clamp( round_half_even( w / float(s) ), -127, 127 ), all q = 0 if s == 0
 * w      : fp32 [n, k], 16-byte aligned.      k % 32 == 0, n >= 1.
 * codes  : int8 [n, k] out, 16-byte aligned.
 * scales : fp16 [n, k/32] out, 2-byte aligned.
 * Bit-exact with the CPU oracle.  Blocks with absmax/127 above the fp16
 * range give an Inf scale (unspecified codes).
 * ------------------------------------------------------------------------- */
QG_API qg_status qg_quantize_block32(const float* w, int64_t n, int64_t k,
                              int8_t* codes, uint16_t* scales,
                              cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * qg_quantize_int4_g64 -- int4 group-64 affine quantization ("Qwen3-VL 4B &
 * 8B -- Core ML stateful", Architecture: INT4 per-grouped-channel, group size
 * 64).  The pages name no formula; this is the plain affine reading:
 *   s = fp16_rne( (max - min) / 15 ),  b = fp16_rne( min )   (fp32 ops)
 *   q = clamp( round_half_even( (w - float(b)) / float(s) ), 0, 15 ),
 *   all q = 0 if s == 0
 * w       : fp32 [n, k], 16-byte aligned.    k % 64 == 0, n >= 1.
 * codes   : uint8 [n, k/2] out (low nibble = even k), 16-byte aligned.
 * scales, biases : fp16 [n, k/64] out, 2-byte aligned.
 * Bit-exact with the CPU oracle.
 * ------------------------------------------------------------------------- */
QG_API qg_status qg_quantize_int4_g64(const float* w, int64_t n, int64_t k,
                               uint8_t* codes, uint16_t* scales,
                               uint16_t* biases, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * qg_gemv_s1 -- one-token (S=1) quantized GEMV, the decode weight stream
 * ("Qwen3-VL 4B -- Core AI (.aimodel)", Measured: decode is bandwidth-bound).
 *   y[r] = sum_k w_dq[r, k] * x[k]     (fp32 accumulation)
 * W   : the weight (int8 block-32, int4 group-64 or plain fp16).
 * x   : fp16 [k], 16-byte aligned.
 * y   : fp32 [n] out (4-byte aligned), or NULL.
 * y16 : fp16 [n] out = fp16_rne(y) (2-byte aligned), or NULL.
 * At least one of y, y16 must be non-NULL.  x must not overlap the outputs.
 * Accuracy: |y - y_ref| <= 2e-3 * sum_k |w_dq x| per row (fp64 oracle).
 * ------------------------------------------------------------------------- */
QG_API qg_status qg_gemv_s1(const qg_weight* W, const uint16_t* x, float* y,
                     uint16_t* y16, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * qg_gemm_s16 -- chunked-prefill skinny GEMM on the tensor cores, S tokens
 * through the same weights ("Qwen3.8-27B ... -- Core AI", The vision path:
 * a static S=16 'prefill' chunk beside the S=1 'main' decode).
 *   Y[s, r] = sum_k X[s, k] * w_dq[r, k],   0 <= s < S
 * W : the weight, int8 block-32 or int4 group-64 (QG_ERR_FORMAT for fp16
 *     weights at S > 1).  For S > 1, k % 512 == 0 (QG_ERR_SHAPE otherwise);
 *     S == 1 runs qg_gemv_s1.  For S > 1 each weight enters the tensor cores
 *     (tcgen05.mma, fp32 accumulation) as fp16(q * s) (int8) or
 *     fp16(q * s + b) (int4), one rounding each.
 * X : fp16 [S, k] row-major, 16-byte aligned.   1 <= S <= 16.
 * Y : fp32 [S, n] out, 4-byte aligned.
 * Accuracy: each row s obeys the qg_gemv_s1 bound for x = X[s].
 * ------------------------------------------------------------------------- */
QG_API qg_status qg_gemm_s16(const qg_weight* W, const uint16_t* X, int S, float* Y,
                      cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * qg_gate_up_swiglu -- fused gate/up projections with the SwiGLU epilogue
 * ("Qwen3-VL (2B / 4B / 8B, vision-language) -- Core AI", architecture: a
 * SwiGLU MLP):
 *   g = W_g x,  u = W_u x,  H[s, i] = fp16_rne( silu(g_i) * u_i ),
 *   silu(g) = g / (1 + exp(-g))
 * Wg, Wu : weights of identical format and shape [n = intermediate, k],
 *          int8 or int4 (fp16 weights: QG_ERR_FORMAT); S > 1 (tensor cores)
 *          needs k % 512 == 0.
 * X      : fp16 [S, k], 16-byte aligned.   1 <= S <= 16.
 * H      : fp16 [S, n] out, 2-byte aligned.
 * ------------------------------------------------------------------------- */
QG_API qg_status qg_gate_up_swiglu(const qg_weight* Wg, const qg_weight* Wu,
                            const uint16_t* X, int S, uint16_t* H,
                            cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * qg_head_argmax -- LM head GEMV fused with the greedy argmax
 * ("Qwen3.8-27B ... -- Core AI", Verified: absmax int8 head, greedy
 * teacher-forced argmax).
 *   logits[v] = sum_k w_dq[v, k] x[k];   idx = the smallest v of the max
 * W         : the head weight [vocab, hidden] (int8, int4, or the tied fp16
 *             embedding table itself).
 * x         : fp16 [k], 16-byte aligned.
 * logits    : fp32 [n] out (4-byte aligned) or NULL.
 * idx       : int32 [1] out, device memory.
 * workspace : device memory of at least qg_head_argmax_workspace_bytes(n)
 *             bytes, 16-byte aligned.  It must be all zero before its first
 *             use; every call that returns QG_OK and runs to completion
 *             leaves it all zero again, so it can be reused without clearing.
 *             Calls that share a workspace must not overlap on the GPU.
 * ------------------------------------------------------------------------- */
QG_API size_t qg_head_argmax_workspace_bytes(int64_t n);
QG_API qg_status qg_head_argmax(const qg_weight* W, const uint16_t* x, float* logits,
                         int32_t* idx, void* workspace, size_t ws_bytes,
                         cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * qg_head_argmax_noalloc -- qg_head_argmax for callers that cannot allocate
 * device memory.  The pages have no counterpart to this call; it exists for
 * callers that cannot provide a workspace: a plugin or custom operator whose
 * host framework owns and budgets every device allocation, or a
 * latency-critical loop where a device allocation is not acceptable.
 * Same arguments, results and accuracy as qg_head_argmax, minus the workspace:
 * the reduction scratch is a 256-byte array inside the library that every GPU
 * loading the library keeps until the process exits.  The call allocates
 * nothing (no cudaMalloc, no cudaFree, no allocating library routine).
 *   - Every call whose stream is not being captured looks up that array's
 *     device address (cudaGetSymbolAddress, with the device current), so a
 *     call after cudaDeviceReset finds the reloaded array.  A call made
 *     while `stream` is being captured into a CUDA graph uses the address
 *     of the last uncaptured call on the device: make one uncaptured call
 *     first (a first call during capture returns QG_ERR_CUDA), and capture
 *     again after a device reset.
 *   - Each call clears the scratch on `stream` before the kernel runs (an
 *     asynchronous memset of 256 bytes), because the array keeps what the
 *     previous call left there.
 *   - All calls on a device share the one array: calls that overlap on the
 *     GPU (different streams without ordering between them) race and give
 *     wrong indices.  Serialize them.
 *   - A weight whose argmax would need more scratch than the 256 bytes is
 *     refused with QG_ERR_WORKSPACE.  Today qg_head_argmax_workspace_bytes
 *     reports 256 bytes for every n (of which the kernel uses 16), so the
 *     refusal only guards future layouts that need more.
 * ------------------------------------------------------------------------- */
QG_API qg_status qg_head_argmax_noalloc(const qg_weight* W, const uint16_t* x, float* logits,
                                        int32_t* idx, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * The rest of a decode step around the weight stream, attention excluded:
 * the embedding row of the chosen token and a decoder layer's pre-norm
 * RMSNorm and residual adds, fused into the S=1 calls so that a chain of
 * calls carries a real fp32 hidden state h from token to token.  The pages'
 * engines gather fp16 embedding rows ("Qwen3.8-27B ... -- Core AI", The
 * vision path: the host gathers text rows from the shipped fp16 embedding
 * table); the norm belongs to the Qwen3-architecture decoders the pages
 * port and is not spelled out there.
 *   RMSNorm:  x[i] = fp16_rne( h[i] * gamma[i] / sqrt(sum_j h[j]^2 / k + eps) )
 *             computed in fp32 inside every CTA that reads x (a fixed-order
 *             reduction: results are deterministic).
 * qg_embedding_gather       h[i] = table[*token][i] (fp16 -> fp32, exact).
 *   table : fp16 [V, H], 2-byte aligned.  token : device int32 [1]; a value
 *           outside [0, V) writes nothing and qg_stream_check reports
 *           QG_ERR_SHAPE.  h : fp32 [H] out, 4-byte aligned.
 * qg_rmsnorm_gemv_s1        qg_gemv_s1 with x = RMSNorm(h; gamma, eps).
 * qg_rmsnorm_gate_up_swiglu qg_gate_up_swiglu (S = 1) with x = RMSNorm(h).
 * qg_rmsnorm_head_argmax    qg_head_argmax with x = RMSNorm(h).
 * qg_gemv_s1_residual       h[r] += (W x)[r] for every row r (the o and down
 *                           projections adding into the residual stream);
 *                           x must not overlap h.
 *   h : fp32 [k] (the normed calls) or [n] (the residual call); gamma :
 *       fp16 [k]; both 16-byte aligned.  0 <= eps <= 1 (QG_ERR_SHAPE).
 * Accuracy: the device computes x in fp32 and rounds it to fp16, so x is
 * within one fp16 ulp of the fp64 RMSNorm rounded to fp16; given that x (see
 * qg_rmsnorm_f16), the outputs obey the plain calls' bound
 * |y - y_ref(x)| <= 2e-3 sum_k |w_dq x|.
 * ------------------------------------------------------------------------- */
QG_API qg_status qg_embedding_gather(const uint16_t* table, int64_t V, int64_t H,
                                     const int32_t* token, float* h, cudaStream_t stream);
QG_API qg_status qg_rmsnorm_gemv_s1(const qg_weight* W, const float* h, const uint16_t* gamma,
                                    float eps, float* y, uint16_t* y16, cudaStream_t stream);
QG_API qg_status qg_rmsnorm_gate_up_swiglu(const qg_weight* Wg, const qg_weight* Wu,
                                           const float* h, const uint16_t* gamma, float eps,
                                           uint16_t* H, cudaStream_t stream);
QG_API qg_status qg_rmsnorm_head_argmax(const qg_weight* W, const float* h,
                                        const uint16_t* gamma, float eps, float* logits,
                                        int32_t* idx, void* workspace, size_t ws_bytes,
                                        cudaStream_t stream);
QG_API qg_status qg_gemv_s1_residual(const qg_weight* W, const uint16_t* x, float* h,
                                     cudaStream_t stream);

/* qg_rmsnorm_f16 -- x16 = fp16_rne(RMSNorm(h; gamma, eps)) for h fp32 [k],
 * computed exactly as the RMSNorm-input calls above stage their x (the same
 * fixed-order reduction and per-element arithmetic), so a caller can see the
 * activation those calls multiply by.  h, gamma, x16 16-byte aligned (x16
 * fp16 [k] out); k % 8 == 0; 0 <= eps <= 1 (QG_ERR_SHAPE otherwise). */
QG_API qg_status qg_rmsnorm_f16(const float* h, const uint16_t* gamma, int64_t k, float eps,
                                uint16_t* x16, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * qg_decode_attention -- the attention core of one decode step over an fp16
 * K/V cache, for the pages' Qwen3-VL decoders ("Qwen3-VL (2B / 4B / 8B,
 * vision-language) -- Core AI", architecture paragraph: pure attention,
 * head_dim 128, 8 kv heads, rope theta 5e6; "Qwen3-VL 4B & 8B -- Core ML
 * stateful", gotchas: for text positions the interleaved M-RoPE is standard
 * 1-D RoPE with the two halves of a head paired; "Qwen3-VL 2B -- Core AI",
 * integration checklist: the KV cache is the native K/V pair).  Readings
 * where the pages are silent: no per-head q/k norm, scale 1/sqrt(d).
 *   RoPE(x, p)[i]       = x[i] cos(p f_i) - x[i+d/2] sin(p f_i)
 *   RoPE(x, p)[i + d/2] = x[i+d/2] cos(p f_i) + x[i] sin(p f_i),  f_i = theta^(-2i/d)
 *   the token at position p = *pos appends K[g][p] = fp16_rne(RoPE(k_g, p)),
 *   V[g][p] = fp16_rne(v_g), then for every query head h (kv head g = h/(hq/hkv))
 *   o_h = fp16_rne( sum_{j <= p} softmax_j( RoPE(q_h, p) . K[g][j] / sqrt(d) ) V[g][j] )
 * qkv    : fp32 [hq*d | hkv*d | hkv*d], the q|k|v projection's output, 16-byte
 *          aligned.
 * kcache, vcache : fp16 [hkv][l_max][d], 16-byte aligned; rows 0..p-1 hold the
 *          earlier tokens (rotated keys), row p is written by this call.
 * pos    : device int32 [1]; outside [0, l_max) the call writes nothing and
 *          qg_stream_check reports QG_ERR_SHAPE.
 * o      : fp16 [hq*d] out, 16-byte aligned (the o projection's input).
 * d == 128 and hq / hkv in {1, 2, 4} (QG_ERR_SHAPE otherwise); theta > 0.
 * workspace : device memory of at least qg_decode_attention_workspace_bytes,
 *          256-byte aligned, ZEROED ONCE before first use.  Its first 256
 *          bytes hold per-kv-head counters that every call leaves zeroed again;
 *          the rest is scratch for the split partials.  Calls sharing one
 *          workspace must be serialized.
 * Accuracy: |o - o_ref| <= 1e-3 * sum_j p_j |V[g][j]| + ulp_f16(o_ref) per
 * element, o_ref the fp64 attention on the same fp16 cache.  Deterministic.
 * The kernel's waits on its own copies are bounded; one that expires makes
 * qg_stream_check report QG_ERR_TIMEOUT (o is then undefined).
 * ------------------------------------------------------------------------- */
QG_API size_t qg_decode_attention_workspace_bytes(int hq, int hkv);
QG_API qg_status qg_decode_attention(const float* qkv, int hq, int hkv, int d,
                                     uint16_t* kcache, uint16_t* vcache, int64_t l_max,
                                     const int32_t* pos, double theta, uint16_t* o,
                                     void* workspace, size_t ws_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * qg_sweep_* -- a whole one-token decode step as ONE persistent launch.
 * A decode step reads every decoder weight once ("Qwen3-VL 4B -- Core AI
 * (.aimodel)", Measured), as an ordered chain of S=1 projections per layer
 * (qkv -> o -> gate/up + SwiGLU -> down) and the LM head with the greedy
 * argmax ("Qwen3.8-27B ... -- Core AI", The vision path: prefill runs as
 * pipelined S=1 steps).  A sweep is that chain: an ordered list of stages,
 * each one of the S=1 calls above with the same arguments and accuracy.  An
 * all-int8 plan whose rows hold whole 512-code steps and fit a 32 KB ring
 * slot (k <= 32768 per weight, a SwiGLU stage's two weights together)
 * runs on the stream kernel: one CTA per SM, results within the same bound
 * as the calls and identical from run to run, each row summed in its own
 * fixed order (not the calls' order).  Other plans run on the general
 * persistent kernels (two CTAs per SM), whose results are bit-identical to
 * the calls.
 *
 * Order: stage i + 1 reads its x only after every part of stage i is done,
 * exactly as if the calls were enqueued one after another on one stream, so
 * a stage may read what an earlier stage wrote.  What the single launch adds
 * is that the WEIGHTS of stage i + 1 (which no stage writes) start streaming
 * while the GPU waits for the last parts of stage i, and no launch gaps.
 *
 *   op     : QG_STAGE_GEMV        y = W x  (y and/or y16, as qg_gemv_s1)
 *            QG_STAGE_SWIGLU      h = fp16(silu(W x) * (w_up x))
 *                                 (as qg_gate_up_swiglu with S = 1)
 *            QG_STAGE_HEAD_ARGMAX logits = W x (optional), idx = argmax
 *                                 (as qg_head_argmax; the workspace is part
 *                                 of the sweep's)
 *   w      : the weight (the gate weight for QG_STAGE_SWIGLU), a copy.
 *   w_up   : QG_STAGE_SWIGLU only: the up weight (same format and shape).
 *   x      : fp16 [k], 16-byte aligned, device.
 *   y, y16 : QG_STAGE_GEMV outputs (at least one), as qg_gemv_s1.
 *   h      : QG_STAGE_SWIGLU output fp16 [n], 2-byte aligned.
 *   logits, idx : QG_STAGE_HEAD_ARGMAX outputs, as qg_head_argmax.
 * Unused pointers must be NULL.  Every pointer stays owned by the caller and
 * must stay valid while a run that uses the plan can execute.
 *
 * Formats: a plan is either all int8, or the int4 run's layout -- every
 *   GEMV and SwiGLU stage int4 and every head int8 (the pages pair an int4
 *   body with an absmax int8 head); other mixes, and fp16 weights, give
 *   QG_ERR_FORMAT.
 *
 * qg_sweep_workspace_bytes(n) -- device bytes a plan of n stages needs.
 * qg_sweep_plan -- validates every stage (the same checks, with the same
 *   status codes, as the single calls; QG_ERR_FORMAT for an unknown op or a
 *   format mix above; QG_ERR_SHAPE if a stage's rows do not hold a multiple
 *   of 8 scales, i.e. k % 256 (int8) or k % 512 (int4), or its x does not
 *   fit the launch's shared memory, k <= 17408 for every shape the pages
 *   use), writes the plan into `workspace` (device memory, 256-byte aligned,
 *   at least qg_sweep_workspace_bytes(n) bytes) with a synchronous
 *   host-to-device copy, and fills `*sweep` (host memory owned by the
 *   caller), which qg_sweep_run reads.  Call it outside stream capture, and
 *   never while a run that uses the same workspace may still execute.
 *   1 <= n_stages <= 65536.
 * qg_sweep_run -- enqueues one run of the plan on `stream` (asynchronous;
 *   safe to capture in a CUDA graph).  It is a cooperative launch (one or
 *   two CTAs per SM, as above) whose CTAs must all be resident at once: it
 *   fails with
 *   QG_ERR_CUDA if the device cannot host them, and runs must not overlap
 *   other runs of the same workspace.  Between stages the CTAs wait on
 *   counters in the workspace; a wait that has not finished after ~2 s gives
 *   up, and qg_stream_check then reports QG_ERR_TIMEOUT; a workspace that
 *   does not hold the plan `sweep` describes is reported as QG_ERR_PLAN.  After either
 *   error, plan the workspace again before the next run.  Every run that
 *   completes leaves the counters zero for the next one.
 * ------------------------------------------------------------------------- */
typedef enum {
    QG_STAGE_GEMV = 0,
    QG_STAGE_SWIGLU = 1,
    QG_STAGE_HEAD_ARGMAX = 2
} qg_stage_op;

typedef struct {
    int32_t op;
    int32_t reserved;
    qg_weight w;
    qg_weight w_up;
    const uint16_t* x;
    float* y;
    uint16_t* y16;
    uint16_t* h;
    float* logits;
    int32_t* idx;
} qg_stage;

/* What qg_sweep_run needs to know about a plan on the host. */
typedef struct {
    int32_t n_stages; /* stages in the plan */
    int32_t kernel;   /* the persistent kernel that runs it: 0 int8, 1 int4 */
    int64_t reserved[3];
} qg_sweep;

QG_API size_t qg_sweep_workspace_bytes(int n_stages);
QG_API qg_status qg_sweep_plan(const qg_stage* stages, int n_stages, void* workspace,
                               size_t ws_bytes, qg_sweep* sweep);
QG_API qg_status qg_sweep_run(const qg_sweep* sweep, void* workspace, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * qg_stream_check -- synchronize `stream` and report asynchronous failures:
 * QG_ERR_CUDA for a CUDA error, QG_ERR_PLAN if a sweep ran on a workspace
 * without its plan, QG_ERR_SHAPE if an embedding gather met a token id out
 * of range, QG_ERR_TIMEOUT if a kernel's bounded wait (on its own
 * copies, or a sweep's wait between stages) expired since the last check
 * (the flags are then cleared).  Kernels never spin without a limit.
 * ------------------------------------------------------------------------- */
QG_API qg_status qg_stream_check(cudaStream_t stream);

/* Human-readable name of a status code (static string). */
QG_API const char* qg_status_string(qg_status status);

/* Name of the CUDA error behind the calling thread's most recent QG_ERR_CUDA
 * ("cudaSuccess" if there was none); a static string. */
QG_API const char* qg_last_cuda_error(void);

/* ABI version of this header (major * 100 + minor). */
QG_API int qg_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QGEMV_H */
