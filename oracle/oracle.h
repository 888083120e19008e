/*
 * oracle.h -- CPU oracle for weight-only quantized decode.
 *
 * TEST INFRASTRUCTURE ONLY.  This code is the correctness reference for the
 * CUDA library in int4_quantized_decode_b200/.  Only tests/, the smoke check in
 * __graft_entry__.py and the CPU-baseline leg of bench.py may load or call it.
 * The product path never routes through it, and it shares no code, header,
 * table or constant with the CUDA sources.
 *
 * What it computes is the plain definition of the method: quantize each weight
 * exactly as specified, dequantize to fp64, and take an fp64 dot product per
 * output row, followed by the SwiGLU and argmax epilogues.  No blocking, fusion
 * or reordering: every sum runs in index order.
 *
 * Sources (web pages on int8/int4 weight-only decode for Qwen3-VL / Qwen3.8):
 *   [HF4B]  "Qwen3-VL 4B -- Core AI (.aimodel)", sections "Files" (SHIP: int8
 *           per-block-32 body + untied absmax int8 head) and "Measured"
 *           (decode is bandwidth-bound, reads ~4.7 GB/token).
 *   [ZOO]   "Qwen3-VL (2B / 4B / 8B, vision-language) -- Core AI", architecture
 *           paragraph (vocab 151 936, SwiGLU) and the "Measured" table
 *           (int8lin per-block-32 body + untied absmax int8 head).
 *   [Q27]   "Qwen3.8-27B (VLM: text decoder + vision path) -- Core AI", section
 *           "Verified" (absmax symmetric per-block-32 head rule, no clipping;
 *           teacher-forced argmax with a margin rule) and "The vision path"
 *           (S=1 'main' vs S=16 'prefill' chunk).
 *   [ANE]   "Qwen3-VL 4B & 8B -- Core ML stateful (text + vision)", section
 *           "Architecture (vs 2B)" (INT4 per-grouped-channel, group size 64).
 *
 * Parity pins: every function here is pinned in tests/test_oracle_pins.py
 * against something other than itself (IEEE library conversions, exact
 * rational arithmetic, brute-force nearest-code search, closed forms and the
 * bundle sizes the pages print).  Nothing here is "parity unpinned".
 */
#ifndef QG_ORACLE_H
#define QG_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* IEEE-754 binary32 -> binary16, round to nearest, ties to even; subnormals
 * kept, overflow to +-Inf, NaN stays NaN.  Written from the IEEE definition. */
uint16_t orc_f32_to_f16(float f);
/* Exact binary16 -> binary64 / binary32. */
double orc_f16_to_f64(uint16_t h);
float orc_f16_to_f32(uint16_t h);
/* Round a float to the nearest integer, ties to even (exact, in fp64). */
double orc_rint_half_even(float r);

/* int8 per-block-32 symmetric absmax ("int8hu" body and head, [HF4B] Files,
 * [ZOO] Measured, [Q27] Verified).  w: fp32 [n,k] row-major, k % 32 == 0.
 * Out: codes int8 [n,k], scales fp16 bits [n,k/32].  Rows run in parallel
 * (OpenMP); the arithmetic inside a row is sequential fp32 IEEE. */
void orc_quantize_block32(const float* w, int64_t n, int64_t k,
                          int8_t* codes, uint16_t* scales);

/* int4 group-64 affine ([ANE] Architecture).  k % 64 == 0.  Out: codes
 * u8 [n,k/2] (low nibble = even k), scale and bias fp16 bits [n,k/64]. */
void orc_quantize_int4_g64(const float* w, int64_t n, int64_t k,
                           uint8_t* codes, uint16_t* scales, uint16_t* biases);

/* Dequantize row r to fp64: w_dq = q*s (int8) or q*s + b (int4). */
void orc_dequant_row_i8(const int8_t* codes, const uint16_t* scales, int64_t k,
                        int64_t r, double* out);
void orc_dequant_row_i4(const uint8_t* codes, const uint16_t* scales,
                        const uint16_t* biases, int64_t k, int64_t r, double* out);

/* fp64 dequantize-then-matvec over all n rows:
 *   y[r]   = sum_k w_dq[r,k] * x[k]       (index order, fp64)
 *   mag[r] = sum_k |w_dq[r,k] * x[k]|     (for the error bound)
 * x is fp16 bits [k].  fmt: 0 = int8 block-32, 1 = int4 group-64
 * (biases ignored for fmt 0), 2 = plain fp16 weights (codes are fp16 bits
 * [n,k], w_dq is their exact value; scales and biases ignored): the tied
 * fp16 head of the pages' "int8lin" bundle ("Qwen3-VL (2B / 4B / 8B) --
 * Core AI", Measured table: 2B int8lin with a tied fp16 head, 2.0 GB).
 * Either output may be NULL. */
void orc_matvec(int fmt, const void* codes, const uint16_t* scales,
                const uint16_t* biases, int64_t n, int64_t k,
                const uint16_t* x, double* y, double* mag);

/* fp64 -> fp16 bits, IEEE-754 binary16 round-to-nearest-even from the
 * definition (one rounding of the fp64 value; subnormals kept, overflow ->
 * +-Inf). */
uint16_t orc_f64_to_f16(double d);

/* The decoder's pre-norm RMSNorm of the fp32 residual stream, which feeds
 * q|k|v, gate/up and the head (the pages' decoders are Qwen3-architecture
 * models; the norm itself is not spelled out on the pages):
 *   rms  = sqrt( sum_i h[i]^2 / k + eps )          (fp64, index order)
 *   x[i] = fp16_rne( h[i] * gamma[i] / rms )       (fp64, one rounding)
 * h fp32 [k], gamma fp16 bits [k]; out x fp16 bits [k], and optionally the
 * fp64 values before the rounding (x_exact, or NULL). */
void orc_rmsnorm(const float* h, const uint16_t* gamma, int64_t k, double eps,
                 uint16_t* x, double* x_exact);

/* silu(g) = g / (1 + exp(-g)) and its derivative, fp64. */
double orc_silu(double g);
double orc_silu_grad(double g);

/* SwiGLU epilogue on fp64 gate/up outputs: h[i] = silu(g[i]) * u[i], and the
 * per-element bound
 *   e = tol * (|silu'(g)| * mag_g * |u| + |silu(g)| * mag_u),
 *   bound = e + ulp_f16(|h| + e) / 2
 * (the second term is the final rounding of h to fp16). */
void orc_swiglu(const double* g, const double* u, const double* mag_g,
                const double* mag_u, int64_t n, double tol, double* h,
                double* bound);

/* Spacing of binary16 numbers at magnitude v (2^-24 below the normal range). */
double orc_ulp_f16(double v);

/* Greedy argmax: the smallest index holding the largest value. */
int64_t orc_argmax(const double* v, int64_t n);

/* ------------------------------------------------------ decode attention ---
 * The attention core of one decode step of the pages' Qwen3-VL decoders
 * ("Qwen3-VL (2B / 4B / 8B, vision-language) -- Core AI", architecture
 * paragraph: pure attention, head_dim 128, 8 kv heads, rope theta 5e6;
 * "Qwen3-VL 4B & 8B -- Core ML stateful", gotchas: for text positions the
 * interleaved M-RoPE is exactly standard 1-D RoPE, and the rotary helper
 * pairs the two halves of a head; "Qwen3-VL 2B -- Core AI", integration
 * checklist: the KV cache is the engine's native K/V pair).  Readings where
 * the pages are silent: no per-head q/k norm, softmax scale 1/sqrt(d).
 *
 * RoPE of one head x[d] at position pos (rotate-half pairing, fp64):
 *   f_i = theta^(-2i/d),  a = pos * f_i,  for i < d/2:
 *   out[i]       = x[i] cos a - x[i+d/2] sin a
 *   out[i+d/2]   = x[i+d/2] cos a + x[i] sin a */
void orc_rope(const double* x, int64_t d, int64_t pos, double theta, double* out);

/* One decode step's attention for the token at position pos:
 *   qkv    fp32 [hq*d | hkv*d | hkv*d]: q, k, v of the token (the q|k|v
 *          projection's output);
 *   kcache, vcache fp16 bits [hkv][l_max][d]: rows 0..pos-1 hold the
 *          earlier tokens (already rotated keys); row pos is not read;
 *   k_new, v_new out fp16 bits [hkv*d]: the rows this token appends,
 *          fp16_rne(RoPE(k)) and fp16_rne(v), which also stand in for row pos;
 *   o, mag out fp64 [hq*d]: o = sum_j p_j v_j and mag = sum_j p_j |v_j| with
 *          p = softmax_j( RoPE(q_h) . k_j / sqrt(d) ), j = 0..pos, query head
 *          h reading kv head h / (hq / hkv).
 * All arithmetic fp64 in index order (the max is subtracted before exp). */
void orc_decode_attention(const float* qkv, int64_t hq, int64_t hkv, int64_t d,
                          const uint16_t* kcache, const uint16_t* vcache, int64_t l_max,
                          int64_t pos, double theta, uint16_t* k_new, uint16_t* v_new,
                          double* o, double* mag);

/* Threads the parallel row loops use (OpenMP). */
int orc_num_threads(void);
void orc_set_num_threads(int n);

#ifdef __cplusplus
}
#endif

#endif /* QG_ORACLE_H */
