// qg_gemv_impl.cuh -- the S=1 decode weight stream on sm_100a (kernel templates).
//
// One kernel family computes y = W_dq x for an int8 block-32 or int4
// group-64 weight, with three epilogues: plain (fp32 and/or fp16 out), fused
// gate/up SwiGLU (two weights, fp16 h out) and fused LM-head argmax.  The
// pages ("Qwen3-VL 4B -- Core AI (.aimodel)", Measured) state that decode is
// bound by reading every weight once per token, so the kernel is built to keep
// HBM saturated:
//
//  * Codes and scales stream straight from HBM into registers with 16-byte
//    coalesced vector loads (L1 bypassed, L2 evict-first).  Each lane keeps
//    DEPTH-1 steps of loads in flight while it computes; a warp owns RG rows
//    (x NMAT weights) at a time, so 64-128 bytes per lane are outstanding.
//    (On this GPU a plain 16-byte load stream reaches ~7.3 TB/s, while 1-D
//    bulk copies need >= 16 KB per copy to get there: every bulk copy carries
//    a fixed cost, and rows of 2-6 KB would pay it too often.)
//  * x (fp16) is staged once per CTA into shared memory, still fp16, in a
//    layout where each 8-lane phase of a 16-byte read hits distinct banks,
//    with (int4) the sum of x per lane granule; one x read serves all RG rows.
//  * Dequantization needs no int->float conversion: one byte permute (int8,
//    two codes) or one mask-and-or (int4, two codes) builds a pair of fp16
//    values 1024 + u, exact, and one packed fp16 subtraction of the constant
//    turns it into the code itself (q, or 16 q for int4's odd nibbles),
//    still exact.  The sm_100 mixed-precision FMA (fma.rn.f32.f16) then
//    multiplies it by the fp16 x pair into an fp32 accumulator with an exact
//    product, so the accumulated terms are q x themselves: the rounding error
//    scales with sum |q x|, never with sum |x| (no large offset cancels).
//    Each block's fp16 scale is applied once per 16 (int8) or 32 (int4)
//    codes; the int4 bias uses sum_k (q s + b) x = s sum (q - q0) x + b' sum x
//    around the group's zero point q0 (see i4_zero_point).
//  * Lanes split K within a row; a warp-shuffle reduction finishes each row.
//  * Programmatic dependent launch: before waiting on the previous kernel in
//    the stream, every warp asks L2 to prefetch (cp.async.bulk.prefetch.L2) the
//    first rows it will read, so a kernel's weight stream overlaps the tail of
//    the kernel before it; only x waits for that kernel.
//
// Included by qg_gemv.cu (plain, SwiGLU and head epilogues; the persistent
// sweep) and qg_gemv_decode.cu (the decode-step variants: RMSNorm input,
// residual epilogue), which compile in parallel.  The including file defines
// the device error flag g_gemv_err (one per translation unit) before this
// header.
#pragma once

#include <cfloat>
#include <climits>

#include "qg_device.cuh"
#include "qg_internal.h"

namespace qg {
namespace {

constexpr int kLanes = 32;
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * kLanes;
// Two CTAs (16 warps) per SM: measured faster than one CTA per SM that would
// leave room for the next kernel to become resident early; the latency hiding
// of 16 warps is worth more than that overlap.
constexpr int kCtasPerSm = 2;
constexpr int kPrefetchBytesPerWarp = 12 * 1024;

// FMT: 0 int8 block-32, 1 int4 group-64, 2 plain fp16 weights (no scales).
template <int FMT>
struct Fmt {
    static constexpr int kCodesPerLane = FMT == 0 ? 16 : (FMT == 1 ? 32 : 8);  // one 16-byte vector
    static constexpr bool kScales = FMT != 2;
    static constexpr int kBlock = FMT == 0 ? 32 : 64;           // codes per scale (FMT 0 and 1)
    static constexpr int kPieces = kCodesPerLane / 8;           // 16-byte fp16 x pieces per lane
    static constexpr int kSums = FMT == 1 ? 1 : 0;              // floats of x sums per granule
    static constexpr bool kBias = FMT == 1;
};

struct Params {
    const uint8_t* codes[2];
    const uint16_t* scales[2];
    const uint16_t* biases[2];
    int64_t n, k;
    const uint16_t* x;
    float* y;
    uint16_t* y16;
    uint16_t* h;
    float* logits;
    int32_t* idx;
    unsigned long long* ws_key;
    unsigned int* ws_ticket;
    int x_words;         // 4-byte words reserved for the staged fp16 x in shared memory
    int prefetch_items;  // items per warp prefetched into L2 before the wait
    int x_bulk;          // ring path: x arrives by one bulk copy into a raw buffer
    float eps;           // RMSNorm epsilon (with h_in)
    const float* h_in;   // if set: x = RMSNorm(h_in; gamma, eps) instead of p.x
    const uint16_t* gamma;
    float* h_res;        // plain epilogue: if set, h_res[r] += y[r] (the residual stream)
};

__host__ __device__ constexpr int align_up(int v, int a) { return (v + a - 1) / a * a; }

// ------------------------------------------------------------- loads -----
__device__ __forceinline__ uint4 ldg_stream_v4(const void* p, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}

__device__ __forceinline__ uint16_t ldg_stream_u16(const void* p, uint64_t pol) {
    uint16_t v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.u16 %0, [%1], %2;"
                 : "=h"(v)
                 : "l"(p), "l"(pol));
    return v;
}

// Ask L2 to fetch [p, p + bytes) (16-byte aligned, multiple of 16): a hint
// that needs no shared memory and no completion tracking.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// ------------------------------------------------------------ dot products --
// acc_a += lo(q2) * lo(x2), acc_b += hi(q2) * hi(x2): fp16 x fp16 -> fp32,
// one rounding (the products of 11-bit significands are exact in fp32).
__device__ __forceinline__ void fma_f16x2_f32(float& acc_a, float& acc_b, uint32_t q2,
                                              uint32_t x2) {
    asm("{\n\t.reg .f16 q0, q1, x0, x1;\n\t"
        "mov.b32 {q0, q1}, %2;\n\t"
        "mov.b32 {x0, x1}, %3;\n\t"
        "fma.rn.f32.f16 %0, q0, x0, %0;\n\t"
        "fma.rn.f32.f16 %1, q1, x1, %1;\n\t}"
        : "+f"(acc_a), "+f"(acc_b)
        : "r"(q2), "r"(x2));
}

// (a - b) on two packed fp16 values; exact whenever the differences are
// integers of magnitude < 2048 (as for every use below).
__device__ __forceinline__ uint32_t hsub2_u32(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// 16 int8 codes (one 16-byte vector) against their 16 fp16 x (two pieces, in
// k order): returns sum_k q_k x_k.  The code byte q (two's complement) is
// turned into offset binary u = q + 128 and permuted under 0x64, the fp16
// encoding of 1024 + u (exact for u < 1024); subtracting 1152 (fp16 0x6480)
// leaves q exactly, so every product q x is exact in fp32.
__device__ __forceinline__ float dot16_i8(const uint4 c, const uint4* xv) {
    float a0 = 0.f, a1 = 0.f;
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    const uint32_t x[8] = {xv[0].x, xv[0].y, xv[0].z, xv[0].w,
                           xv[1].x, xv[1].y, xv[1].z, xv[1].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t u = w[i] ^ 0x80808080u;
        fma_f16x2_f32(a0, a1, hsub2_u32(__byte_perm(u, 0x64646464u, 0x4140), 0x64806480u),
                      x[2 * i]);
        fma_f16x2_f32(a0, a1, hsub2_u32(__byte_perm(u, 0x64646464u, 0x4342), 0x64806480u),
                      x[2 * i + 1]);
    }
    return a0 + a1;
}

// 8 fp16 weights (one 16-byte vector) against their 8 fp16 x: sum_k w_k x_k.
__device__ __forceinline__ float dot8_f16(const uint4 c, const uint4* xv) {
    float a0 = 0.f, a1 = 0.f;
    fma_f16x2_f32(a0, a1, c.x, xv[0].x);
    fma_f16x2_f32(a0, a1, c.y, xv[0].y);
    fma_f16x2_f32(a0, a1, c.z, xv[0].z);
    fma_f16x2_f32(a0, a1, c.w, xv[0].w);
    return a0 + a1;
}

// The zero point of an int4 group: q0 = clamp(rint(-b / s), 0, 15), the code
// whose dequantized value lies nearest 0, as the packed fp16 constants
// (1024 + q0, 1024 + q0) and (1024 + 16 q0, 1024 + 16 q0) that dot32_i4
// subtracts, and the shifted bias b' = b + q0 s (exact in fp32 whenever the
// two terms nearly cancel).  With it, w = q s + b = (q - q0) s + b', and a
// term (q - q0) s is never larger than |w| + |b'| <= 2 |w| unless q = q0, in
// which case w = b' itself: no term of the sum is much larger than the
// weight it stands for, so s sum (q - q0) x + b' sum x does not cancel
// catastrophically when w is near 0 (an affine group that straddles 0).
// q0 only has to be near the zero crossing; any value in [0, 15] is exact.
struct I4Zero {
    uint32_t lo, hi;
    float bias;
};
// q0 comes from an approximate reciprocal (nearness is all it needs): with
// s = 0 (a constant group) the product is +-inf or NaN, the conversion
// saturates or gives 0, and any q0 is exact because every term (q - q0) s
// is 0.
__device__ __forceinline__ I4Zero i4_zero_point(float s, float b) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
    const int q0 = min(15, max(0, __float2int_rn(-b * r)));
    const uint32_t u = static_cast<uint32_t>(q0);
    return {0x64006400u + u * 0x00010001u, 0x64006400u + u * 0x00100010u,
            fmaf(static_cast<float>(q0), s, b)};
}

// 32 int4 codes (one 16-byte vector, even k in the low nibble) against their
// 32 fp16 x, staged per 8-code word as the pairs (x0,x4) (x1,x5) (x2,x6)
// (x3,x7).  One mask-and-or per pair puts nibbles 0/4 and 2/6 (after a shift
// by 8) in the low bits of the fp16 mantissa (1024 + q) and nibbles 1/5 and
// 3/7 four bits higher (1024 + 16 q); subtracting the zero point's constants
// leaves q - q0 and 16 (q - q0) exactly.  Returns sum_k (q_k - q0) x_k (every
// product exact in fp32).
__device__ __forceinline__ float dot32_i4(const uint4 c, const uint4* xv, const I4Zero& z) {
    float l0 = 0.f, l1 = 0.f, h0 = 0.f, h1 = 0.f;
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    constexpr uint32_t k1024 = 0x64006400u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t v = w[i], v8 = v >> 8;
        fma_f16x2_f32(l0, l1, hsub2_u32((v & 0x000F000Fu) | k1024, z.lo), xv[i].x);
        fma_f16x2_f32(h0, h1, hsub2_u32((v & 0x00F000F0u) | k1024, z.hi), xv[i].y);
        fma_f16x2_f32(l0, l1, hsub2_u32((v8 & 0x000F000Fu) | k1024, z.lo), xv[i].z);
        fma_f16x2_f32(h0, h1, hsub2_u32((v8 & 0x00F000F0u) | k1024, z.hi), xv[i].w);
    }
    return (l0 + l1) + (h0 + h1) * 0.0625f;
}

// acc += sum over one lane's 32 int4 codes of (q s + b) x, given the scale,
// the bias and sx = the sum of those 32 x.
__device__ __forceinline__ float i4_accumulate(float acc, float s, float b, const uint4 c,
                                               const uint4* xv, float sx) {
    const I4Zero z = i4_zero_point(s, b);
    return fmaf(s, dot32_i4(c, xv, z), fmaf(z.bias, sx, acc));
}

// 16-byte index of piece `i` of lane-granule `g` in the staged x: the eight
// granules read by one 8-lane phase of a 16-byte shared load are adjacent.
template <int FMT>
__device__ __forceinline__ int x_piece(int g, int i) {
    return ((g >> 3) * Fmt<FMT>::kPieces + i) * 8 + (g & 7);
}

__device__ __forceinline__ unsigned long long argmax_key(float v, int idx) {
    uint32_t b = __float_as_uint(v);
    b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);  // order-preserving map
    return (static_cast<unsigned long long>(b) << 32) |
           static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(idx));
}

// Steps of loads kept in the register pipeline: enough that (DEPTH-1) x rows
// x 16 bytes per lane stay outstanding (an int4 vector carries twice the
// weights and needs more registers to dequantize, so its pipeline is shorter).
template <int FMT, int ROWS>
struct Depth {
    static constexpr int value = FMT == 0 ? (ROWS >= 8 ? 2 : (ROWS >= 4 ? 3 : (ROWS >= 2 ? 5 : 8)))
                                          : (ROWS >= 4 ? 2 : (ROWS >= 2 ? 3 : 6));
};

template <int ROWS>
struct Frag {
    uint4 c[ROWS];
    uint16_t s[ROWS];
    uint16_t b[ROWS];
};

// ------------------------------------------------------ shared kernel parts --
// Stage x (fp16 in global memory, written by the previous kernel or by an
// earlier stage of the same sweep, hence read through L2; or already copied
// raw into shared memory; or computed as an RMSNorm) into shared memory, still fp16, in the
// conflict-free piece layout (int4: each 8-code word as the pairs the dot
// product wants), and for int4 per lane granule the sum the bias term
// needs: sums[g] = sum x over the granule (int8 and fp16 weights need none).
// Sources of x: kXGlobal (fp16 in global memory), kXShared (fp16 already in
// shared memory), kXNorm (the RMSNorm of an fp32 hidden state: x = fp16(h *
// rstd * gamma), rstd computed beforehand).
enum XSource : int { kXGlobal = 0, kXShared = 1, kXNorm = 2 };

__device__ __forceinline__ uint4 norm_piece(const float* h, const uint16_t* gamma, float rstd) {
    // h: written by the previous kernel, which griddepcontrol.wait has made
    // visible; read with plain (L1-cached) loads, hitting the lines that
    // rmsnorm_rstd brought in.  (No stage of a persistent sweep takes an
    // RMSNorm input, so no CTA of this grid writes h.)
    const float4 a = *reinterpret_cast<const float4*>(h);
    const float4 b = *reinterpret_cast<const float4*>(h + 4);
    const uint4 gv = *reinterpret_cast<const uint4*>(gamma);
    const float hv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float x0 = hv[2 * e] * rstd * h2f(static_cast<uint16_t>(gw[e] & 0xFFFFu));
        const float x1 = hv[2 * e + 1] * rstd * h2f(static_cast<uint16_t>(gw[e] >> 16));
        o[e] = static_cast<uint32_t>(f2h_rn(x0)) | (static_cast<uint32_t>(f2h_rn(x1)) << 16);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

template <int FMT, int SRC = kXGlobal>
__device__ __forceinline__ void stage_x(const uint16_t* __restrict__ x, uint4* xs, float* sums,
                                        int granules, const float* h = nullptr,
                                        const uint16_t* gamma = nullptr, float rstd = 0.f) {
    using F = Fmt<FMT>;
    for (int g = threadIdx.x; g < granules; g += blockDim.x) {
        const int64_t k0 = static_cast<int64_t>(g) * F::kCodesPerLane;
        const uint16_t* xg = x + k0;
        float se = 0.f, so = 0.f;  // sums over even and odd k (int4 only)
#pragma unroll
        for (int c = 0; c < F::kPieces; ++c) {
            const uint4 v = SRC == kXShared ? *reinterpret_cast<const uint4*>(xg + 8 * c)
                          : SRC == kXGlobal ? ldg_cg_v4(xg + 8 * c)
                                            : norm_piece(h + k0 + 8 * c, gamma + k0 + 8 * c, rstd);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            if (FMT == 1) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    se += h2f(static_cast<uint16_t>(w[e] & 0xFFFFu));
                    so += h2f(static_cast<uint16_t>(w[e] >> 16));
                }
            }
            if (FMT != 1) {
                xs[x_piece<FMT>(g, c)] = v;
            } else {  // (x0,x1)(x2,x3)(x4,x5)(x6,x7) -> (x0,x4)(x1,x5)(x2,x6)(x3,x7)
                xs[x_piece<FMT>(g, c)] =
                    make_uint4(__byte_perm(w[0], w[2], 0x5410), __byte_perm(w[0], w[2], 0x7632),
                               __byte_perm(w[1], w[3], 0x5410), __byte_perm(w[1], w[3], 0x7632));
            }
        }
        if (FMT == 1) sums[g] = se + so;
    }
}

// The residual stream's value at row r0 + lane, for lane < RG, read at the
// start of an item so that its latency hides behind the item's steps.
template <int RG, int EPI>
__device__ __forceinline__ float residual_old(const Params& p, int64_t r0, int64_t N, int lane) {
    if constexpr (epi_kind(EPI) != kEpiResidual) {
        return 0.f;
    } else {
        if (lane >= RG) return 0.f;
        const int64_t r = r0 + lane < N ? r0 + lane : N - 1;
        return p.h_res[r];
    }
}

// The pre-norm RMSNorm's 1/rms of the fp32 hidden state h [k]: per-thread
// sums of squares in index order, then the warp and the CTA in a fixed order;
// every thread returns the same value.  red: kWarps floats of shared memory.
__device__ __forceinline__ float rmsnorm_rstd(const float* h, const uint16_t* gamma, int64_t k,
                                              float eps, float* red) {
    float ss = 0.f;
    for (int64_t i = threadIdx.x; i < k / 4; i += blockDim.x) {
        const float4 v = *reinterpret_cast<const float4*>(h + 4 * i);
        // bring the gains into L1 in the same round trip (the staging reads them)
        if ((i & 1) == 0) asm volatile("prefetch.global.L1 [%0];" ::"l"(gamma + 4 * i));
        ss = fmaf(v.x, v.x, ss);
        ss = fmaf(v.y, v.y, ss);
        ss = fmaf(v.z, v.z, ss);
        ss = fmaf(v.w, v.w, ss);
    }
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) tot += red[w];
    __syncthreads();  // red is free again
    return __fdiv_rn(1.0f, __fsqrt_rn(__fdiv_rn(tot, static_cast<float>(k)) + eps));
}

// Finish the RG rows (x NMAT weights) of one warp item: reduce across lanes
// and apply the epilogue; lane j writes row r0 + j.  h_old: lane j's value of
// the residual stream at row r0 + j, read when the item started (no other
// lane or CTA writes that row).
template <int NMAT, int RG, int EPI>
__device__ __forceinline__ void finish_item(float (&acc)[NMAT * RG], int64_t r0, int64_t N,
                                            const Params& p, int lane, float& best_v,
                                            int& best_i, float h_old = 0.f) {
#pragma unroll
    for (int j = 0; j < NMAT * RG; ++j) acc[j] = warp_sum(acc[j]);
    if (lane < RG && r0 + lane < N) {
        const int64_t r = r0 + lane;
        float v0 = acc[0], v1 = 0.f;
#pragma unroll
        for (int j = 0; j < RG; ++j)
            if (lane == j) {
                v0 = acc[j];
                if (NMAT == 2) v1 = acc[(NMAT - 1) * RG + j];
            }
        constexpr int kKind = epi_kind(EPI);
        if (kKind == kEpiPlain) {
            if (p.y) p.y[r] = v0;
            if (p.y16) p.y16[r] = f2h_rn(v0);
        } else if (kKind == kEpiResidual) {
            p.h_res[r] = h_old + v0;  // residual stream (one lane owns the row)
        } else if (kKind == kEpiSwiglu) {
            p.h[r] = f2h_rn(v0 / (1.0f + expf(-v0)) * v1);
        } else {
            if (p.logits) p.logits[r] = v0;
            if (v0 > best_v) {  // rows arrive in increasing order per lane
                best_v = v0;
                best_i = static_cast<int>(r);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < NMAT * RG; ++j) acc[j] = 0.f;
}

// Head epilogue of a whole CTA: lane -> warp -> CTA (value, lowest index),
// then one atomicMax per CTA and a ticket; the last CTA publishes the index
// and re-zeroes the workspace.  No CTA ever waits on another.
__device__ __forceinline__ void head_finish(const Params& p, float best_v, int best_i, int warp,
                                            int lane, float* red_v, int* red_i, int nwarps) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, best_v, o);
        const int oi = __shfl_xor_sync(0xffffffffu, best_i, o);
        if (ov > best_v || (ov == best_v && oi < best_i)) {
            best_v = ov;
            best_i = oi;
        }
    }
    if (lane == 0) {
        red_v[warp] = best_v;
        red_i[warp] = best_i;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float bv = red_v[0];
        int bi = red_i[0];
        for (int w = 1; w < nwarps; ++w)
            if (red_v[w] > bv || (red_v[w] == bv && red_i[w] < bi)) {
                bv = red_v[w];
                bi = red_i[w];
            }
        if (bi != INT_MAX) atomicMax(p.ws_key, argmax_key(bv, bi));
        __threadfence();
        const unsigned int ticket = atomicAdd(p.ws_ticket, 1u);
        if (ticket == gridDim.x - 1) {
            __threadfence();
            const unsigned long long key = atomicAdd(p.ws_key, 0ull);
            *p.idx = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(key & 0xFFFFFFFFull));
            *p.ws_key = 0ull;
            *p.ws_ticket = 0u;
        }
    }
}

// L2 prefetch of items [first, first + count) of a warp (bulk prefetch hint).
template <int FMT, int NMAT, int RG>
__device__ __forceinline__ void prefetch_items(const Params& p, int64_t wg, int64_t tw,
                                               int first, int count, int my_items) {
    using F = Fmt<FMT>;
    const int64_t N = p.n, K = p.k;
    const int64_t row_bytes = FMT == 0 ? K : (FMT == 1 ? K / 2 : K * 2);
    const int64_t side_per_row = F::kScales ? K / F::kBlock : 0;
    for (int i = first; i < first + count && i < my_items; ++i) {
        const int64_t r0 = (wg + i * tw) * RG;
        const int64_t rows = N - r0 < RG ? N - r0 : RG;
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
            const uint8_t* cm = m == 0 ? p.codes[0] : p.codes[1];
            prefetch_l2(cm + r0 * row_bytes, static_cast<uint32_t>(rows * row_bytes));
            const uintptr_t sa = reinterpret_cast<uintptr_t>(
                (m == 0 ? p.scales[0] : p.scales[1]) + r0 * side_per_row);
            const uint32_t sbytes = static_cast<uint32_t>(rows * side_per_row * 2);
            if (F::kScales && sa % 16 == 0 && sbytes % 16 == 0) {
                prefetch_l2(reinterpret_cast<const void*>(sa), sbytes);
                if (F::kBias)
                    prefetch_l2((m == 0 ? p.biases[0] : p.biases[1]) + r0 * side_per_row, sbytes);
            }
        }
    }
}

// ----------------------------------------------------------------------- //
// Register-pipeline kernel: loads land in registers DEPTH-1 steps ahead.    //
// Used when a row's scale count is not a multiple of 8 (the shared-memory   //
// ring below copies scales as 16-byte pieces).                              //
// ----------------------------------------------------------------------- //
template <int FMT, int NMAT, int RG, int EPI>
__global__ void __launch_bounds__(kThreads, 2) gemv_kernel(const Params p) {
    using F = Fmt<FMT>;
    constexpr int ROWS = NMAT * RG;
    constexpr int DEPTH = Depth<FMT, ROWS>::value;
    constexpr int kStepBytes = kLanes * 16;  // code bytes of one warp step along a row
    constexpr int kStepSides = kStepBytes * (FMT == 0 ? 1 : 2) / F::kBlock;  // scales per step
    extern __shared__ __align__(128) unsigned char smem[];
    uint4* xs = reinterpret_cast<uint4*>(smem);
    float* sums = reinterpret_cast<float*>(smem) + p.x_words;
    __shared__ float red_v[kWarps];
    __shared__ int red_i[kWarps];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t N = p.n, K = p.k;
    const int granules = static_cast<int>(K / F::kCodesPerLane);  // 16-byte vectors per row
    const int nst = (granules + kLanes - 1) / kLanes;              // warp steps per row
    const int64_t items = (N + RG - 1) / RG;
    const int64_t wg = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
    const int64_t tw = static_cast<int64_t>(gridDim.x) * kWarps;
    const int my_items = wg < items ? static_cast<int>((items - wg + tw - 1) / tw) : 0;
    const int total = my_items * nst;
    const int64_t row_bytes = FMT == 0 ? K : K / 2;
    const int64_t side_per_row = K / F::kBlock;
    const uint64_t pol = l2_policy_evict_first();

    // load cursor: per-row pointers of the next step (lane offset included)
    const uint8_t* lc[ROWS];
    const uint16_t* ls[ROWS];
    const uint16_t* lb[ROWS];
    int ld_st = 0, ld_item = 0;
    auto set_item = [&](int il) {
        const int64_t r0 = (wg + il * tw) * RG;
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
            const uint8_t* cm = m == 0 ? p.codes[0] : p.codes[1];
            const uint16_t* sm = m == 0 ? p.scales[0] : p.scales[1];
            const uint16_t* bm = m == 0 ? p.biases[0] : p.biases[1];
#pragma unroll
            for (int j = 0; j < RG; ++j) {
                const int64_t r = r0 + j < N ? r0 + j : N - 1;  // tail rows: load, discard
                lc[m * RG + j] = cm + r * row_bytes + lane * 16;
                ls[m * RG + j] = sm + r * side_per_row + (lane >> 1);
                if (F::kBias) lb[m * RG + j] = bm + r * side_per_row + (lane >> 1);
            }
        }
    };
    auto load = [&](Frag<ROWS>& f) {
        if (ld_st * kLanes + lane < granules) {
#pragma unroll
            for (int j = 0; j < ROWS; ++j) {
                f.c[j] = ldg_stream_v4(lc[j], pol);
                f.s[j] = ldg_stream_u16(ls[j], pol);
                if (F::kBias) f.b[j] = ldg_stream_u16(lb[j], pol);
            }
        }
        if (++ld_st == nst) {
            ld_st = 0;
            if (++ld_item < my_items) set_item(ld_item);
        } else {
#pragma unroll
            for (int j = 0; j < ROWS; ++j) {
                lc[j] += kStepBytes;
                ls[j] += kStepSides;
                if (F::kBias) lb[j] += kStepSides;
            }
        }
    };

    // 1) weight prologue (independent of the previous kernel): the first
    //    DEPTH steps into registers, the next items into L2.
    Frag<ROWS> buf[DEPTH];
    if (my_items > 0) set_item(0);
#pragma unroll
    for (int d = 0; d < DEPTH; ++d)
        if (d < total) load(buf[d]);
    if (lane == 0) prefetch_items<FMT, NMAT, RG>(p, wg, tw, 1, p.prefetch_items - 1, my_items);

    // 2) x from the previous kernel
    griddep_wait();
    if constexpr ((EPI & kEpiNormIn) != 0) {
        const float rstd = rmsnorm_rstd(p.h_in, p.gamma, K, p.eps, red_v);
        stage_x<FMT, kXNorm>(p.x, xs, sums, granules, p.h_in, p.gamma, rstd);
    } else {
        stage_x<FMT>(p.x, xs, sums, granules);
    }
    __syncthreads();
    griddep_launch_dependents();

    // 3) stream
    const int x_lane = ((lane >> 3) * F::kPieces) * 8 + (lane & 7);  // x_piece(lane, 0)
    constexpr int kXStep = 4 * F::kPieces * 8;                      // per 32 granules
    float acc[ROWS];
#pragma unroll
    for (int j = 0; j < ROWS; ++j) acc[j] = 0.f;
    float best_v = -FLT_MAX;
    int best_i = INT_MAX;
    int cu_st = 0, cu_item = 0;
    float h_old = 0.f;
    auto consume = [&](const Frag<ROWS>& f) {
        if (cu_st == 0) h_old = residual_old<RG, EPI>(p, (wg + cu_item * tw) * RG, N, lane);
        const int g = cu_st * kLanes + lane;
        if (g < granules) {
            uint4 xv[F::kPieces];
            const uint4* xp = xs + x_lane + cu_st * kXStep;
#pragma unroll
            for (int i = 0; i < F::kPieces; ++i) xv[i] = xp[i * 8];
            const float c1 = FMT == 1 ? sums[g] : 0.f;
#pragma unroll
            for (int j = 0; j < ROWS; ++j) {
                if (FMT == 0)
                    acc[j] = fmaf(h2f(f.s[j]), dot16_i8(f.c[j], xv), acc[j]);
                else
                    acc[j] = i4_accumulate(acc[j], h2f(f.s[j]), h2f(f.b[j]), f.c[j], xv, c1);
            }
        }
        if (++cu_st == nst) {
            finish_item<NMAT, RG, EPI>(acc, (wg + cu_item * tw) * RG, N, p, lane, best_v, best_i,
                                       h_old);
            cu_st = 0;
            ++cu_item;
        }
    };
    for (int t = 0; t < total; t += DEPTH) {
#pragma unroll
        for (int d = 0; d < DEPTH; ++d) {
            if (t + d < total) {
                consume(buf[d]);
                if (t + d + DEPTH < total) load(buf[d]);
            }
        }
    }
    if (epi_kind(EPI) == kEpiHead) head_finish(p, best_v, best_i, warp, lane, red_v, red_i, kWarps);
}

// ----------------------------------------------------------------------- //
// Shared-memory rings: the fast path, as a launch of its own or as one     //
// stage of a persistent sweep.                                             //
// ----------------------------------------------------------------------- //
constexpr int kRing = 4;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint64_t pol) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst),
                 "l"(src), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a));
    return v;
}
__device__ __forceinline__ uint16_t lds16(uint32_t a) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}

template <int FMT, int NMAT>
struct RingLayout {
    // bytes per (slot, row): the 32 lanes' code vectors, then the step's 16
    // fp16 scales (and 16 biases for int4)
    static constexpr int kCodes = kLanes * 16;
    static constexpr int kSide = 32;
    static constexpr int kPerRow = kCodes + kSide * (FMT == 1 ? 2 : (FMT == 0 ? 1 : 0));
};

// Shared memory of one CTA's rings; x (and the int4 sums) follow it.
__host__ __device__ constexpr uint32_t ring_bytes(int fmt, int rows) {
    return static_cast<uint32_t>(kWarps * kRing * rows *
                                 (kLanes * 16 + 32 * (fmt == 1 ? 2 : (fmt == 0 ? 1 : 0))));
}

// How a ring stage orders itself after the work before it.
//  * StreamSync -- a launch of its own: programmatic dependent launch.  The
//    weight prologue runs while the previous kernel in the stream finishes;
//    x is read after griddepcontrol.wait.
//  * GridSync -- one stage of a persistent sweep: when every warp of the CTA
//    is done with the previous stage, the CTA arrives on that stage's counter
//    and issues this stage's weight prologue, then waits (bounded) until all
//    CTAs have arrived before it reads x, which the previous stage may have
//    written.
struct StreamSync {
    __device__ __forceinline__ void before_prologue() {}
    __device__ __forceinline__ bool wait_input() {
        griddep_wait();
        return true;
    }
    __device__ __forceinline__ void input_staged() { griddep_launch_dependents(); }
};

struct GridSync {
    unsigned int* prev;        // arrival counter of the previous stage, or nullptr
    int* go;                   // shared: the outcome of thread 0's wait
    const uint4* next_src;     // the next stage's descriptor (global), or nullptr
    uint4* next_dst;           // where the CTA keeps it (shared)
    int next_pieces;           // its 16-byte pieces
    // (the sweep kernel has synchronized the CTA: every warp is done with the
    // previous stage's outputs, x and rings)
    __device__ __forceinline__ void before_prologue() {
        if (prev && threadIdx.x == 0) red_release_gpu_inc(prev);
    }
    __device__ __forceinline__ bool wait_input() {
        // the next stage's descriptor is fetched while the grid waits
        if (next_src && static_cast<int>(threadIdx.x) < next_pieces)
            next_dst[threadIdx.x] = ldg_nc_v4(next_src + threadIdx.x);
        if (threadIdx.x == 0)
            *go = (prev == nullptr || wait_counter_bounded(prev, gridDim.x)) ? 1 : 0;
        __syncthreads();
        return *go != 0;
    }
    __device__ __forceinline__ void input_staged() {}
};

// One weight (or gate/up pair) streamed through per-lane shared-memory rings:
// every lane copies the 16-byte code vectors it will consume with cp.async
// into its own ring slots, kRing-1 steps ahead; a few lanes copy each step's
// scales (and biases) as 16-byte pieces, read by the warp after a __syncwarp.
// Bytes in flight cost no registers: 3 steps x RG rows x 16 B per lane stay
// outstanding.  Requires a multiple of 8 scales per row (16-byte pieces).
// WHOLE selects the loop for rows of at least kRing - 1 whole steps (see
// below); both loops add the same products in the same order, so the two
// variants give bit-identical results.
// Returns false, with its copies drained, if the wait for x gave up.
template <int FMT, int NMAT, int RG, int EPI, bool WHOLE = false, class SYNC>
__device__ __forceinline__ bool ring_stage(const Params& p, unsigned char* smem, SYNC& sync,
                                           float* red_v, int* red_i) {
    using F = Fmt<FMT>;
    using RL = RingLayout<FMT, NMAT>;
    constexpr int ROWS = NMAT * RG;
    constexpr int kStepBytes = kLanes * 16;
    constexpr int kStepSides = F::kScales ? kStepBytes * (FMT == 0 ? 1 : 2) / F::kBlock : 0;  // 16
    constexpr int kSideLanes = F::kScales ? 2 * ROWS * (F::kBias ? 2 : 1) : 0;  // side-data copiers

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t N = p.n, K = p.k;
    const int granules = static_cast<int>(K / F::kCodesPerLane);
    const int nst = (granules + kLanes - 1) / kLanes;
    const int64_t items = (N + RG - 1) / RG;
    const int64_t wg = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
    const int64_t tw = static_cast<int64_t>(gridDim.x) * kWarps;
    const int my_items = wg < items ? static_cast<int>((items - wg + tw - 1) / tw) : 0;
    const int total = my_items * nst;
    const int64_t row_bytes = FMT == 0 ? K : (FMT == 1 ? K / 2 : K * 2);
    const int64_t side_per_row = F::kScales ? K / F::kBlock : 0;  // a multiple of 8 (16-byte pieces)
    const uint64_t pol = l2_policy_evict_first();

    // shared memory: [rings of this CTA's warps][x fp16][x sums][x fp16 raw]
    const uint32_t ring = smem_u32(smem) + warp * (kRing * ROWS * RL::kPerRow);
    uint4* xs = reinterpret_cast<uint4*>(smem + ring_bytes(FMT, ROWS));
    float* sums = reinterpret_cast<float*>(xs) + p.x_words;
    uint16_t* xraw = reinterpret_cast<uint16_t*>(sums + align_up(F::kSums * granules, 4));
    // x by bulk copy: one 1-D copy of k fp16 values, completing on xbar (its
    // requests do not queue behind the ring's 16-byte copies)
    __shared__ __align__(8) uint64_t xbar;
    if (p.x_bulk) {
        if (threadIdx.x == 0) {
            mbar_init(&xbar, 1);
            fence_mbar_init();
        }
        __syncthreads();
    }
    auto slot_codes = [&](int s, int j) -> uint32_t {  // this lane's code vector
        return ring + (s * ROWS + j) * RL::kPerRow + lane * 16;
    };
    auto slot_side = [&](int s, int j, int which) -> uint32_t {  // the step's 16 sides
        return ring + (s * ROWS + j) * RL::kPerRow + RL::kCodes + which * RL::kSide;
    };

    // Side data: each step of a row needs 16 consecutive scales (32 B) and,
    // for int4, 16 biases.  Lane l < kSideLanes copies one 16-byte piece of
    // one of them (no two lanes copy the same bytes); the warp then
    // synchronizes before reading.
    const bool side_lane = lane < kSideLanes;
    const int side_which = lane / (2 * ROWS);          // 0: scales, 1: biases
    const int side_row = (lane % (2 * ROWS)) >> 1;     // row slot 0..ROWS-1
    const int side_half = lane & 1;                    // which 16-byte piece
    const int side_m = side_row / RG, side_j = side_row % RG;

    // load cursor (global addresses of the next step)
    const uint8_t* lc[ROWS];
    const uint16_t* lside = nullptr;
    int ld_st = 0, ld_item = 0, ld_slot = 0;
    auto set_item = [&](int il) {
        const int64_t r0 = (wg + il * tw) * RG;
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
            const uint8_t* cm = m == 0 ? p.codes[0] : p.codes[1];
#pragma unroll
            for (int j = 0; j < RG; ++j) {
                const int64_t r = r0 + j < N ? r0 + j : N - 1;  // tail rows: copy, discard
                lc[m * RG + j] = cm + r * row_bytes + lane * 16;
            }
        }
        if (side_lane) {
            const int64_t r = r0 + side_j < N ? r0 + side_j : N - 1;
            const uint16_t* base =
                side_which == 0 ? (side_m == 0 ? p.scales[0] : p.scales[1])
                                : (side_m == 0 ? p.biases[0] : p.biases[1]);
            lside = base + r * side_per_row + side_half * 8;
        }
    };
    auto issue = [&]() {
        if (ld_st * kLanes + lane < granules) {
#pragma unroll
            for (int j = 0; j < ROWS; ++j) cp_async16(slot_codes(ld_slot, j), lc[j], pol);
        }
        if (side_lane && ld_st * kStepSides + side_half * 8 + 8 <= side_per_row)
            cp_async16(slot_side(ld_slot, side_row, side_which) + side_half * 16, lside, pol);
        cp_async_commit();
        if (++ld_slot == kRing) ld_slot = 0;
        if (++ld_st == nst) {
            ld_st = 0;
            if (++ld_item < my_items) set_item(ld_item);
        } else {
#pragma unroll
            for (int j = 0; j < ROWS; ++j) lc[j] += kStepBytes;
            if (side_lane) lside += kStepSides;
        }
    };

    // WHOLE: rows of whole steps (every lane has a code vector in every step,
    // every step has its 16 sides) and at least kRing - 1 steps.  The load
    // cursor below then moves on to the next item only at step
    // nst - (kRing - 1) of each item, so the streaming loop needs no per-step
    // bounds or item tests.  The launcher picks it only for such rows.
    if constexpr (WHOLE) {
        if (granules % kLanes != 0 || nst < kRing - 1) {
            if (threadIdx.x == 0) atomicOr(&g_gemv_err, kGemvErrBadPlan);
            return false;
        }
    }
    constexpr uint32_t kSlotBytes = ROWS * RL::kPerRow;
    const uint32_t ring_end = ring + kRing * kSlotBytes;
    const uint32_t side_ld =
        side_row * RL::kPerRow + RL::kCodes + side_which * RL::kSide + side_half * 16;
    uint32_t ld_addr = ring;  // the slot the whole-step cursor fills next
    auto issue_whole = [&]() {
        const uint32_t a = ld_addr + lane * 16;
#pragma unroll
        for (int j = 0; j < ROWS; ++j) {
            cp_async16(a + j * RL::kPerRow, lc[j], pol);
            lc[j] += kStepBytes;
        }
        if (side_lane) {
            cp_async16(ld_addr + side_ld, lside, pol);
            lside += kStepSides;
        }
        ld_addr = ld_addr + kSlotBytes == ring_end ? ring : ld_addr + kSlotBytes;
    };

    // 1) weight prologue (independent of the work before this stage)
    sync.before_prologue();
    if (my_items > 0) set_item(0);
    if constexpr (WHOLE) {
#pragma unroll
        for (int d = 0; d < kRing - 1; ++d) {
            if (my_items > 0) issue_whole();
            cp_async_commit();
        }
    } else {
#pragma unroll
        for (int d = 0; d < kRing - 1; ++d) {
            if (d < total) issue();
            else cp_async_commit();
        }
    }
    if (lane == 0) prefetch_items<FMT, NMAT, RG>(p, wg, tw, 1, p.prefetch_items - 1, my_items);

    // 2) x, which the work before this stage may have written
    if (!sync.wait_input()) {
        cp_async_wait<0>();
        return false;
    }
    if constexpr ((EPI & kEpiNormIn) != 0) {  // x = RMSNorm(h): computed, not copied
        const float rstd = rmsnorm_rstd(p.h_in, p.gamma, K, p.eps, red_v);
        stage_x<FMT, kXNorm>(p.x, xs, sums, granules, p.h_in, p.gamma, rstd);
    } else if (p.x_bulk) {
        if (threadIdx.x == 0) {
            const uint32_t bytes = static_cast<uint32_t>(K * 2);
            mbar_arrive_expect_tx(&xbar, bytes);
            bulk_g2s(xraw, p.x, bytes, &xbar, l2_policy_evict_last());
        }
        if (!mbar_wait_bounded(&xbar, 0)) {
            if (threadIdx.x == 0) atomicOr(&g_gemv_err, kGemvErrTimeout);
            mbar_wait_bounded(&xbar, 0);  // the copy may still land: wait again, bounded
            cp_async_wait<0>();
            return false;
        }
        stage_x<FMT, kXShared>(xraw, xs, sums, granules);
    } else {
        stage_x<FMT>(p.x, xs, sums, granules);
    }
    __syncthreads();
    sync.input_staged();

    // 3) stream: issue step t + kRing - 1, wait for step t, compute it
    const int x_lane = ((lane >> 3) * F::kPieces) * 8 + (lane & 7);  // x_piece(lane, 0)
    constexpr int kXStep = 4 * F::kPieces * 8;                      // per 32 granules
    const int side_off = (lane >> 1) * 2;  // this lane's scale (bias) inside the step's 16
    float acc[ROWS];
#pragma unroll
    for (int j = 0; j < ROWS; ++j) acc[j] = 0.f;
    float best_v = -FLT_MAX;
    int best_i = INT_MAX;
    // One step of every row of the item from the ring slot at `slot`: the
    // lane's code vectors and sides, against the x pieces at xp (c1: the sum
    // of the lane's x, int4).
    auto compute = [&](uint32_t slot, const uint4* xp, float c1) {
        uint4 xv[F::kPieces];
#pragma unroll
        for (int i = 0; i < F::kPieces; ++i) xv[i] = xp[i * 8];
        const uint32_t cl = slot + lane * 16;
        const uint32_t cs = slot + RL::kCodes + side_off;
#pragma unroll
        for (int j = 0; j < ROWS; ++j) {
            const uint4 c = lds128(cl + j * RL::kPerRow);
            if (FMT == 2) {
                acc[j] += dot8_f16(c, xv);
                continue;
            }
            const float sc = h2f(lds16(cs + j * RL::kPerRow));
            if (FMT == 0) {
                acc[j] = fmaf(sc, dot16_i8(c, xv), acc[j]);
            } else {
                const float bi = h2f(lds16(cs + j * RL::kPerRow + RL::kSide));
                acc[j] = i4_accumulate(acc[j], sc, bi, c, xv, c1);
            }
        }
    };
    if constexpr (WHOLE) {
        // the cursor filled steps 0 .. kRing - 2 of item 0; in every step it
        // fills one more, moving to the next item at step nst - (kRing - 1)
        bool more = my_items > 0;
        uint32_t cu = ring;
        for (int il = 0; il < my_items; ++il) {
            const int64_t r0 = (wg + il * tw) * RG;
            const float h_old = residual_old<RG, EPI>(p, r0, N, lane);
            const uint4* xp = xs + x_lane;
            const float* sp = sums + lane;
            for (int st = 0; st < nst; ++st) {
                if (st == nst - (kRing - 1)) {
                    if (il + 1 < my_items) set_item(il + 1);
                    else more = false;
                }
                if (more) issue_whole();
                cp_async_commit();
                cp_async_wait<kRing - 1>();
                __syncwarp();  // side pieces copied by other lanes are now visible
                compute(cu, xp, FMT == 1 ? *sp : 0.f);
                __syncwarp();  // every lane is done with this slot before it is refilled
                xp += kXStep;
                sp += kLanes;
                cu = cu + kSlotBytes == ring_end ? ring : cu + kSlotBytes;
            }
            finish_item<NMAT, RG, EPI>(acc, r0, N, p, lane, best_v, best_i, h_old);
        }
    } else {
        int cu_st = 0, cu_item = 0, cu_slot = 0;
        float h_old = 0.f;
        for (int t = 0; t < total; ++t) {
            if (cu_st == 0) h_old = residual_old<RG, EPI>(p, (wg + cu_item * tw) * RG, N, lane);
            if (t + kRing - 1 < total) issue();
            else cp_async_commit();
            cp_async_wait<kRing - 1>();
            __syncwarp();  // side pieces copied by other lanes are now visible
            const int g = cu_st * kLanes + lane;
            if (g < granules) {
                uint4 xv[F::kPieces];
                const uint4* xp = xs + x_lane + cu_st * kXStep;
#pragma unroll
                for (int i = 0; i < F::kPieces; ++i) xv[i] = xp[i * 8];
                const float c1 = FMT == 1 ? sums[g] : 0.f;
#pragma unroll
                for (int j = 0; j < ROWS; ++j) {
                    const uint4 c = lds128(slot_codes(cu_slot, j));
                    if (FMT == 2) {
                        acc[j] += dot8_f16(c, xv);
                        continue;
                    }
                    const float sc = h2f(lds16(slot_side(cu_slot, j, 0) + side_off));
                    if (FMT == 0) {
                        acc[j] = fmaf(sc, dot16_i8(c, xv), acc[j]);
                    } else {
                        const float bi = h2f(lds16(slot_side(cu_slot, j, 1) + side_off));
                        acc[j] = i4_accumulate(acc[j], sc, bi, c, xv, c1);
                    }
                }
            }
            __syncwarp();  // every lane is done with this slot before it is refilled
            if (++cu_slot == kRing) cu_slot = 0;
            if (++cu_st == nst) {
                finish_item<NMAT, RG, EPI>(acc, (wg + cu_item * tw) * RG, N, p, lane, best_v,
                                           best_i, h_old);
                cu_st = 0;
                ++cu_item;
            }
        }
    }
    cp_async_wait<0>();
    if (epi_kind(EPI) == kEpiHead) head_finish(p, best_v, best_i, warp, lane, red_v, red_i, kWarps);
    return true;
}

template <int FMT, int NMAT, int RG, int EPI, bool WHOLE = false>
__global__ void __launch_bounds__(kThreads, 2) gemv_ring_kernel(const Params p) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ float red_v[kWarps];
    __shared__ int red_i[kWarps];
    StreamSync sync;
    ring_stage<FMT, NMAT, RG, EPI, WHOLE>(p, smem, sync, red_v, red_i);
}

// x's shared memory: the staged fp16 x, its per-granule sums, and the raw
// fp16 copy if x arrives by bulk copy.
size_t x_smem_bytes(int fmt, const Params& p) {
    const int cpl = fmt == QG_FMT_I8_B32 ? Fmt<0>::kCodesPerLane
                    : (fmt == QG_FMT_I4_G64 ? Fmt<1>::kCodesPerLane : Fmt<2>::kCodesPerLane);
    const int granules = static_cast<int>(p.k / cpl);
    const int nsums = (fmt == QG_FMT_I4_G64 ? Fmt<1>::kSums : 0) * granules;
    size_t b = static_cast<size_t>(p.x_words) * 4 + static_cast<size_t>(align_up(nsums, 4)) * 4;
    if (p.x_bulk) b += static_cast<size_t>(p.k) * 2;
    return b;
}

template <int FMT, int NMAT, int RG>
constexpr size_t ring_smem_bytes() {
    return ring_bytes(FMT, NMAT * RG);
}

// Per-CTA shared memory that still lets two CTAs share an SM.
constexpr size_t kSmemPerCtaBudget = 112 * 1024;

// Rows of whole warp steps (512 int8, 1024 int4 or 256 fp16 codes), at least
// kRing - 1 of them, stream through the ring kernel's whole-step loop, which
// drops the per-step bounds and item tests: about a fifth of the thread
// instructions of a one-row-per-item launch (ncu, 2048x6144 int8: 8.1 -> 6.7
// per weight).  Timed on B200 (graphs of every layer's launches, L2 flushed):
// down projections of the 2B / 4B / 8B / 27B decoders 5.19 -> 4.83,
// 9.34 -> 8.48, 11.72 -> 10.89 and 24.3 -> 22.7 us, then, for rows of 4-10
// steps, 4B q|k|v 4.63 -> 4.55, o 4.67 -> 4.54, 8B q|k|v 6.20 -> 5.99, o
// 4.99 -> 4.72, 8B int4 gate/up 17.6 -> 17.0 us.
constexpr int kWholeMinSteps = kRing - 1;
inline bool whole_step_rows(int fmt, int64_t k) {
    const int64_t step = static_cast<int64_t>(kLanes) *
                         (fmt == 0 ? Fmt<0>::kCodesPerLane
                                   : (fmt == 1 ? Fmt<1>::kCodesPerLane : Fmt<2>::kCodesPerLane));
    return k % step == 0 && k / step >= kWholeMinSteps;
}

template <int FMT, int NMAT, int RG, int EPI, bool RING>
qg_status launch_t(Params p, const DeviceInfo& dev, cudaStream_t stream) {
    void (*kern)(Params);  // only the chosen family is instantiated
    int variant = 0;
    if constexpr (RING) {
        if (whole_step_rows(FMT, p.k)) {
            kern = gemv_ring_kernel<FMT, NMAT, RG, EPI, true>;
            variant = 1;
        } else {
            kern = gemv_ring_kernel<FMT, NMAT, RG, EPI, false>;
        }
    } else {
        kern = gemv_kernel<FMT, NMAT, RG, EPI>;
    }
    size_t smem = x_smem_bytes(FMT, p) + (RING ? ring_smem_bytes<FMT, NMAT, RG>() : 0);
    if (smem + 1024 > static_cast<size_t>(dev.max_smem_optin)) return QG_ERR_SHAPE;
    if (variant == 1) {
        // A whole-step kernel holds fewer registers than the general one (67
        // against 90 for one int8 row per item), so a third CTA would fit on an
        // SM, and launches chained by programmatic dependent launch then crowd
        // the SMs that free first (2B down 4.90 -> 5.93 us).  Its shared-memory
        // request is padded past a third of the SM's to keep kCtasPerSm per SM.
        const size_t two_per_sm = (static_cast<size_t>(dev.smem_per_sm) / (kCtasPerSm + 1) + 16) /
                                  16 * 16;
        if (smem < two_per_sm && two_per_sm + 1024 <= static_cast<size_t>(dev.max_smem_optin))
            smem = two_per_sm;
    }
    // Opt in to exactly the dynamic shared memory this launch needs (static
    // shared memory counts against the same per-block limit).
    static size_t attr_set[2][64] = {};  // per kernel variant and device
    if (dev.device >= 64 || attr_set[variant][dev.device] < smem) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return cuda_status(e);
        if (dev.device < 64) attr_set[variant][dev.device] = smem;
    }
    const int64_t items = (p.n + RG - 1) / RG;
    int64_t grid = (items + kWarps - 1) / kWarps;
    const int64_t max_grid = static_cast<int64_t>(dev.num_sms) * kCtasPerSm;
    if (grid > max_grid) grid = max_grid;
    const int64_t item_bytes =
        static_cast<int64_t>(NMAT) * RG * (FMT == 0 ? p.k : (FMT == 1 ? p.k / 2 : p.k * 2));
    p.prefetch_items = static_cast<int>(kPrefetchBytesPerWarp / item_bytes);
    if (p.prefetch_items < 1) p.prefetch_items = 1;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, p));
}

// Rows per warp item.  More rows per step amortize a step's fixed work (ring
// bookkeeping, waits, x loads) over more bytes, at the cost of idle warps
// when items run short: timed on B200 over the 2B and 4B int8 and int4
// projections (CUDA graphs, HBM-resident copies), two rows per item win once
// the items cover half of the grid's warps and four rows once they cover 60%
// (2B qkv 3.87 -> 3.22 us, 4B o 5.42 -> 4.50 us, 4B qkv 5.62 -> 4.56 us
// against one or two rows per warp).
int pick_rg(int64_t n, int max_rg, int total_warps) {
    if (max_rg >= 4 && 10 * n >= 24LL * total_warps) return 4;  // n / 4 >= 0.6 warps
    if (max_rg >= 2 && n >= total_warps) return 2;              // n / 2 >= 0.5 warps
    return 1;
}

template <int FMT, int NMAT, int RG, int EPI>
qg_status launch_pick(const Params& p0, const DeviceInfo& dev, cudaStream_t stream) {
    // The ring kernel copies side data (scales, biases) as 16-byte pieces of 8:
    // a row's count must be a multiple of 8; its ring must fit beside x in the
    // per-CTA budget, with x's raw bulk-copy buffer if there is room for it.
    Params p = p0;
    const bool even_sides = !Fmt<FMT>::kScales || (p.k / Fmt<FMT>::kBlock) % 8 == 0;
    if (even_sides) {
        p.x_bulk = (EPI & kEpiNormIn) ? 0 : 1;  // an RMSNorm input is computed, not copied
        if (x_smem_bytes(FMT, p) + ring_smem_bytes<FMT, NMAT, RG>() <= kSmemPerCtaBudget)
            return launch_t<FMT, NMAT, RG, EPI, true>(p, dev, stream);
        p.x_bulk = 0;
        if (x_smem_bytes(FMT, p) + ring_smem_bytes<FMT, NMAT, RG>() <= kSmemPerCtaBudget)
            return launch_t<FMT, NMAT, RG, EPI, true>(p, dev, stream);
    }
    p.x_bulk = 0;
    if constexpr (Fmt<FMT>::kScales) {
        return launch_t<FMT, NMAT, RG, EPI, false>(p, dev, stream);
    } else {
        return QG_ERR_SHAPE;  // fp16 weights run on the ring path only
    }
}

// Launch one S=1 call of format FMT.  PLAIN is the single-weight epilogue
// (kEpiPlain, or kEpiResidual for the residual-stream update); XF adds
// kEpiNormIn when x is the RMSNorm of an fp32 hidden state.
// Rows (or gate/up pairs) per warp item times the most items any warp gets:
// the warp makespan, in rows, of round-robin items over tw warps.  Items of
// three rows are taken (int8) when they cut that makespan by a quarter or
// more against the measured rule above: timed on B200, the 2B gate/up (6144
// pairs on 2368 warps: 4 -> 3 pairs for the busiest warp), the 4B / 8B q|k|v
// and the 27B o and down, sweeps 2B / 4B / 8B / 27B +2.7 / +2.0 / +0.5 / +6.4%.
inline int64_t makespan_rows(int64_t n, int rg, int tw) {
    const int64_t items = (n + rg - 1) / rg;
    return (items + tw - 1) / tw * rg;
}

// Three-row items (int8) run on the shared-memory ring only, with x by bulk
// copy unless x is an RMSNorm input; callers check that this fits first.
template <int NMAT, int EPI>
bool ring3_fits(const Params& p0) {
    Params p = p0;
    p.x_bulk = (EPI & kEpiNormIn) ? 0 : 1;
    return (p.k / Fmt<0>::kBlock) % 8 == 0 &&
           x_smem_bytes(0, p) + ring_smem_bytes<0, NMAT, 3>() <= kSmemPerCtaBudget;
}
template <int NMAT, int EPI>
qg_status launch_ring3(const Params& p0, const DeviceInfo& dev, cudaStream_t stream) {
    Params p = p0;
    p.x_bulk = (EPI & kEpiNormIn) ? 0 : 1;
    return launch_t<0, NMAT, 3, EPI, true>(p, dev, stream);
}

template <int FMT, int PLAIN = kEpiPlain, int XF = 0>
qg_status dispatch_fmt(const GemvLaunch& L, const Params& p, const DeviceInfo& dev,
                       cudaStream_t stream) {
    const int tw = dev.num_sms * kCtasPerSm * kWarps;
    const int rg = pick_rg(L.n, 4, tw);
    if constexpr (PLAIN == kEpiPlain) {
        if (L.epilogue == kEpiSwiglu) {
            if constexpr (FMT == 2) {
                return QG_ERR_FORMAT;  // fp16 weights: GEMV and head only
            } else {
                const int rg2 = pick_rg(L.n, 2, tw);
                if constexpr (FMT == 0) {
                    if (4 * makespan_rows(L.n, 3, tw) <= 3 * makespan_rows(L.n, rg2, tw) &&
                        ring3_fits<2, kEpiSwiglu | XF>(p))
                        return launch_ring3<2, kEpiSwiglu | XF>(p, dev, stream);
                }
                if (rg2 == 2)
                    return launch_pick<FMT, 2, 2, kEpiSwiglu | XF>(p, dev, stream);
                return launch_pick<FMT, 2, 1, kEpiSwiglu | XF>(p, dev, stream);
            }
        }
        if (L.epilogue == kEpiHead) {
            if (rg == 4) return launch_pick<FMT, 1, 4, kEpiHead | XF>(p, dev, stream);
            if (rg == 2) return launch_pick<FMT, 1, 2, kEpiHead | XF>(p, dev, stream);
            return launch_pick<FMT, 1, 1, kEpiHead | XF>(p, dev, stream);
        }
    }
    if constexpr (FMT == 0) {
        if (4 * makespan_rows(L.n, 3, tw) <= 3 * makespan_rows(L.n, rg, tw) &&
            ring3_fits<1, PLAIN | XF>(p))
            return launch_ring3<1, PLAIN | XF>(p, dev, stream);
    }
    if (rg == 4) return launch_pick<FMT, 1, 4, PLAIN | XF>(p, dev, stream);
    if (rg == 2) return launch_pick<FMT, 1, 2, PLAIN | XF>(p, dev, stream);
    return launch_pick<FMT, 1, 1, PLAIN | XF>(p, dev, stream);
}

Params make_params(const GemvLaunch& L) {
    Params p = {};
    for (int m = 0; m < 2; ++m) {
        const int src = m < L.nmat ? m : 0;
        p.codes[m] = static_cast<const uint8_t*>(L.codes[src]);
        p.scales[m] = L.scales[src];
        p.biases[m] = L.biases[src];
    }
    p.n = L.n;
    p.k = L.k;
    p.x = L.x;
    p.y = L.y;
    p.y16 = L.y16;
    p.h = L.h;
    p.logits = L.logits;
    p.idx = L.idx;
    p.h_in = L.h_in;
    p.gamma = L.gamma;
    p.eps = L.eps;
    p.h_res = L.h_res;
    p.ws_key = static_cast<unsigned long long*>(L.workspace);
    p.ws_ticket = L.workspace
                      ? reinterpret_cast<unsigned int*>(static_cast<char*>(L.workspace) + 8)
                      : nullptr;
    const int cpl = L.fmt == QG_FMT_I8_B32 ? Fmt<0>::kCodesPerLane
                    : (L.fmt == QG_FMT_I4_G64 ? Fmt<1>::kCodesPerLane : Fmt<2>::kCodesPerLane);
    const int granules = static_cast<int>(L.k / cpl);
    p.x_words = align_up(granules, 8) * cpl / 2;  // fp16 x, padded to whole 8-granule phases
    return p;
}

}  // namespace
}  // namespace qg
