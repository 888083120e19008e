// qg_gemv.cu -- the S=1 decode weight stream on sm_100a.
//
// One kernel family computes y = W_dq x for an int8 block-32 or int4
// group-64 weight, with three epilogues: plain (fp32 and/or fp16 out), fused
// gate/up SwiGLU (two weights, fp16 h out) and fused LM-head argmax.  The
// pages ("Qwen3-VL 4B -- Core AI (.aimodel)", Measured) state that decode is
// bound by reading the weights once per token, so the design goal is to keep
// HBM busy:
//
//  * Persistent CTAs (one per SM, 8 warps).  Every warp owns a private ring of
//    STAGES shared-memory stages and streams its rows through it with 1-D bulk
//    async copies (cp.async.bulk, mbarrier completion, L2 evict-first, never
//    multicast).  A stage is RG rows (x NMAT weights) by 512 code bytes plus
//    the matching fp16 scales (and biases).  Bytes in flight per SM =
//    8 warps x STAGES x stage size, independent of registers.
//  * The activation x (fp16) is staged once per CTA into shared memory as
//    fp32, laid out so that each lane's 16-byte reads are bank-conflict free.
//  * Dequantization happens in registers with no int->float conversion
//    instruction: int8 codes become floats by byte-permuting them into the
//    mantissa of 2^23 and subtracting the offset; int4 nibbles by masking them
//    into that mantissa in place.  Products accumulate in fp32 with the packed
//    sm_100 f32x2 FMA; each block's fp16 scale is applied once per 16/32
//    codes; the int4 bias uses sum_k (q s + b) x = s sum q x + b sum x with
//    the per-half-group sum of x computed once per CTA.
//  * Lanes split K within a row; a warp-shuffle reduction finishes each row.
//  * Programmatic dependent launch: the weight prologue (first STAGES bulk
//    copies) is issued before griddepcontrol.wait, so a kernel's weight
//    stream overlaps the tail of the previous kernel in the stream; only the
//    x staging waits for it.
#include <cfloat>
#include <climits>

#include "qg_device.cuh"
#include "qg_internal.h"

namespace qg {

QG_DEFINE_ERROR_FLAG(g_gemv_err);

namespace {

constexpr int kLanes = 32;
constexpr int kNumWarps = 8;
constexpr int kStages = 4;
constexpr int kStageRowBytes = 512;   // code bytes per row per stage
constexpr int kStageSideBytes = 32;   // scale (or bias) bytes per row per stage

template <int FMT>
struct Fmt {
    static constexpr int kCodesPerStage = FMT == 0 ? 512 : 1024;
    static constexpr int kCodesPerLane = FMT == 0 ? 16 : 32;
    static constexpr int kBlock = FMT == 0 ? 32 : 64;
    static constexpr int kPieces = kCodesPerLane / 4;  // float4 pieces of x per lane
    static constexpr bool kBias = FMT == 1;
};

template <int FMT, int ROWS>
struct Stage {
    static constexpr int kCodes = ROWS * kStageRowBytes;
    static constexpr int kScales = ROWS * kStageSideBytes;
    static constexpr int kBiases = Fmt<FMT>::kBias ? ROWS * kStageSideBytes : 0;
    static constexpr int kBytes = kCodes + kScales + kBiases;
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
    int x_floats;  // floats reserved for x in shared memory
};

__host__ __device__ constexpr int align_up(int v, int a) { return (v + a - 1) / a * a; }
__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

// ------------------------------------------------------------ dot products --
// 16 int8 codes (one 16-byte vector) against 16 fp32 activations.
__device__ __forceinline__ float dot16_i8(const uint4 c, const float4* xv) {
    const float2 off = make_float2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)
    float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t u = w[i] ^ 0x80808080u;  // two's complement -> q + 128
        const float f0 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7440));
        const float f1 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7441));
        const float f2 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7442));
        const float f3 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7443));
        const float2 q01 = __fadd2_rn(make_float2(f0, f1), off);  // exact q
        const float2 q23 = __fadd2_rn(make_float2(f2, f3), off);
        a0 = __ffma2_rn(q01, make_float2(xv[i].x, xv[i].y), a0);
        a1 = __ffma2_rn(q23, make_float2(xv[i].z, xv[i].w), a1);
    }
    return (a0.x + a0.y) + (a1.x + a1.y);
}

// 32 int4 codes (one 16-byte vector) against 32 activations that the staging
// step stored per 8-code word as (x0, x5, x1, x6, x2, x7, x3, x4/16): nibble j
// is masked in place into the mantissa of 2^23, giving 2^23 + n_j 16^e_j, and
// the accumulators are kept per power of 16 and rescaled exactly at the end.
__device__ __forceinline__ float dot32_i4(const uint4 c, const float4* xv) {
    const float2 off = make_float2(-8388608.0f, -8388608.0f);  // -2^23
    const uint32_t M = 0x4B000000u;
    float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0, a3 = a0;
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t v = w[i];
        const uint32_t s = v >> 20;
        const float n0 = __uint_as_float((v & 0x0000000Fu) | M);   // n0
        const float n1 = __uint_as_float((v & 0x000000F0u) | M);   // 16 n1
        const float n2 = __uint_as_float((v & 0x00000F00u) | M);   // 256 n2
        const float n3 = __uint_as_float((v & 0x0000F000u) | M);   // 4096 n3
        const float n4 = __uint_as_float((v & 0x000F0000u) | M);   // 65536 n4
        const float n5 = __uint_as_float((s & 0x0000000Fu) | M);   // n5
        const float n6 = __uint_as_float((s & 0x000000F0u) | M);   // 16 n6
        const float n7 = __uint_as_float((s & 0x00000F00u) | M);   // 256 n7
        const float4 xa = xv[2 * i], xb = xv[2 * i + 1];
        a0 = __ffma2_rn(__fadd2_rn(make_float2(n0, n5), off), make_float2(xa.x, xa.y), a0);
        a1 = __ffma2_rn(__fadd2_rn(make_float2(n1, n6), off), make_float2(xa.z, xa.w), a1);
        a2 = __ffma2_rn(__fadd2_rn(make_float2(n2, n7), off), make_float2(xb.x, xb.y), a2);
        a3 = __ffma2_rn(__fadd2_rn(make_float2(n3, n4), off), make_float2(xb.z, xb.w), a3);
    }
    return ((a0.x + a0.y) + (a1.x + a1.y) * 0.0625f) +
           ((a2.x + a2.y) * 0.00390625f + (a3.x + a3.y) * 0.000244140625f);
}

// float4 index of piece `i` of lane-granule `g` in the staged x: the eight
// granules read by one 8-lane phase of an LDS.128 are adjacent.
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

template <int FMT, int NMAT, int RG, int EPI, bool SC_TMA>
__global__ void __launch_bounds__(kNumWarps* kLanes, 1) gemv_s1_kernel(const Params p) {
    using F = Fmt<FMT>;
    constexpr int ROWS = NMAT * RG;
    using L = Stage<FMT, ROWS>;
    constexpr int kBarBytes = align_up(kNumWarps * kStages * 8, 128);

    extern __shared__ __align__(128) unsigned char smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem) + warp * kStages;
    unsigned char* ring = smem + kBarBytes + warp * kStages * L::kBytes;
    float* xs = reinterpret_cast<float*>(smem + kBarBytes + kNumWarps * kStages * L::kBytes);
    float* hsum = xs + p.x_floats;  // int4: per-lane-granule sum of x
    __shared__ float red_v[kNumWarps];
    __shared__ int red_i[kNumWarps];

    const int64_t N = p.n, K = p.k;
    const int nst = static_cast<int>((K + F::kCodesPerStage - 1) / F::kCodesPerStage);
    const int64_t items = (N + RG - 1) / RG;
    const int64_t wg = static_cast<int64_t>(blockIdx.x) * kNumWarps + warp;
    const int64_t tw = static_cast<int64_t>(gridDim.x) * kNumWarps;
    const int64_t my_items = wg < items ? (items - wg + tw - 1) / tw : 0;
    const int64_t total = my_items * nst;
    const int64_t row_bytes = FMT == 0 ? K : K / 2;
    const int64_t side_per_row = K / F::kBlock;  // fp16 scales (biases) per row

    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    const uint64_t pol = l2_policy_evict_first();

    // Producer step (lane 0): bring stage t of this warp's sequence into slot
    // t % kStages.  Stage t is (item t / nst, K-chunk t % nst).
    auto issue = [&](int64_t t) {
        const int64_t il = t / nst;
        const int st = static_cast<int>(t - il * nst);
        const int64_t r0 = (wg + il * tw) * RG;
        const int rows = static_cast<int>(min64(RG, N - r0));
        const int64_t k0 = static_cast<int64_t>(st) * F::kCodesPerStage;
        const int kc = static_cast<int>(min64(F::kCodesPerStage, K - k0));
        const uint32_t cbytes = FMT == 0 ? kc : kc / 2;
        const uint32_t sbytes = static_cast<uint32_t>(kc / F::kBlock) * 2u;
        unsigned char* stage = ring + (t % kStages) * L::kBytes;
        uint64_t* bar = &bars[t % kStages];
        uint32_t tx = cbytes;
        if (SC_TMA) tx += F::kBias ? 2u * sbytes : sbytes;
        mbar_arrive_expect_tx(bar, tx * static_cast<uint32_t>(rows * NMAT));
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
            for (int j = 0; j < rows; ++j) {
                const int64_t r = r0 + j;
                const int slot_row = m * RG + j;
                bulk_g2s(stage + slot_row * kStageRowBytes,
                         p.codes[m] + r * row_bytes + (FMT == 0 ? k0 : k0 / 2), cbytes, bar, pol);
                if (SC_TMA) {
                    const int64_t so = r * side_per_row + k0 / F::kBlock;
                    bulk_g2s(stage + L::kCodes + slot_row * kStageSideBytes, p.scales[m] + so,
                             sbytes, bar, pol);
                    if (F::kBias)
                        bulk_g2s(stage + L::kCodes + L::kScales + slot_row * kStageSideBytes,
                                 p.biases[m] + so, sbytes, bar, pol);
                }
            }
        }
    };

    // 1) weight prologue: independent of the previous kernel in the stream.
    if (lane == 0) {
        const int64_t pre = total < kStages ? total : kStages;
        for (int64_t t = 0; t < pre; ++t) issue(t);
    }

    // 2) the activation is produced by the previous kernel: wait for it, then
    //    stage it as fp32 in the conflict-free layout (int4: pair-permuted and
    //    with the half-group sums).
    griddep_wait();
    {
        const int granules = static_cast<int>(K / F::kCodesPerLane);
        for (int g = threadIdx.x; g < granules; g += blockDim.x) {
            const uint16_t* xg = p.x + static_cast<int64_t>(g) * F::kCodesPerLane;
            float4* xs4 = reinterpret_cast<float4*>(xs);
            float gsum = 0.f;
#pragma unroll
            for (int c = 0; c < F::kCodesPerLane / 8; ++c) {
                const uint4 v = *reinterpret_cast<const uint4*>(xg + 8 * c);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                float a[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    a[2 * e] = h2f(static_cast<uint16_t>(w[e] & 0xFFFFu));
                    a[2 * e + 1] = h2f(static_cast<uint16_t>(w[e] >> 16));
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) gsum += a[e];
                if (FMT == 0) {
                    xs4[x_piece<FMT>(g, 2 * c)] = make_float4(a[0], a[1], a[2], a[3]);
                    xs4[x_piece<FMT>(g, 2 * c + 1)] = make_float4(a[4], a[5], a[6], a[7]);
                } else {
                    // one 8-code word: (x0, x5, x1, x6) (x2, x7, x3, x4/16)
                    xs4[x_piece<FMT>(g, 2 * c)] = make_float4(a[0], a[5], a[1], a[6]);
                    xs4[x_piece<FMT>(g, 2 * c + 1)] =
                        make_float4(a[2], a[7], a[3], a[4] * 0.0625f);
                }
            }
            if (FMT == 1) hsum[g] = gsum;
        }
    }
    __syncthreads();
    griddep_launch_dependents();

    // 3) consume.
    float acc[ROWS];
#pragma unroll
    for (int j = 0; j < ROWS; ++j) acc[j] = 0.f;
    float best_v = -FLT_MAX;
    int best_i = INT_MAX;
    bool failed = false;

    int64_t t = 0;
    for (int64_t il = 0; il < my_items && !failed; ++il) {
        const int64_t r0 = (wg + il * tw) * RG;
        for (int st = 0; st < nst; ++st, ++t) {
            unsigned char* stage = ring + (t % kStages) * L::kBytes;
            const bool ok = mbar_wait_bounded(&bars[t % kStages],
                                              static_cast<uint32_t>((t / kStages) & 1));
            if (!__all_sync(0xffffffffu, ok)) {
                failed = true;
                break;
            }
            const int g = st * kLanes + lane;  // lane-granule index within the row
            if (static_cast<int64_t>(g) * F::kCodesPerLane < K) {
                float4 xv[F::kPieces];
                const float4* xs4 = reinterpret_cast<const float4*>(xs);
#pragma unroll
                for (int i = 0; i < F::kPieces; ++i) xv[i] = xs4[x_piece<FMT>(g, i)];
                const float hs = FMT == 1 ? hsum[g] : 0.f;
#pragma unroll
                for (int j = 0; j < ROWS; ++j) {
                    const uint4 c =
                        *reinterpret_cast<const uint4*>(stage + j * kStageRowBytes + lane * 16);
                    uint16_t sb, bb = 0;
                    if (SC_TMA) {
                        sb = *reinterpret_cast<const uint16_t*>(stage + L::kCodes +
                                                                j * kStageSideBytes + (lane >> 1) * 2);
                        if (F::kBias)
                            bb = *reinterpret_cast<const uint16_t*>(
                                stage + L::kCodes + L::kScales + j * kStageSideBytes + (lane >> 1) * 2);
                    } else {
                        const int m = j / RG;
                        const int64_t r = min64(r0 + (j % RG), N - 1);
                        const int64_t so = r * side_per_row +
                                           (static_cast<int64_t>(g) * F::kCodesPerLane) / F::kBlock;
                        sb = ldg_nc_u16(p.scales[m] + so);
                        if (F::kBias) bb = ldg_nc_u16(p.biases[m] + so);
                    }
                    if (FMT == 0) {
                        acc[j] = fmaf(h2f(sb), dot16_i8(c, xv), acc[j]);
                    } else {
                        acc[j] = fmaf(h2f(sb), dot32_i4(c, xv), fmaf(h2f(bb), hs, acc[j]));
                    }
                }
            }
            __syncwarp();
            if (lane == 0 && t + kStages < total) {
                fence_proxy_async_smem();
                issue(t + kStages);
            }
        }
        if (failed) break;

        // item epilogue: finish the rows across lanes.
#pragma unroll
        for (int j = 0; j < ROWS; ++j) acc[j] = warp_sum(acc[j]);
        if (lane < RG && r0 + lane < N) {
            const int64_t r = r0 + lane;
            float v0 = acc[0], v1 = 0.f;
#pragma unroll
            for (int j = 0; j < RG; ++j)
                if (lane == j) {
                    v0 = acc[j];
                    if (NMAT == 2) v1 = acc[(NMAT - 1) * RG + j];
                }
            if (EPI == kEpiPlain) {
                if (p.y) p.y[r] = v0;
                if (p.y16) p.y16[r] = f2h_rn(v0);
            } else if (EPI == kEpiSwiglu) {
                const float sg = v0 / (1.0f + expf(-v0));
                p.h[r] = f2h_rn(sg * v1);
            } else {
                if (p.logits) p.logits[r] = v0;
                if (v0 > best_v) {  // rows arrive in increasing order per lane
                    best_v = v0;
                    best_i = static_cast<int>(r);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < ROWS; ++j) acc[j] = 0.f;
    }

    if (failed) {
        // Drain: wait (bounded) for this warp's copies still in flight so no
        // bulk copy targets shared memory after the CTA exits.
        if (lane == 0) {
            atomicOr(&g_gemv_err, 1u);
            const int64_t issued_end = min64(total, t + kStages);
            for (int64_t u = t; u < issued_end; ++u)
                mbar_wait_bounded(&bars[u % kStages], static_cast<uint32_t>((u / kStages) & 1));
        }
        __syncwarp();
    }

    if (EPI == kEpiHead) {
        // lane -> warp -> CTA (value, lowest index), then one atomicMax per CTA
        // and a ticket: the last CTA publishes the index and re-zeroes the
        // workspace.  No CTA ever waits on another.
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
            for (int w = 1; w < kNumWarps; ++w)
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
}

template <int FMT, int NMAT, int RG, int EPI, bool SC>
size_t smem_bytes(const Params& p) {
    using L = Stage<FMT, NMAT * RG>;
    size_t b = align_up(kNumWarps * kStages * 8, 128);
    b += static_cast<size_t>(kNumWarps) * kStages * L::kBytes;
    b += static_cast<size_t>(p.x_floats) * 4;
    if (FMT == 1) b += static_cast<size_t>(p.k / Fmt<1>::kCodesPerLane) * 4;
    return b;
}

template <int FMT, int NMAT, int RG, int EPI, bool SC>
qg_status launch_t(const Params& p, const DeviceInfo& dev, cudaStream_t stream) {
    auto kern = gemv_s1_kernel<FMT, NMAT, RG, EPI, SC>;
    const size_t smem = smem_bytes<FMT, NMAT, RG, EPI, SC>(p);
    if (smem + 1024 > static_cast<size_t>(dev.max_smem_optin)) return QG_ERR_SHAPE;
    // Opt in to exactly the dynamic shared memory this launch needs (static
    // shared memory counts against the same per-block limit).
    static size_t attr_set[64] = {0};
    if (dev.device >= 64 || attr_set[dev.device] < smem) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return cuda_status(e);
        if (dev.device < 64) attr_set[dev.device] = smem;
    }
    const int64_t items = (p.n + RG - 1) / RG;
    int64_t grid = (items + kNumWarps - 1) / kNumWarps;
    if (grid > dev.num_sms) grid = dev.num_sms;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kNumWarps * kLanes);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, p));
}

// Rows per warp item: as many as still leave every warp of the grid at least
// two items, so small matrices spread over all SMs.
int pick_rg(int64_t n, int max_rg, int total_warps) {
    if (max_rg >= 4 && n >= 8LL * total_warps) return 4;
    if (max_rg >= 2 && n >= 2LL * total_warps) return 2;
    return 1;
}

template <int FMT, bool SC>
qg_status dispatch_fmt(const GemvLaunch& L, const Params& p, const DeviceInfo& dev,
                       cudaStream_t stream) {
    const int tw = dev.num_sms * kNumWarps;
    if (L.epilogue == kEpiSwiglu) {
        const int rg = pick_rg(L.n, 2, tw);
        if (rg == 2) return launch_t<FMT, 2, 2, kEpiSwiglu, SC>(p, dev, stream);
        return launch_t<FMT, 2, 1, kEpiSwiglu, SC>(p, dev, stream);
    }
    const int rg = pick_rg(L.n, 4, tw);
    if (L.epilogue == kEpiHead) {
        if (rg == 4) return launch_t<FMT, 1, 4, kEpiHead, SC>(p, dev, stream);
        if (rg == 2) return launch_t<FMT, 1, 2, kEpiHead, SC>(p, dev, stream);
        return launch_t<FMT, 1, 1, kEpiHead, SC>(p, dev, stream);
    }
    if (rg == 4) return launch_t<FMT, 1, 4, kEpiPlain, SC>(p, dev, stream);
    if (rg == 2) return launch_t<FMT, 1, 2, kEpiPlain, SC>(p, dev, stream);
    return launch_t<FMT, 1, 1, kEpiPlain, SC>(p, dev, stream);
}

}  // namespace

qg_status launch_gemv_s1(const GemvLaunch& L, cudaStream_t stream) {
    DeviceInfo dev;
    qg_status st = device_info(&dev);
    if (st != QG_OK) return st;
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
    p.ws_key = static_cast<unsigned long long*>(L.workspace);
    p.ws_ticket = L.workspace
                      ? reinterpret_cast<unsigned int*>(static_cast<char*>(L.workspace) + 8)
                      : nullptr;
    const int cpl = L.fmt == QG_FMT_I8_B32 ? Fmt<0>::kCodesPerLane : Fmt<1>::kCodesPerLane;
    const int granules = static_cast<int>(L.k / cpl);
    p.x_floats = align_up(granules, 8) * cpl;

    // Scales (and biases) ride the bulk copies when every per-row, per-stage
    // window of them is 16-byte aligned; otherwise lanes load them directly.
    if (L.fmt == QG_FMT_I8_B32) {
        if (L.k % 256 == 0) return dispatch_fmt<0, true>(L, p, dev, stream);
        return dispatch_fmt<0, false>(L, p, dev, stream);
    }
    if (L.k % 512 == 0) return dispatch_fmt<1, true>(L, p, dev, stream);
    return dispatch_fmt<1, false>(L, p, dev, stream);
}

unsigned int gemv_read_and_clear_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_gemv_err, sizeof v) != cudaSuccess) return 0;
    if (v) cudaMemcpyToSymbol(g_gemv_err, &zero, sizeof zero);
    return v;
}

}  // namespace qg
