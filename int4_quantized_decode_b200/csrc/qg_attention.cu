// qg_attention.cu -- the attention core of one decode step over an fp16 K/V
// cache, for the pages' Qwen3-VL decoders ("Qwen3-VL (2B / 4B / 8B,
// vision-language) -- Core AI", architecture paragraph: pure attention,
// head_dim 128, 8 kv heads, rope theta 5e6; "Qwen3-VL 4B & 8B -- Core ML
// stateful", gotchas: for text positions the interleaved M-RoPE is standard
// 1-D RoPE, the rotary helper pairing the two halves of a head; "Qwen3-VL 2B
// -- Core AI", integration checklist: the KV cache is the native K/V pair).
//
//   q_h = RoPE(q_h, pos),  k = fp16(RoPE(k, pos)),  v = fp16(v)  (appended at row pos)
//   o_h = sum_{j <= pos} softmax_j( q_h . K[g][j] / sqrt(d) ) V[g][j],  g = h / (hq / hkv)
//
// Like the weight stream, this is a bandwidth-bound read (every cached row
// once per token), split the flash-decoding way:
//  * grid = splits x kv heads; a CTA takes one contiguous chunk of the
//    positions 0..pos of one kv head and all G query heads that read it, so
//    each K/V row is read once per token;
//  * one CTA per SM: a producer warp streams the chunk through a six-stage
//    ring, 64 rows of K then 64 of V per stage, each stage two 1-D bulk copies
//    completing on the stage's mbarrier (the rows of one kv head are
//    contiguous), after an L2 prefetch of the chunk's first rows issued before
//    the wait on the previous kernel;
//  * eight compute warps take 8 rows of every stage each: 8 lanes per row
//    (16 dims per lane, two 16-byte shared loads), a score per query head
//    summed over the 8 lanes, softmax in base 2 (log2 e folded into q) with a
//    running maximum per warp that is raised, and the state rescaled, only
//    when a score exceeds it by more than 8 (so every weight stays <= 2^8);
//    warps then merge their (max, sum, acc) states in shared memory;
//  * every CTA writes its partial state; the last CTA of a kv head (an atomic
//    ticket, no CTA ever waits) merges the splits in one pass, writes o in fp16
//    and re-zeroes its ticket;
//  * the new token's key and value are computed by every CTA (RoPE angles in
//    fp64, one fp16 rounding) and stand in for row pos, which no CTA reads from
//    the cache; the CTA whose chunk holds pos writes them into the cache once
//    its own copies have landed.
#include <cfloat>
#include <cmath>

#include "qg_device.cuh"
#include "qg_internal.h"

namespace qg {

QG_DEFINE_ERROR_FLAG(g_attn_err);  // bit 0: position out of range; bit 1: a wait expired

namespace {

constexpr int kD = 128;               // head_dim of the pages' Qwen3-VL decoders
constexpr int kRowBytes = kD * 2;     // one fp16 row of K or V
constexpr int kLanesPerRow = 8;       // a row's 128 dims over 8 lanes
constexpr int kRowGroups = 32 / kLanesPerRow;        // 4 rows in flight per warp
constexpr int kComputeWarps = 8;
constexpr int kComputeThreads = kComputeWarps * 32;
constexpr int kThreadsA = kComputeThreads + 32;      // + the producer warp
constexpr int kStageRows = 64;
constexpr int kRowsPerWarp = kStageRows / kComputeWarps;   // 8
constexpr int kRowsPerGroup = kRowsPerWarp / kRowGroups;   // 2 rows per lane group per stage
constexpr int kStages = 6;
constexpr int kStageBytes = 2 * kStageRows * kRowBytes;    // K rows, then V rows: 32 KB
constexpr int kRingBytesA = kStages * kStageBytes;          // 192 KB
constexpr int kMaxSplitsK = 32;       // splits of one kv head's rows, at most
constexpr int kPrefetchRows = 256;    // rows of a chunk prefetched into L2
constexpr float kLazyRescale = 8.f;   // base-2 headroom of the running maximum
constexpr double kLog2e = 1.4426950408889634;
constexpr int kComputeBar = 1;        // named barrier of the compute warps
static_assert(kStageRows % (kComputeWarps * kRowGroups) == 0, "whole rows per lane group");

struct AttnParams {
    const float* qkv;
    uint16_t* kc;
    uint16_t* vc;
    uint16_t* o;
    const int32_t* pos;
    float* part;              // [hkv][splits][G][kD + 2]: m (base 2), l, acc
    unsigned int* ticket;     // [hkv]
    int64_t l_max;
    int hq, hkv, splits;
    double theta;
    double qscale;            // log2(e) / sqrt(d): scores in base 2
};

__device__ __forceinline__ void prefetch_l2_a(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ uint4 lds128_a(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a));
    return v;
}
// 2^x (the hardware approximation; -inf gives +0)
__device__ __forceinline__ float ex2_a(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// two fp32 lanes in one 64-bit register: the packed FMA does both products
__device__ __forceinline__ uint64_t pack2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void unpack2(uint64_t r, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// The ticket: release orders this CTA's partial stores (seen by the calling
// thread through the CTA barrier before it) ahead of the increment; acquire
// orders the other CTAs' partials ahead of the reads that follow the barrier
// after it.
__device__ __forceinline__ unsigned int atom_add_acq_rel_gpu(unsigned int* p, unsigned int v) {
    unsigned int old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
                 : "memory");
    return old;
}
__device__ __forceinline__ void compute_bar() {
    asm volatile("bar.sync %0, %1;" ::"n"(kComputeBar), "n"(kComputeThreads) : "memory");
}

// Rows [j0, j1) of split `split` when the token is at pos (empty past the end).
__device__ __forceinline__ void chunk_of(int64_t pos, int splits, int split, int64_t& j0,
                                         int64_t& j1) {
    const int64_t n = pos + 1;
    const int64_t chunk = (n + splits - 1) / splits;
    j0 = split * chunk;
    j1 = j0 >= n ? j0 : (j0 + chunk < n ? j0 + chunk : n);  // empty past the end
}

__device__ __forceinline__ void unpack8h(const uint4 a, float* out) {
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        out[2 * i] = h2f(static_cast<uint16_t>(w[i] & 0xFFFFu));
        out[2 * i + 1] = h2f(static_cast<uint16_t>(w[i] >> 16));
    }
}

template <int G>
__global__ void __launch_bounds__(kThreadsA, 1) decode_attention_kernel(const AttnParams p) {
    __shared__ float q_s[G][kD];
    __shared__ __align__(16) uint16_t kn_h[kD];
    __shared__ __align__(16) uint16_t vn_h[kD];
    __shared__ float wst[kComputeWarps][G][kD + 2];  // per-warp states
    __shared__ __align__(8) uint64_t full_bar[kStages];
    __shared__ __align__(8) uint64_t empty_bar[kStages];
    __shared__ unsigned int last_s;
    __shared__ float sm_m[kMaxSplitsK][G];  // split maxima (the last CTA)
    __shared__ float sm_l[kMaxSplitsK][G];  // split sums
    extern __shared__ __align__(128) unsigned char ring[];

    const int split = blockIdx.x, g = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], kComputeWarps);
        }
        fence_mbar_init();
    }

    // Before the wait on the previous kernel: ask L2 for the first rows of
    // this CTA's chunk (at most kPrefetchRows, so that long caches do not
    // overflow L2).  A prefetch is only a hint (L2 stays coherent with whatever
    // the previous kernel writes), and the position is read again after the wait.
    const int32_t pg = *reinterpret_cast<const volatile int32_t*>(p.pos);
    // RoPE angles a_i = pos * theta^(-2i/d) in fp64 for that early read of the
    // position (thread i < d/2 keeps pair i's cos and sin in registers)
    double rc = 1.0, rs = 0.0;
    auto angles = [&](int32_t at) {
        const double f = pow(p.theta, -2.0 * static_cast<double>(tid) / kD);
        sincos(static_cast<double>(at) * f, &rs, &rc);
    };
    if (tid < kD / 2 && pg >= 0 && pg < p.l_max) angles(pg);
    if (lane == 0 && warp < kComputeWarps && pg >= 0 && pg < p.l_max) {
        int64_t a0, a1;
        chunk_of(pg, p.splits, split, a0, a1);
        if (a1 > a0 + kPrefetchRows) a1 = a0 + kPrefetchRows;
        // warp w prefetches its eighth of those rows, in pieces of <= 16 KB
        const int64_t q0 = a0 + (a1 - a0) * warp / kComputeWarps;
        const int64_t q1 = a0 + (a1 - a0) * (warp + 1) / kComputeWarps;
        for (int64_t r = q0; r < q1; r += 64) {
            const int64_t rows = q1 - r < 64 ? q1 - r : 64;
            const int64_t off = (static_cast<int64_t>(g) * p.l_max + r) * kD;
            prefetch_l2_a(p.kc + off, static_cast<uint32_t>(rows * kRowBytes));
            prefetch_l2_a(p.vc + off, static_cast<uint32_t>(rows * kRowBytes));
        }
    }
    __syncthreads();  // the barriers are initialised
    griddep_wait();   // q|k|v come from the projection kernel before this one
    const int32_t pos = *p.pos;
    // the new token's inputs, loaded together with the position
    double k0 = 0.0, k1 = 0.0, q0[G], q1[G];
    float vin = 0.f;
    if (tid < kD / 2) {
        const float* kin = p.qkv + static_cast<int64_t>(p.hq) * kD + g * kD;
        k0 = kin[tid];
        k1 = kin[tid + kD / 2];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float* qin = p.qkv + static_cast<int64_t>(g * G + h) * kD;
            q0[h] = qin[tid];
            q1[h] = qin[tid + kD / 2];
        }
    } else if (tid < kD / 2 + kD) {
        vin = p.qkv[static_cast<int64_t>(p.hq + p.hkv) * kD + g * kD + (tid - kD / 2)];
    }
    if (pos < 0 || pos >= p.l_max) {
        if (tid == 0 && split == 0 && g == 0) atomicOr(&g_attn_err, 1u);
        return;
    }
    int64_t j0, j1;
    chunk_of(pos, p.splits, split, j0, j1);
    const int nstages = static_cast<int>((j1 - j0 + kStageRows - 1) / kStageRows);

    if (warp == kComputeWarps) {
        // ---- producer: stage st -> slot st % kStages, rows j0 + 64 st ... of K
        // then of V (row pos comes along with its old bytes and is never used)
        griddep_launch_dependents();
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            const uint16_t* kb = p.kc + (static_cast<int64_t>(g) * p.l_max + j0) * kD;
            const uint16_t* vb = p.vc + (static_cast<int64_t>(g) * p.l_max + j0) * kD;
            for (int st = 0; st < nstages; ++st) {
                const int slot = st % kStages;
                if (st >= kStages &&
                    !mbar_wait_bounded(&empty_bar[slot], ((st / kStages) - 1) & 1)) {
                    atomicOr(&g_attn_err, 2u);
                    break;
                }
                const int64_t r0 = static_cast<int64_t>(st) * kStageRows;
                const int64_t left = j1 - j0 - r0;
                const uint32_t bytes =
                    static_cast<uint32_t>(left < kStageRows ? left : kStageRows) * kRowBytes;
                unsigned char* dst = ring + slot * kStageBytes;
                mbar_arrive_expect_tx(&full_bar[slot], 2 * bytes);
                bulk_g2s(dst, kb + r0 * kD, bytes, &full_bar[slot], pol);
                bulk_g2s(dst + kStageRows * kRowBytes, vb + r0 * kD, bytes, &full_bar[slot], pol);
            }
        }
        return;
    }

    // ---- the new token: thread i < d/2 rotates pair i of the key (fp64,
    // rounded once to fp16) and of every query head that reads this kv head
    if (tid < kD / 2) {
        if (pos != pg) angles(pos);  // the position changed after the early read
        kn_h[tid] = __half_as_ushort(__double2half(k0 * rc - k1 * rs));
        kn_h[tid + kD / 2] = __half_as_ushort(__double2half(k1 * rc + k0 * rs));
#pragma unroll
        for (int h = 0; h < G; ++h) {
            q_s[h][tid] = static_cast<float>((q0[h] * rc - q1[h] * rs) * p.qscale);
            q_s[h][tid + kD / 2] = static_cast<float>((q1[h] * rc + q0[h] * rs) * p.qscale);
        }
    } else if (tid < kD / 2 + kD) {
        vn_h[tid - kD / 2] = f2h_rn(vin);
    }
    compute_bar();
    griddep_launch_dependents();

    // ---- stream: in each stage, warp w takes rows 8w .. 8w + 7; lane group
    // rg = lane / 8 takes rows 8w + rg and 8w + 4 + rg, lane gl = lane % 8 of
    // the group dims 8 gl .. 8 gl + 7 and 64 + 8 gl .. 64 + 8 gl + 7 (each
    // group's two 16-byte loads cover 128 contiguous bytes: no bank conflict)
    const int rg = lane / kLanesPerRow, gl = lane % kLanesPerRow;
    // the lane's 16 dims as 8 pairs: pair i < 4 holds dims 8 gl + 2i, + 1;
    // pair 4 + i dims 64 + 8 gl + 2i, + 1
    uint64_t q2[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            q2[h][i] = pack2(q_s[h][8 * gl + 2 * i], q_s[h][8 * gl + 2 * i + 1]);
            q2[h][4 + i] =
                pack2(q_s[h][kD / 2 + 8 * gl + 2 * i], q_s[h][kD / 2 + 8 * gl + 2 * i + 1]);
        }
    float m[G], l[G];
    uint64_t acc2[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc2[h][i] = 0ull;
    }
    const uint32_t ring0 = smem_u32(ring), kn_a = smem_u32(kn_h), vn_a = smem_u32(vn_h);
    for (int st = 0; st < nstages; ++st) {
        const int slot = st % kStages;
        if (!mbar_wait_bounded(&full_bar[slot], (st / kStages) & 1)) {
            if (lane == 0) atomicOr(&g_attn_err, 2u);
            break;
        }
        const uint32_t kst = ring0 + slot * kStageBytes;
        const uint32_t vst = kst + kStageRows * kRowBytes;
        const int64_t jb = j0 + static_cast<int64_t>(st) * kStageRows;
        float s[kRowsPerGroup][G];
        bool valid[kRowsPerGroup];
        uint32_t vaddr[kRowsPerGroup];
#pragma unroll
        for (int u = 0; u < kRowsPerGroup; ++u) {
            const int rr = warp * kRowsPerWarp + u * kRowGroups + rg;
            const int64_t j = jb + rr;
            valid[u] = j < j1;
            // row pos (and, with weight 0, rows past the chunk) read the new token
            const bool fresh = !valid[u] || j == pos;
            const uint32_t ka = fresh ? kn_a : kst + rr * kRowBytes;
            vaddr[u] = fresh ? vn_a : vst + rr * kRowBytes;
            float kf[16];
            unpack8h(lds128_a(ka + 16 * gl), kf);
            unpack8h(lds128_a(ka + kD + 16 * gl), kf + 8);
            uint64_t k2[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) k2[i] = pack2(kf[2 * i], kf[2 * i + 1]);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                uint64_t a2 = fma2(q2[h][0], k2[0], 0ull);
#pragma unroll
                for (int i = 1; i < 8; ++i) a2 = fma2(q2[h][i], k2[i], a2);
                float a0, a1;
                unpack2(a2, a0, a1);
                float a = a0 + a1;
                a += __shfl_xor_sync(0xffffffffu, a, 1);
                a += __shfl_xor_sync(0xffffffffu, a, 2);
                a += __shfl_xor_sync(0xffffffffu, a, 4);
                s[u][h] = a;
            }
        }
        // the warp's running maximum (the same in every lane) is raised only
        // when a score passes it by more than kLazyRescale
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float mx = -INFINITY;
#pragma unroll
            for (int u = 0; u < kRowsPerGroup; ++u)
                if (valid[u]) mx = fmaxf(mx, s[u][h]);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            if (mx > m[h] + kLazyRescale) {
                const float c = ex2_a(m[h] - mx);  // 0 while m is -inf
                const uint64_t c2 = pack2(c, c);
                l[h] *= c;
#pragma unroll
                for (int i = 0; i < 8; ++i) acc2[h][i] = mul2(acc2[h][i], c2);
                m[h] = mx;
            }
        }
#pragma unroll
        for (int u = 0; u < kRowsPerGroup; ++u) {
            float vf[16];
            unpack8h(lds128_a(vaddr[u] + 16 * gl), vf);
            unpack8h(lds128_a(vaddr[u] + kD + 16 * gl), vf + 8);
            uint64_t v2[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v2[i] = pack2(vf[2 * i], vf[2 * i + 1]);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float pj = valid[u] ? ex2_a(s[u][h] - m[h]) : 0.f;
                const uint64_t p2 = pack2(pj, pj);
                l[h] += pj;
#pragma unroll
                for (int i = 0; i < 8; ++i) acc2[h][i] = fma2(p2, v2[i], acc2[h][i]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[slot]);  // this warp is done with the slot
    }

    // ---- the warp's four lane groups share its maximum: sum their states
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float acc[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) unpack2(acc2[h][i], acc[2 * i], acc[2 * i + 1]);
        l[h] += __shfl_xor_sync(0xffffffffu, l[h], 8);
        l[h] += __shfl_xor_sync(0xffffffffu, l[h], 16);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 8);
            acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 16);
        }
        if (rg == 0) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                wst[warp][h][2 + 8 * gl + i] = acc[i];
                wst[warp][h][2 + kD / 2 + 8 * gl + i] = acc[8 + i];
            }
            if (gl == 0) {
                wst[warp][h][0] = m[h];
                wst[warp][h][1] = l[h];
            }
        }
    }
    compute_bar();

    // ---- merge the warps (thread t: dim t % 128 of head t / 128, and of head
    // t / 128 + 2 when G = 4) and write this split's partial
    float* part = p.part + (static_cast<int64_t>(g) * p.splits + split) * G * (kD + 2);
    for (int e = tid; e < G * kD; e += kComputeThreads) {
        const int h = e / kD, dim = e % kD;
        float mm = -INFINITY;
#pragma unroll
        for (int w = 0; w < kComputeWarps; ++w) mm = fmaxf(mm, wst[w][h][0]);
        float ll = 0.f, aa = 0.f;
#pragma unroll
        for (int w = 0; w < kComputeWarps; ++w) {
            const float mw = wst[w][h][0];
            const float c = mw == -INFINITY ? 0.f : ex2_a(mw - mm);
            ll = fmaf(c, wst[w][h][1], ll);
            aa = fmaf(c, wst[w][h][2 + dim], aa);
        }
        part[h * (kD + 2) + 2 + dim] = aa;
        if (dim == 0) {
            part[h * (kD + 2)] = mm;
            part[h * (kD + 2) + 1] = ll;
        }
    }
    // the CTA whose chunk holds pos appends the new rows (its copies have landed)
    if (pos >= j0 && pos < j1 && tid < kD) {
        const int64_t row = (static_cast<int64_t>(g) * p.l_max + pos) * kD;
        p.kc[row + tid] = kn_h[tid];
        p.vc[row + tid] = vn_h[tid];
    }

    // ---- the last CTA of this kv head merges the splits
    compute_bar();  // every partial of this CTA is stored
    if (tid == 0)
        last_s = atom_add_acq_rel_gpu(&p.ticket[g], 1u) == static_cast<unsigned int>(p.splits - 1);
    compute_bar();
    if (!last_s) return;
    // Every split's max and sum go to shared memory once; thread t owns
    // kDpt adjacent dims (d0 = kDpt t of the [G][128] outputs) and loads them
    // from every split, all in flight together; then per output
    // o = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s,  M = max_s m_s.
    const float* base = p.part + static_cast<int64_t>(g) * p.splits * G * (kD + 2);
    const int64_t stride = static_cast<int64_t>(G) * (kD + 2);
    constexpr int kDpt = G * kD > kComputeThreads ? G * kD / kComputeThreads : 1;
    static_assert(kDpt * kComputeThreads >= G * kD && kDpt <= 2, "one pass over the outputs");
    const int d0 = tid * kDpt;
    const bool mine = d0 < G * kD;
    const int h = mine ? d0 / kD : 0, dim = d0 % kD;
    float as[kMaxSplitsK][kDpt];
#pragma unroll
    for (int sidx = 0; sidx < kMaxSplitsK; ++sidx) {
        const float* src = base + sidx * stride + h * (kD + 2) + 2 + dim;
        if (kDpt == 2) {  // 8-byte aligned: every term of the offset is even
            const float2 v = mine && sidx < p.splits ? __ldcg(reinterpret_cast<const float2*>(src))
                                                      : make_float2(0.f, 0.f);
            as[sidx][0] = v.x;
            as[sidx][kDpt - 1] = v.y;
        } else {
            as[sidx][0] = mine && sidx < p.splits ? __ldcg(src) : 0.f;
        }
    }
    // (after the acc loads are issued, so that none waits behind these)
    if (tid < p.splits * G) {
        const int sidx = tid / G, hh = tid % G;
        const float mv = __ldcg(base + sidx * stride + hh * (kD + 2));
        const float lv = __ldcg(base + sidx * stride + hh * (kD + 2) + 1);
        sm_m[sidx][hh] = mv;
        sm_l[sidx][hh] = lv;
    }
    compute_bar();
    if (mine) {
        float mm = -INFINITY;
#pragma unroll
        for (int sidx = 0; sidx < kMaxSplitsK; ++sidx)
            if (sidx < p.splits) mm = fmaxf(mm, sm_m[sidx][h]);
        float ll = 0.f, aa[kDpt];
#pragma unroll
        for (int i = 0; i < kDpt; ++i) aa[i] = 0.f;
#pragma unroll
        for (int sidx = 0; sidx < kMaxSplitsK; ++sidx) {
            if (sidx < p.splits) {
                const float ms = sm_m[sidx][h];
                const float c = ms == -INFINITY ? 0.f : ex2_a(ms - mm);
                ll = fmaf(c, sm_l[sidx][h], ll);
#pragma unroll
                for (int i = 0; i < kDpt; ++i) aa[i] = fmaf(c, as[sidx][i], aa[i]);
            }
        }
#pragma unroll
        for (int i = 0; i < kDpt; ++i)
            p.o[static_cast<int64_t>(g * G + h) * kD + dim + i] = f2h_rn(aa[i] / ll);
    }
    if (tid == 0) p.ticket[g] = 0u;
}

constexpr int kMaxSplits = kMaxSplitsK;

int pick_splits(int hkv, int group, int64_t l_max, int num_sms) {
    (void)group;
    // one CTA per SM (the kernel's shared memory allows no more), in one wave:
    // long chunks keep the final merge of the splits short
    int s = num_sms / hkv;
    if (s > kMaxSplits) s = kMaxSplits;
    if (s > l_max) s = static_cast<int>(l_max);
    return s < 1 ? 1 : s;
}

}  // namespace

size_t decode_attention_workspace_bytes(int hq, int hkv) {
    const size_t tickets = (static_cast<size_t>(hkv) * 4 + 255) / 256 * 256;
    return tickets + static_cast<size_t>(hkv) * kMaxSplits * (hq / hkv) * (kD + 2) * 4;
}

qg_status launch_decode_attention(const AttentionLaunch& L, cudaStream_t stream) {
    DeviceInfo dev;
    qg_status st = device_info(&dev);
    if (st != QG_OK) return st;
    if (L.d != kD) return QG_ERR_SHAPE;
    const int G = L.hq / L.hkv;
    if (G != 1 && G != 2 && G != 4) return QG_ERR_SHAPE;
    if (L.ws_bytes < decode_attention_workspace_bytes(L.hq, L.hkv)) return QG_ERR_WORKSPACE;
    AttnParams p = {};
    p.qkv = L.qkv;
    p.kc = L.kcache;
    p.vc = L.vcache;
    p.o = L.o;
    p.pos = L.pos;
    p.l_max = L.l_max;
    p.hq = L.hq;
    p.hkv = L.hkv;
    p.splits = pick_splits(L.hkv, G, L.l_max, dev.num_sms);
    p.theta = L.theta;
    p.qscale = kLog2e / std::sqrt(static_cast<double>(kD));
    const size_t tickets = (static_cast<size_t>(L.hkv) * 4 + 255) / 256 * 256;
    p.ticket = static_cast<unsigned int*>(L.workspace);
    p.part = reinterpret_cast<float*>(static_cast<char*>(L.workspace) + tickets);

    void (*kern)(AttnParams) = G == 1 ? decode_attention_kernel<1>
                               : (G == 2 ? decode_attention_kernel<2> : decode_attention_kernel<4>);
    static bool attr_done[3][64] = {{false}};
    const int gi = G == 1 ? 0 : (G == 2 ? 1 : 2);
    if (dev.device >= 64 || !attr_done[gi][dev.device]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kRingBytesA);
        if (e != cudaSuccess) return cuda_status(e);
        if (dev.device < 64) attr_done[gi][dev.device] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(p.splits), static_cast<unsigned>(L.hkv));
    cfg.blockDim = dim3(kThreadsA);
    cfg.dynamicSmemBytes = kRingBytesA;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, p));
}

unsigned int attention_read_and_clear_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_attn_err, sizeof v) != cudaSuccess) return 0;
    if (v) cudaMemcpyToSymbol(g_attn_err, &zero, sizeof zero);
    return v;
}

}  // namespace qg
