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
//  * one CTA of 8 warps per SM takes a long chunk, streamed through a
//    three-stage cp.async ring of 64 rows of K and V (after an L2 prefetch of
//    the chunk issued before the wait on the previous kernel);
//  * inside a CTA, each group of 16 lanes takes four rows of every stage
//    (8 dims per lane, 16-byte shared loads) with an online softmax per query
//    head, rescaled once per stage; groups, then warps, merge their (max,
//    sum, acc) states;
//  * every CTA writes its partial state; the last CTA of a kv head (an atomic
//    ticket, no CTA ever waits) merges the splits, writes o in fp16 and
//    re-zeroes its ticket;
//  * the new token's key and value are computed by every CTA (RoPE angles in
//    fp64, one fp16 rounding) and used for row pos, which no CTA reads from
//    the cache; the CTA whose chunk holds pos writes them into the cache.
#include <cfloat>
#include <cmath>

#include "qg_device.cuh"
#include "qg_internal.h"

namespace qg {

QG_DEFINE_ERROR_FLAG(g_attn_err);

namespace {

constexpr int kD = 128;            // head_dim of the pages' Qwen3-VL decoders
constexpr int kWarpsA = 8;
constexpr int kThreadsA = kWarpsA * 32;
constexpr int kGroupLanes = 16;    // lanes per subsequence: 16 x 8 dims = one row
constexpr int kSubseq = kThreadsA / kGroupLanes;  // 16 subsequences per CTA
constexpr int kDimsPerLane = kD / kGroupLanes;    // 8: one 16-byte load per row
constexpr int kUnroll = 4;                        // rows of a subsequence per stage
constexpr int kStageRows = kSubseq * kUnroll;     // 64 rows of K and of V per stage
constexpr int kStages = 3;                        // ring depth: two stages in flight
constexpr int kRowBytes = kD * 2;
constexpr int kStageBytes = 2 * kStageRows * kRowBytes;  // K rows, then V rows: 32 KB
constexpr int kRingBytesA = kStages * kStageBytes;
constexpr int kMaxSplitsK = 32;                   // splits of one kv head's rows, at most
constexpr int kPrefetchRows = 256;                // rows of a chunk prefetched into L2

struct AttnParams {
    const float* qkv;
    uint16_t* kc;
    uint16_t* vc;
    uint16_t* o;
    const int32_t* pos;
    float* part;              // [hkv][splits][G][kD + 2]: m, l, acc
    unsigned int* ticket;     // [hkv]
    int64_t l_max;
    int hq, hkv, splits;
    double theta;
    float scale;              // 1 / sqrt(d)
};

__device__ __forceinline__ void cp_async16_a(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit_a() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait_a() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
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

// Merge the online-softmax state (m2, l2, a2) into (m, l, a).
template <int N>
__device__ __forceinline__ void merge_state(float& m, float& l, float* a, float m2, float l2,
                                            const float* a2) {
    const float mn = fmaxf(m, m2);
    const float c1 = m == -INFINITY ? 0.f : expf(m - mn);
    const float c2 = m2 == -INFINITY ? 0.f : expf(m2 - mn);
    l = l * c1 + l2 * c2;
#pragma unroll
    for (int i = 0; i < N; ++i) a[i] = a[i] * c1 + a2[i] * c2;
    m = mn;
}

template <int G>
__global__ void __launch_bounds__(kThreadsA, 1) decode_attention_kernel(const AttnParams p) {
    __shared__ float q_s[G][kD];
    __shared__ __align__(16) uint16_t kn_h[kD];
    __shared__ __align__(16) uint16_t vn_h[kD];
    __shared__ float wst[kWarpsA][G][kD + 2];  // per-warp merged states
    __shared__ unsigned int last_s;
    __shared__ float sm_m[G][kMaxSplitsK];  // split maxima (then weights)
    __shared__ float sm_l[G][kMaxSplitsK];  // split sums

    const int split = blockIdx.x, g = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    extern __shared__ __align__(128) unsigned char ring[];
    const uint32_t ring0 = smem_u32(ring);

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
    if (lane == 0) {
        if (pg >= 0 && pg < p.l_max) {
            int64_t a0, a1;
            chunk_of(pg, p.splits, split, a0, a1);
            if (a1 > a0 + kPrefetchRows) a1 = a0 + kPrefetchRows;
            // warp w prefetches its quarter of the chunk, in pieces of <= 16 KB
            const int64_t q0 = a0 + (a1 - a0) * warp / kWarpsA;
            const int64_t q1 = a0 + (a1 - a0) * (warp + 1) / kWarpsA;
            for (int64_t r = q0; r < q1; r += 64) {
                const int64_t rows = q1 - r < 64 ? q1 - r : 64;
                const int64_t off = (static_cast<int64_t>(g) * p.l_max + r) * kD;
                prefetch_l2_a(p.kc + off, static_cast<uint32_t>(rows * kRowBytes));
                prefetch_l2_a(p.vc + off, static_cast<uint32_t>(rows * kRowBytes));
            }
        }
    }
    griddep_wait();  // q|k|v come from the projection kernel before this one
    const int32_t pos = *p.pos;
    if (pos < 0 || pos >= p.l_max) {
        if (tid == 0 && split == 0 && g == 0) atomicOr(&g_attn_err, 1u);
        return;
    }
    int64_t j0, j1;
    chunk_of(pos, p.splits, split, j0, j1);
    const int nstages = static_cast<int>((j1 - j0 + kStageRows - 1) / kStageRows);
    // Stage st of the chunk -> ring slot st % kStages: rows j0 + 64 st ..., K
    // then V, 16 pieces of 16 bytes per row; row pos (not written yet) is
    // skipped, its values come from shared memory below.
    auto issue = [&](int st) {
        const uint32_t slot = ring0 + (st % kStages) * kStageBytes;
#pragma unroll
        for (int k = 0; k < 2 * kStageRows * 16 / kThreadsA; ++k) {
            const int i = tid + k * kThreadsA;
            const int kv = i / (kStageRows * 16), rr = (i / 16) % kStageRows, col = i % 16;
            const int64_t j = j0 + static_cast<int64_t>(st) * kStageRows + rr;
            if (j < j1 && j != pos) {
                const uint16_t* src = (kv == 0 ? p.kc : p.vc) +
                                      (static_cast<int64_t>(g) * p.l_max + j) * kD + col * 8;
                cp_async16_a(slot + (kv * kStageRows + rr) * kRowBytes + col * 16, src);
            }
        }
    };
    // the first stages stream while q, k and v are rotated
#pragma unroll
    for (int st = 0; st < kStages - 1; ++st) {
        if (st < nstages) issue(st);
        cp_async_commit_a();
    }

    // Thread i < d/2 rotates pair i of the new key (fp64, rounded once to
    // fp16) and of every query head that reads this kv head; its loads of the
    // key and query pairs go out together.
    if (tid < kD / 2) {
        if (pos != pg) angles(pos);  // the position changed after the early read
        const float* kin = p.qkv + static_cast<int64_t>(p.hq) * kD + g * kD;
        const double k0 = kin[tid], k1 = kin[tid + kD / 2];
        double q0[G], q1[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float* qin = p.qkv + static_cast<int64_t>(g * G + h) * kD;
            q0[h] = qin[tid];
            q1[h] = qin[tid + kD / 2];
        }
        const uint16_t r0 = __half_as_ushort(__double2half(k0 * rc - k1 * rs));
        const uint16_t r1 = __half_as_ushort(__double2half(k1 * rc + k0 * rs));
        kn_h[tid] = r0;
        kn_h[tid + kD / 2] = r1;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            q_s[h][tid] = static_cast<float>(q0[h] * rc - q1[h] * rs);
            q_s[h][tid + kD / 2] = static_cast<float>(q1[h] * rc + q0[h] * rs);
        }
    }
    if (tid < kD) {
        const float* vin = p.qkv + static_cast<int64_t>(p.hq + p.hkv) * kD + g * kD;
        const uint16_t v = f2h_rn(vin[tid]);
        vn_h[tid] = v;
    }
    __syncthreads();
    griddep_launch_dependents();

    // the CTA whose chunk holds pos appends the new rows
    if (pos >= j0 && pos < j1 && tid < kD) {
        const int64_t row = (static_cast<int64_t>(g) * p.l_max + pos) * kD;
        p.kc[row + tid] = kn_h[tid];
        p.vc[row + tid] = vn_h[tid];
    }

    // ---- stream: in each stage, subsequence sq = tid / 16 takes rows sq,
    // sq + 16, sq + 32, sq + 48 (one rescale per stage)
    const int sq = tid / kGroupLanes, gl = tid % kGroupLanes;
    const int d0 = gl * kDimsPerLane;
    float qr[G][kDimsPerLane];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int i = 0; i < kDimsPerLane; ++i) qr[h][i] = q_s[h][d0 + i] * p.scale;
    float m[G], l[G], acc[G][kDimsPerLane];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int i = 0; i < kDimsPerLane; ++i) acc[h][i] = 0.f;
    }
    const uint4 kn4 = *reinterpret_cast<const uint4*>(kn_h + d0);
    const uint4 vn4 = *reinterpret_cast<const uint4*>(vn_h + d0);
    // Every thread runs every stage (the shuffles take the whole warp and the
    // ring is refilled by the whole CTA); rows past the end are skipped.
    for (int st = 0; st < nstages; ++st) {
        if (st + kStages - 1 < nstages) issue(st + kStages - 1);
        cp_async_commit_a();
        cp_async_wait_a<kStages - 1>();
        __syncthreads();  // every thread's copies of stage st have landed
        const uint32_t slot = ring0 + (st % kStages) * kStageBytes;
        uint4 kr[kUnroll], vr[kUnroll];
        bool valid[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int rr = sq + u * kSubseq;
            const int64_t j = j0 + static_cast<int64_t>(st) * kStageRows + rr;
            valid[u] = j < j1;
            if (valid[u] && j != pos) {
                kr[u] = lds128_a(slot + rr * kRowBytes + d0 * 2);
                vr[u] = lds128_a(slot + (kStageRows + rr) * kRowBytes + d0 * 2);
            } else {
                kr[u] = valid[u] ? kn4 : make_uint4(0u, 0u, 0u, 0u);
                vr[u] = valid[u] ? vn4 : make_uint4(0u, 0u, 0u, 0u);
            }
        }
        float kv[kUnroll][kDimsPerLane];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) unpack8h(kr[u], kv[u]);
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float s[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                float a = 0.f;
#pragma unroll
                for (int i = 0; i < kDimsPerLane; ++i) a = fmaf(qr[h][i], kv[u][i], a);
                a += __shfl_xor_sync(0xffffffffu, a, 1);
                a += __shfl_xor_sync(0xffffffffu, a, 2);
                a += __shfl_xor_sync(0xffffffffu, a, 4);
                a += __shfl_xor_sync(0xffffffffu, a, 8);
                s[u] = a;
            }
            float mx = m[h];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u)
                if (valid[u]) mx = fmaxf(mx, s[u]);
            if (mx == -INFINITY) continue;  // no valid row yet (uniform in the group)
            const float corr = m[h] == -INFINITY ? 0.f : expf(m[h] - mx);
            l[h] *= corr;
#pragma unroll
            for (int i = 0; i < kDimsPerLane; ++i) acc[h][i] *= corr;
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                if (!valid[u]) continue;
                const float pj = expf(s[u] - mx);
                float vv[kDimsPerLane];
                unpack8h(vr[u], vv);
                l[h] += pj;
#pragma unroll
                for (int i = 0; i < kDimsPerLane; ++i) acc[h][i] = fmaf(pj, vv[i], acc[h][i]);
            }
            m[h] = mx;
        }
        __syncthreads();  // the slot is consumed before it is refilled
    }
    cp_async_wait_a<0>();

    // ---- merge the 2 subsequences of a warp (lanes 16 apart hold the same dims)
#pragma unroll
    for (int h = 0; h < G; ++h) {
        {
            const int off = kGroupLanes;
            const float m2 = __shfl_xor_sync(0xffffffffu, m[h], off);
            const float l2 = __shfl_xor_sync(0xffffffffu, l[h], off);
            float a2[kDimsPerLane];
#pragma unroll
            for (int i = 0; i < kDimsPerLane; ++i)
                a2[i] = __shfl_xor_sync(0xffffffffu, acc[h][i], off);
            merge_state<kDimsPerLane>(m[h], l[h], acc[h], m2, l2, a2);
        }
        if (lane < kGroupLanes) {
#pragma unroll
            for (int i = 0; i < kDimsPerLane; ++i) wst[warp][h][2 + d0 + i] = acc[h][i];
            if (lane == 0) {
                wst[warp][h][0] = m[h];
                wst[warp][h][1] = l[h];
            }
        }
    }
    __syncthreads();

    // ---- merge the warps: thread tid owns dim tid % 128 of heads tid / 128,
    // tid / 128 + 2, ...; write the partial
    float* part = p.part + (static_cast<int64_t>(g) * p.splits + split) * G * (kD + 2);
    const int dim = tid & (kD - 1), hh = tid / kD;
#pragma unroll
    for (int hb = 0; hb < G; hb += kThreadsA / kD) {
        const int h = hb + hh;
        if (h < G) {
            float mm = wst[0][h][0], ll = wst[0][h][1], aa = wst[0][h][2 + dim];
            for (int w = 1; w < kWarpsA; ++w)
                merge_state<1>(mm, ll, &aa, wst[w][h][0], wst[w][h][1], &wst[w][h][2 + dim]);
            part[h * (kD + 2) + 2 + dim] = aa;
            if (dim == 0) {
                part[h * (kD + 2)] = mm;
                part[h * (kD + 2) + 1] = ll;
            }
        }
    }

    // ---- the last CTA of this kv head merges the splits
    __threadfence();
    __syncthreads();
    if (tid == 0) last_s = atomicAdd(&p.ticket[g], 1u) == static_cast<unsigned int>(p.splits - 1);
    __syncthreads();
    if (!last_s) return;
    __threadfence();
    // Merge the splits of every head in one pass (threads 0-127 take heads
    // 0, 2, ..., threads 128-255 heads 1, 3, ...): thread s (< splits) of a
    // head fetches split s's max and sum and forms its weight e^(m_s - M);
    // every thread sums its dim over all splits with loads that are all in
    // flight at once.
    const float* base = p.part + static_cast<int64_t>(g) * p.splits * G * (kD + 2);
    const int64_t stride = static_cast<int64_t>(G) * (kD + 2);
    constexpr int kHalves = kThreadsA / kD;                // 2: threads 0-127 and 128-255
    constexpr int kHpt = (G + kHalves - 1) / kHalves;      // heads per thread
    float v[kHpt][kMaxSplitsK];
#pragma unroll
    for (int e = 0; e < kHpt; ++e) {
        const int h = hh + kHalves * e;
        const float* col = base + static_cast<int64_t>(h < G ? h : 0) * (kD + 2);
#pragma unroll
        for (int sidx = 0; sidx < kMaxSplitsK; ++sidx)
            v[e][sidx] = h < G && sidx < p.splits ? __ldcg(col + sidx * stride + 2 + dim) : 0.f;
        if (h < G && dim < p.splits) {
            sm_m[h][dim] = __ldcg(col + dim * stride);
            sm_l[h][dim] = __ldcg(col + dim * stride + 1);
        }
    }
    __syncthreads();
    float mx[kHpt];
#pragma unroll
    for (int e = 0; e < kHpt; ++e) {
        const int h = hh + kHalves * e;
        mx[e] = -INFINITY;
        if (h < G)
            for (int sidx = 0; sidx < p.splits; ++sidx) mx[e] = fmaxf(mx[e], sm_m[h][sidx]);
    }
    __syncthreads();  // every thread has its maxima
#pragma unroll
    for (int e = 0; e < kHpt; ++e) {
        const int h = hh + kHalves * e;
        if (h < G && dim < p.splits)
            sm_m[h][dim] = sm_m[h][dim] == -INFINITY ? 0.f : expf(sm_m[h][dim] - mx[e]);
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < kHpt; ++e) {
        const int h = hh + kHalves * e;
        if (h >= G) continue;
        float ll = 0.f, aa = 0.f;
#pragma unroll
        for (int sidx = 0; sidx < kMaxSplitsK; ++sidx) {
            if (sidx < p.splits) {
                ll = fmaf(sm_m[h][sidx], sm_l[h][sidx], ll);
                aa = fmaf(sm_m[h][sidx], v[e][sidx], aa);
            }
        }
        p.o[static_cast<int64_t>(g * G + h) * kD + dim] = f2h_rn(aa / ll);
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
    p.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(kD)));
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
