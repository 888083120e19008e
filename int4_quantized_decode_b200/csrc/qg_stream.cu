// qg_stream.cu -- a whole int8 decode sweep as one persistent launch whose
// weight stream does not stop at stage boundaries.
//
// A decode step reads every decoder weight once ("Qwen3-VL 4B -- Core AI
// (.aimodel)", Measured: decode is the weight read), as an ordered chain of
// S=1 projections in which each stage needs the whole output of the stage
// before it ("Qwen3.8-27B ... -- Core AI", The vision path: prefill runs as
// pipelined S=1 steps).  Only the activation depends on the previous stage,
// never the weights; so one thread per SM streams the SM's share of every
// stage's weights, in plan order, into a shared-memory ring and never waits
// for an activation: while the compute warps wait at a stage boundary the
// ring keeps filling.
//
//  * One CTA per SM (cooperative launch): 16 compute warps, a producer warp
//    and a sync warp.
//  * Each CTA owns a contiguous range of every stage's rows (n / G rounded,
//    so no CTA has more than one row above the average), cut into chunks of
//    whole rows (a SwiGLU chunk: the same rows of gate and of up) of at most
//    32 KB of codes, so that every chunk is a few large 1-D bulk copies (on
//    this GPU a bulk copy costs ~450 cycles of the SM's copy engine whatever
//    its size, and only copies of 16 KB or more reach the HBM rate).
//  * Producer: one lane issues each chunk's copies (codes and fp16 scales of
//    each matrix) into the chunk's ring slot, completing on the slot's
//    mbarrier; it refills a slot once every compute warp has released it.
//  * Compute warps: row u of a stage's range belongs to warp u % 16, which
//    computes it whole (lane l takes the 16 codes at 16 l of each 512-code
//    step against x[16 l .. 16 l + 16), raw fp16 in shared memory; codes
//    become exact fp16 q by a byte permute into 1024 + (q + 128) and a packed
//    subtraction of 1152, and the sm_100 mixed-precision FMA accumulates the
//    exact products q x in fp32; each block scale multiplies its 16-code
//    partial; one warp reduction per row).  Every compute warp walks every
//    chunk in ring order -- waits for its copies, computes its own rows in it,
//    releases it -- so it sees each slot's fills in order and no parity wait
//    can match a stale phase.
//  * Sync warp: when every compute warp of its CTA is done with stage s (an
//    mbarrier), it arrives on the grid counter of stage s (release), waits
//    for every CTA (acquire, bounded) and fetches x of stage s + 1 with one
//    bulk copy into the other half of a double buffer, on an mbarrier the
//    compute warps wait on.  It also finishes a head stage's argmax for its
//    CTA (atomicMax of an order-preserving key, last-CTA ticket).
//  * Every wait is bounded; one that gives up sets the device error flag and
//    the CTA's abort flag, after which the CTA drains its own copies and
//    returns.
#include <cfloat>
#include <climits>
#include <vector>

#include "qg_device.cuh"
#include "qg_internal.h"

namespace qg {

QG_DEFINE_ERROR_FLAG(g_stream_err);

namespace {

constexpr int kSwW = 16;                      // compute warps per CTA
constexpr int kProdWarp = kSwW;               // the producer warp
constexpr int kSyncWarp = kSwW + 1;           // the sync warp
constexpr int kSwThreads = (kSwW + 2) * 32;
constexpr int kSwStep = 512;                  // codes of one warp step along a row
constexpr int kChunkCodes = 32768;            // code bytes a ring slot holds
constexpr int kSlotBytes = kChunkCodes + kChunkCodes / 16;  // + their fp16 scales
constexpr int kMaxSlots = 8;
constexpr int kMinSlots = 3;
constexpr int kSwMaxStages = 320;
constexpr uint32_t kStreamMagic = 0x34575351u;

enum StreamOp : int32_t { kOpGemv = 0, kOpSwiglu = 1, kOpHead = 2 };

// What the warps' cursors read of a stage (kept in shared memory).
// Rows are output rows: a SwiGLU row is the pair (gate r, up r).
struct StreamStage {
    const uint8_t* codes[2];    // gemv/head: [0]; swiglu: gate, up
    const uint16_t* scales[2];
    int32_t n, k;               // rows, columns (k % 512 == 0)
    int32_t op;                 // StreamOp
    int32_t nmat;               // 1, or 2 for SwiGLU
    int32_t nrc;                // rows per chunk: nmat * nrc * k <= kChunkCodes
    int32_t nst;                // steps per row: k / 512
    int32_t xext;               // x is a run input: no stage of the plan writes it
    int32_t pad;
};
static_assert(sizeof(StreamStage) == 64, "stage descriptors are 64 bytes");

// What a stage writes (read from global memory when an item finishes).
struct StreamOut {
    const uint16_t* x;          // fp16 [k] activation
    float* y;
    uint16_t* y16;
    uint16_t* h;
    float* logits;
    int32_t* idx;
    unsigned long long* key;    // head scratch: argmax key and ticket
    unsigned int* ticket;
};
static_assert(sizeof(StreamOut) == 64, "outputs are 64 bytes");

struct StreamHeader {
    uint32_t magic;
    int32_t n_stages;
    int32_t slots;              // ring slots the plan was made for
    int32_t xmax;               // the largest k of the plan
    uint32_t reserved[60];
};
static_assert(sizeof(StreamHeader) == 256, "header is 256 bytes");

__host__ __device__ constexpr size_t a256(size_t v) { return (v + 255) / 256 * 256; }
// Grid counters: each stage has kSwCtr counters in separate 128-byte lines;
// CTA i arrives on counter i % kSwCtr, so the arrivals spread over several
// L2 lines and a waiter reads all of them with parallel loads.
constexpr int kSwCtr = 8;
constexpr int kSwCtrStride = 32;  // unsigned ints: 128 bytes
__host__ __device__ constexpr size_t sw_ctr_words(int n) {
    return static_cast<size_t>(n) * kSwCtr * kSwCtrStride + 32;  // + the exit counter's line
}
// Workspace: [header][grid counters][16 B head scratch per stage]
// [StreamStage x n][StreamOut x n]
__host__ __device__ constexpr size_t sw_ctr_off() { return sizeof(StreamHeader); }
__host__ __device__ constexpr size_t sw_scr_off(int n) {
    return sw_ctr_off() + a256(sw_ctr_words(n) * 4);
}
__host__ __device__ constexpr size_t sw_stage_off(int n) {
    return sw_scr_off(n) + a256(static_cast<size_t>(n) * 16);
}
__host__ __device__ constexpr size_t sw_out_off(int n) {
    return sw_stage_off(n) + static_cast<size_t>(n) * sizeof(StreamStage);
}
__host__ __device__ constexpr size_t sw_bytes(int n) {
    return sw_out_off(n) + static_cast<size_t>(n) * sizeof(StreamOut);
}
// Dynamic shared memory: [stage descriptors][x double buffer][rings]
__host__ __device__ constexpr size_t sw_desc_bytes(int n) {
    return a256(static_cast<size_t>(n) * sizeof(StreamStage));
}
__host__ __device__ constexpr size_t sw_x_bytes(int xmax) {
    return a256(static_cast<size_t>(xmax) * 2);
}
__host__ __device__ constexpr size_t sw_smem(int n, int xmax, int slots) {
    return sw_desc_bytes(n) + 2 * sw_x_bytes(xmax) + static_cast<size_t>(slots) * kSlotBytes;
}

// Expect `bytes` more on the current phase without arriving (the phase then
// completes when they have landed and the arrivals it counts are made).
__device__ __forceinline__ void mbar_expect_tx_only(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0u;
}
// Spin (no suspension) until the phase of `parity` completes, bounded.
__device__ __forceinline__ bool mbar_spin_bounded(uint64_t* bar, uint32_t parity) {
    if (mbar_test(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_test(bar, parity))
        if (clock64() - t0 > kWaitLimitCycles) return false;
    return true;
}
__device__ __forceinline__ unsigned int ld_relaxed_gpu(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Wait until *c >= target (relaxed polls, one acquire fence after), bounded.
__device__ __forceinline__ bool poll_counter(const unsigned int* c, unsigned int target) {
    const long long t0 = clock64();
    while (ld_relaxed_gpu(c) < target)
        if (clock64() - t0 > kWaitLimitCycles) return false;
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    return true;
}

__device__ __forceinline__ void bulk_g2s_u32(uint32_t dst, const void* src, uint32_t bytes,
                                             uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}
__device__ __forceinline__ uint4 lds128s(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a));
    return v;
}
__device__ __forceinline__ uint16_t lds16s(uint32_t a) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t hsub2s(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ void fma_mixed(float& a0, float& a1, uint32_t q2, uint32_t x2) {
    asm("{\n\t.reg .f16 q0, q1, x0, x1;\n\t"
        "mov.b32 {q0, q1}, %2;\n\t"
        "mov.b32 {x0, x1}, %3;\n\t"
        "fma.rn.f32.f16 %0, q0, x0, %0;\n\t"
        "fma.rn.f32.f16 %1, q1, x1, %1;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "r"(q2), "r"(x2));
}
__device__ __forceinline__ unsigned long long key_of(float v, int idx) {
    uint32_t b = __float_as_uint(v);
    b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);  // order-preserving
    return (static_cast<unsigned long long>(b) << 32) |
           static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(idx));
}

// 16 int8 codes (k order, byte 0 first) against their 16 fp16 x (xa: the
// first 8, xb: the last 8): sum q x with exact products.
__device__ __forceinline__ float dot16(uint4 c, uint4 xa, uint4 xb) {
    float a0 = 0.f, a1 = 0.f;
    const uint32_t u0 = c.x ^ 0x80808080u, u1 = c.y ^ 0x80808080u;
    const uint32_t u2 = c.z ^ 0x80808080u, u3 = c.w ^ 0x80808080u;
    fma_mixed(a0, a1, hsub2s(__byte_perm(u0, 0x64646464u, 0x4140), 0x64806480u), xa.x);
    fma_mixed(a0, a1, hsub2s(__byte_perm(u0, 0x64646464u, 0x4342), 0x64806480u), xa.y);
    fma_mixed(a0, a1, hsub2s(__byte_perm(u1, 0x64646464u, 0x4140), 0x64806480u), xa.z);
    fma_mixed(a0, a1, hsub2s(__byte_perm(u1, 0x64646464u, 0x4342), 0x64806480u), xa.w);
    fma_mixed(a0, a1, hsub2s(__byte_perm(u2, 0x64646464u, 0x4140), 0x64806480u), xb.x);
    fma_mixed(a0, a1, hsub2s(__byte_perm(u2, 0x64646464u, 0x4342), 0x64806480u), xb.y);
    fma_mixed(a0, a1, hsub2s(__byte_perm(u3, 0x64646464u, 0x4140), 0x64806480u), xb.z);
    fma_mixed(a0, a1, hsub2s(__byte_perm(u3, 0x64646464u, 0x4342), 0x64806480u), xb.w);
    return a0 + a1;
}

// One whole row (NR = 1) or a gate/up pair (NR = 2) of a chunk: codes at
// ca / cb in shared memory (k bytes each), scales at sa / sb (k / 16 bytes);
// returns this lane's partial sums (the warp reduces them).
template <int NR>
__device__ __forceinline__ void row_dot(uint32_t ca, uint32_t cb, uint32_t sa, uint32_t sb,
                                        uint32_t xs, int nst, int lane, float& acc0,
                                        float& acc1) {
    const uint32_t cl = lane * 16, sl = (lane >> 1) * 2, xl = xs + lane * 32;
#pragma unroll 2
    for (int st = 0; st < nst; ++st) {
        const uint4 xa = lds128s(xl + st * (kSwStep * 2));
        const uint4 xb = lds128s(xl + st * (kSwStep * 2) + 16);
        const uint4 c0 = lds128s(ca + cl + st * kSwStep);
        const float s0 = h2f(lds16s(sa + sl + st * 32));
        acc0 = fmaf(s0, dot16(c0, xa, xb), acc0);
        if (NR == 2) {
            const uint4 c1 = lds128s(cb + cl + st * kSwStep);
            const float s1 = h2f(lds16s(sb + sl + st * 32));
            acc1 = fmaf(s1, dot16(c1, xa, xb), acc1);
        }
    }
}

// This CTA's rows [r0, r0 + R) of stage S.
__device__ __forceinline__ void rows_of(const StreamStage& S, int cta, int G, int64_t& r0, int& R) {
    r0 = static_cast<int64_t>(cta) * S.n / G;
    R = static_cast<int>(static_cast<int64_t>(cta + 1) * S.n / G - r0);
}

__global__ void __launch_bounds__(kSwThreads, 1) stream_sweep_kernel(unsigned char* ws, int n,
                                                                     int NS) {
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ __align__(8) uint64_t xfull[2];  // x of stage s landed (tx bytes)
    __shared__ __align__(8) uint64_t sdone[2];  // every compute warp done with stage s
    __shared__ __align__(8) uint64_t full[kMaxSlots];   // a slot's copies landed (tx bytes)
    __shared__ __align__(8) uint64_t empty[kMaxSlots];  // every compute warp done with a slot
    __shared__ float best_v[2][kSwW];
    __shared__ int best_i[2][kSwW];
    __shared__ volatile int abort_sh;

    const StreamHeader* hdr = reinterpret_cast<const StreamHeader*>(ws);
    uint32_t dyn_smem;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_smem));
    if (hdr->magic != kStreamMagic || hdr->n_stages != n || hdr->slots != NS ||
        NS < kMinSlots || NS > kMaxSlots || hdr->xmax < kSwStep ||
        sw_smem(n, hdr->xmax, NS) > dyn_smem) {
        if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(&g_stream_err, kGemvErrBadPlan);
        return;
    }
    unsigned int* ctr = reinterpret_cast<unsigned int*>(ws + sw_ctr_off());
    const StreamOut* outs = reinterpret_cast<const StreamOut*>(ws + sw_out_off(n));
    const int xmax = hdr->xmax;
    const int G = static_cast<int>(gridDim.x), cta = static_cast<int>(blockIdx.x);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    StreamStage* st = reinterpret_cast<StreamStage*>(smem);
    const uint32_t xbuf0 = smem_u32(smem) + static_cast<uint32_t>(sw_desc_bytes(n));
    const uint32_t xstride = static_cast<uint32_t>(sw_x_bytes(xmax));
    const uint32_t ring0 = xbuf0 + 2 * xstride;

    {  // stage descriptors into shared memory
        const uint4* src = reinterpret_cast<const uint4*>(ws + sw_stage_off(n));
        uint4* dst = reinterpret_cast<uint4*>(smem);
        const int pieces = n * static_cast<int>(sizeof(StreamStage) / 16);
        for (int i = threadIdx.x; i < pieces; i += kSwThreads) dst[i] = ldg_nc_v4(src + i);
    }
    if (threadIdx.x == 0) {
        abort_sh = 0;
        mbar_init(&xfull[0], 1);
        mbar_init(&xfull[1], 1);
        mbar_init(&sdone[0], kSwW);
        mbar_init(&sdone[1], kSwW);
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kSwW);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kSyncWarp) {
        // ------------------------------------------------------ sync warp ---
        const uint64_t pol_x = l2_policy_evict_last();
        // x of stage s into its half of the buffer.  A run input may be copied
        // a stage early with the expected bytes only: the plain arrival that
        // completes the phase (and lets the warps compute) comes after the
        // grid has finished stage s - 1.
        auto copy_x = [&](int s, bool arrive) {
            asm volatile("fence.proxy.async.global;" ::: "memory");
            const uint32_t bytes = static_cast<uint32_t>(st[s].k) * 2;
            if (arrive)
                mbar_arrive_expect_tx(&xfull[s & 1], bytes);
            else
                mbar_expect_tx_only(&xfull[s & 1], bytes);
            bulk_g2s_u32(xbuf0 + (s & 1) * xstride, outs[s].x, bytes, &xfull[s & 1], pol_x);
        };
        bool early = false;  // x of the next stage was copied ahead
        if (lane == 0) {
            copy_x(0, true);
            if (n > 1 && st[1].xext) {
                copy_x(1, false);
                early = true;
            }
        }
        int issued = n > 1 && st[1].xext ? 2 : 1;  // x copies issued (stages 0 .. issued-1)
        for (int s = 1; s <= n; ++s) {
            const int p = s - 1;
            int ok = abort_sh ? 0 : (mbar_spin_bounded(&sdone[p & 1], (p >> 1) & 1) ? 1 : 0);
            if (ok && st[p].op == kOpHead && lane == 0) {
                // this CTA's best of stage p, then the grid's through the key
                float bv = -FLT_MAX;
                int bi = INT_MAX;
                for (int w = 0; w < kSwW; ++w) {
                    const float v = best_v[p & 1][w];
                    const int i = best_i[p & 1][w];
                    if (v > bv || (v == bv && i < bi)) {
                        bv = v;
                        bi = i;
                    }
                }
                const StreamOut& o = outs[p];
                if (bi != INT_MAX) atomicMax(o.key, key_of(bv, bi));
                __threadfence();
                if (atomicAdd(o.ticket, 1u) == static_cast<unsigned>(G) - 1) {
                    __threadfence();
                    const unsigned long long key = atomicAdd(o.key, 0ull);
                    *o.idx = static_cast<int32_t>(0xFFFFFFFFu -
                                                  static_cast<uint32_t>(key & 0xFFFFFFFFull));
                    *o.key = 0ull;
                    *o.ticket = 0u;
                }
            }
            if (s == n) {
                if (!ok && lane == 0 && !abort_sh) {
                    atomicOr(&g_stream_err, kGemvErrTimeout);
                    abort_sh = 1;
                }
                break;
            }
            if (ok) {
                unsigned int* c = ctr + static_cast<size_t>(p) * kSwCtr * kSwCtrStride;
                if (lane == 0) red_release_gpu_inc(c + (cta % kSwCtr) * kSwCtrStride);
                // lanes 0..7 each watch one counter: CTAs lane, lane + 8, ...
                if (lane < kSwCtr) {
                    const unsigned target = static_cast<unsigned>((G - lane + kSwCtr - 1) / kSwCtr);
                    ok = poll_counter(c + lane * kSwCtrStride, target) ? 1 : 0;
                }
                ok = __all_sync(0xffffffffu, ok != 0) ? 1 : 0;
            }
            if (!ok) {
                if (lane == 0) {
                    if (!abort_sh) atomicOr(&g_stream_err, kGemvErrTimeout);
                    abort_sh = 1;
                }
                break;
            }
            if (lane == 0) {
                // every CTA is done with stage s - 1: stage s may compute
                if (early)
                    mbar_arrive(&xfull[s & 1]);
                else
                    copy_x(s, true);
                early = false;
                // the other half held stage s - 1's x, which this CTA's warps
                // are done with: copy a run input of stage s + 1 now
                if (s + 1 < n && st[s + 1].xext) {
                    copy_x(s + 1, false);
                    early = true;
                }
            }
            early = __shfl_sync(0xffffffffu, early ? 1 : 0, 0) != 0;
            issued = early ? s + 2 : s + 1;
        }
        // the x copies issued land before the CTA may exit (bounded); an early
        // copy's phase lacks its arrival, so its bytes are waited for by
        // arriving now (the warps no longer wait on it)
        if (lane == 0) {
            if (early) mbar_arrive(&xfull[(issued - 1) & 1]);
            for (int s = issued > 2 ? issued - 2 : 0; s < issued; ++s)
                mbar_wait_bounded(&xfull[s & 1], (s >> 1) & 1);
        }
        __syncwarp();
    } else if (warp == kProdWarp) {
        // --------------------------------------------------- producer warp ---
        // Chunk C of the CTA's ring order goes to slot C % NS, after the
        // compute warps have released the chunk that slot held (C - NS).
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            int slot = 0;
            uint32_t round = 0;
            bool ok = true;
            for (int s = 0; s < n && ok; ++s) {
                const StreamStage& S = st[s];
                int64_t r0;
                int R;
                rows_of(S, cta, G, r0, R);
                const int64_t kb = S.k;  // code bytes per row
                for (int u0 = 0; u0 < R && ok; u0 += S.nrc) {
                    if (round > 0) {
                        ok = !abort_sh && mbar_wait_bounded(&empty[slot], (round - 1) & 1);
                        if (!ok) break;
                    }
                    const int rows = min(S.nrc, R - u0);
                    const int64_t row = r0 + u0;
                    const uint32_t cbytes = static_cast<uint32_t>(rows * kb);
                    const uint32_t sbytes = static_cast<uint32_t>(rows * kb / 16);
                    const uint32_t sb = ring0 + static_cast<uint32_t>(slot) * kSlotBytes;
                    mbar_arrive_expect_tx(&full[slot], S.nmat * (cbytes + sbytes));
                    for (int m = 0; m < S.nmat; ++m) {
                        bulk_g2s_u32(sb + static_cast<uint32_t>(m * S.nrc * kb),
                                     S.codes[m] + row * kb, cbytes, &full[slot], pol);
                        bulk_g2s_u32(sb + kChunkCodes + static_cast<uint32_t>(m * S.nrc * kb / 16),
                                     S.scales[m] + row * (kb / 32), sbytes, &full[slot], pol);
                    }
                    if (++slot == NS) {
                        slot = 0;
                        ++round;
                    }
                }
            }
            if (!ok) {
                if (!abort_sh) atomicOr(&g_stream_err, kGemvErrTimeout);
                abort_sh = 1;
            }
            // the copies issued land before the CTA may exit (bounded)
            for (int i = 0; i < NS; ++i) {
                const uint32_t filled = round * NS + slot;  // chunks issued so far
                const uint32_t c = filled >= static_cast<uint32_t>(NS) ? filled - NS + i : i;
                if (c < filled) mbar_wait_bounded(&full[c % NS], (c / NS) & 1);
            }
        }
        __syncwarp();
    } else {
        // ----------------------------------------------------- compute warp --
        int slot = 0;
        uint32_t ph = 0;  // parity of the current pass over the ring
        bool aborted = false;
        for (int s = 0; s < n && !aborted; ++s) {
            const StreamStage& S = st[s];
            const StreamOut& o = outs[s];
            int64_t r0;
            int R;
            rows_of(S, cta, G, r0, R);
            const int64_t kb = S.k;
            const uint32_t xs = xbuf0 + (s & 1) * xstride;
            bool have_x = false;
            float bv = -FLT_MAX;  // head: this warp's best row of the stage
            int bidx = INT_MAX;
            for (int u0 = 0; u0 < R && !aborted; u0 += S.nrc) {
                const bool okf = mbar_wait_bounded(&full[slot], ph);
                if (!__all_sync(0xffffffffu, okf)) {
                    aborted = true;
                    break;
                }
                const int rows = min(S.nrc, R - u0);
                const uint32_t sb = ring0 + static_cast<uint32_t>(slot) * kSlotBytes;
                // this warp's rows of the chunk: u = u0 + i with u % kSwW == warp
                int i = (warp - u0 % kSwW + kSwW) % kSwW;
                for (; i < rows; i += kSwW) {
                    if (!have_x) {
                        const bool okx = !abort_sh && mbar_wait_bounded(&xfull[s & 1], (s >> 1) & 1);
                        if (!__all_sync(0xffffffffu, okx)) {
                            aborted = true;
                            break;
                        }
                        have_x = true;
                    }
                    float acc0 = 0.f, acc1 = 0.f;
                    const uint32_t ca = sb + static_cast<uint32_t>(i * kb);
                    const uint32_t sa = sb + kChunkCodes + static_cast<uint32_t>(i * kb / 16);
                    if (S.op == kOpSwiglu)
                        row_dot<2>(ca, ca + static_cast<uint32_t>(S.nrc * kb), sa,
                                   sa + static_cast<uint32_t>(S.nrc * kb / 16), xs, S.nst, lane,
                                   acc0, acc1);
                    else
                        row_dot<1>(ca, ca, sa, sa, xs, S.nst, lane, acc0, acc1);
                    acc0 = warp_sum(acc0);
                    if (S.op == kOpSwiglu) acc1 = warp_sum(acc1);
                    if (lane == 0) {
                        const int64_t row = r0 + u0 + i;
                        if (S.op == kOpSwiglu) {
                            o.h[row] = f2h_rn(acc0 / (1.0f + expf(-acc0)) * acc1);
                        } else if (S.op == kOpGemv) {
                            if (o.y) o.y[row] = acc0;
                            if (o.y16) o.y16[row] = f2h_rn(acc0);
                        } else {
                            if (o.logits) o.logits[row] = acc0;
                            if (acc0 > bv) {  // rows arrive in increasing order
                                bv = acc0;
                                bidx = static_cast<int>(row);
                            }
                        }
                    }
                }
                if (aborted) break;
                __syncwarp();  // every lane is done with the slot before it is released
                if (lane == 0) mbar_arrive(&empty[slot]);
                if (++slot == NS) {
                    slot = 0;
                    ph ^= 1u;
                }
            }
            if (aborted) break;
            // Done with stage s: arrive on its completion barrier.  Only once x
            // of stage s - 1 has landed: the sync warp copies it after it has
            // seen stage s - 2 complete, so the barrier of parity s & 1 is then
            // in stage s's phase (a warp without rows must not run two phases
            // ahead).
            if (s >= 1) {
                const bool okp = mbar_wait_bounded(&xfull[(s - 1) & 1], ((s - 1) >> 1) & 1);
                if (!__all_sync(0xffffffffu, okp)) {
                    aborted = true;
                    break;
                }
            }
            if (S.op == kOpHead && lane == 0) {
                best_v[s & 1][warp] = bv;
                best_i[s & 1][warp] = bidx;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sdone[s & 1]);
        }
        if (aborted && lane == 0) {
            if (!abort_sh) atomicOr(&g_stream_err, kGemvErrTimeout);
            abort_sh = 1;
        }
        __syncwarp();
    }

    // The last CTA to get here re-zeroes every grid counter for the next run
    // (no CTA reads a counter after it has got here).
    __syncthreads();
    unsigned int* exit_ctr = ctr + static_cast<size_t>(n) * kSwCtr * kSwCtrStride;
    if (threadIdx.x == 0 && !abort_sh) {
        if (atomicAdd(exit_ctr, 1u) == static_cast<unsigned>(G) - 1) {
            for (size_t i = 0; i < static_cast<size_t>(n) * kSwCtr; ++i) ctr[i * kSwCtrStride] = 0u;
            *exit_ctr = 0u;
            __threadfence();
        }
    }
}

}  // namespace

// ------------------------------------------------------------------ host ---

size_t stream_workspace_bytes(int n_stages) { return sw_bytes(n_stages); }

// Plan: every stage int8 block-32 with k % 512 == 0 and one row (or gate/up
// pair) within a ring slot, at most kSwMaxStages stages, shared memory for the
// descriptors, x and at least kMinSlots ring slots.  Returns QG_ERR_FORMAT /
// QG_ERR_SHAPE when the plan does not qualify (the caller then plans the
// general persistent kernel).
qg_status plan_stream(const GemvLaunch* L, int n, void* ws, size_t ws_bytes, int* slots_out,
                      int* xmax_out) {
    DeviceInfo dev;
    qg_status st = device_info(&dev);
    if (st != QG_OK) return st;
    if (n > kSwMaxStages) return QG_ERR_SHAPE;
    if (ws_bytes < sw_bytes(n)) return QG_ERR_WORKSPACE;
    int xmax = 0;
    for (int i = 0; i < n; ++i) {
        if (L[i].fmt != QG_FMT_I8_B32) return QG_ERR_FORMAT;
        const int64_t nmat = L[i].epilogue == kEpiSwiglu ? 2 : 1;
        if (L[i].k % kSwStep != 0 || L[i].n > (1LL << 30) || nmat * L[i].k > kChunkCodes)
            return QG_ERR_SHAPE;
        if (reinterpret_cast<uintptr_t>(L[i].x) % 16 != 0) return QG_ERR_SHAPE;
        if (L[i].k > xmax) xmax = static_cast<int>(L[i].k);
    }
    const size_t fixed = sw_smem(n, xmax, 0) + 1024;
    if (fixed >= static_cast<size_t>(dev.max_smem_optin)) return QG_ERR_SHAPE;
    int slots = static_cast<int>((static_cast<size_t>(dev.max_smem_optin) - fixed) / kSlotBytes);
    if (slots > kMaxSlots) slots = kMaxSlots;
    if (slots < kMinSlots) return QG_ERR_SHAPE;
    std::vector<unsigned char> host(sw_bytes(n), 0);
    StreamHeader* hdr = reinterpret_cast<StreamHeader*>(host.data());
    hdr->magic = kStreamMagic;
    hdr->n_stages = n;
    hdr->slots = slots;
    hdr->xmax = xmax;
    StreamStage* S = reinterpret_cast<StreamStage*>(host.data() + sw_stage_off(n));
    StreamOut* O = reinterpret_cast<StreamOut*>(host.data() + sw_out_off(n));
    unsigned char* dev_base = static_cast<unsigned char*>(ws);
    // byte ranges every stage writes: an x outside all of them is a run input
    std::vector<std::pair<uintptr_t, uintptr_t>> written;
    for (int i = 0; i < n; ++i) {
        const GemvLaunch& l = L[i];
        auto add = [&](const void* ptr, int64_t bytes) {
            if (ptr) written.emplace_back(reinterpret_cast<uintptr_t>(ptr),
                                          reinterpret_cast<uintptr_t>(ptr) + static_cast<uintptr_t>(bytes));
        };
        add(l.y, l.n * 4);
        add(l.y16, l.n * 2);
        add(l.h, l.n * 2);
        add(l.logits, l.n * 4);
        add(l.idx, 4);
    }
    for (int i = 0; i < n; ++i) {
        const GemvLaunch& l = L[i];
        StreamStage& s = S[i];
        s.codes[0] = static_cast<const uint8_t*>(l.codes[0]);
        s.codes[1] = static_cast<const uint8_t*>(l.codes[l.nmat > 1 ? 1 : 0]);
        s.scales[0] = l.scales[0];
        s.scales[1] = l.scales[l.nmat > 1 ? 1 : 0];
        s.n = static_cast<int32_t>(l.n);
        s.k = static_cast<int32_t>(l.k);
        s.nst = static_cast<int32_t>(l.k / kSwStep);
        const uintptr_t x0 = reinterpret_cast<uintptr_t>(l.x), x1 = x0 + static_cast<uintptr_t>(l.k) * 2;
        s.xext = 1;
        for (const auto& w : written)
            if (x0 < w.second && w.first < x1) s.xext = 0;
        s.op = l.epilogue == kEpiSwiglu ? kOpSwiglu : (l.epilogue == kEpiHead ? kOpHead : kOpGemv);
        s.nmat = l.epilogue == kEpiSwiglu ? 2 : 1;
        s.nrc = static_cast<int32_t>(kChunkCodes / (static_cast<int64_t>(s.nmat) * l.k));
        StreamOut& o = O[i];
        o.x = l.x;
        o.y = l.y;
        o.y16 = l.y16;
        o.h = l.h;
        o.logits = l.logits;
        o.idx = l.idx;
        unsigned char* scr = dev_base + sw_scr_off(n) + 16 * static_cast<size_t>(i);
        o.key = reinterpret_cast<unsigned long long*>(scr);
        o.ticket = reinterpret_cast<unsigned int*>(scr + 8);
    }
    st = cuda_status(cudaMemcpy(ws, host.data(), host.size(), cudaMemcpyHostToDevice));
    if (st == QG_OK) {
        *slots_out = slots;
        *xmax_out = xmax;
    }
    return st;
}

qg_status launch_stream(void* ws, int n, int slots, int xmax, cudaStream_t stream) {
    DeviceInfo dev;
    qg_status st = device_info(&dev);
    if (st != QG_OK) return st;
    if (n < 1 || n > kSwMaxStages || xmax < kSwStep || slots < kMinSlots || slots > kMaxSlots)
        return QG_ERR_PLAN;
    void (*kern)(unsigned char*, int, int) = stream_sweep_kernel;
    const size_t smem = sw_smem(n, xmax, slots);
    if (smem + 1024 > static_cast<size_t>(dev.max_smem_optin)) return QG_ERR_PLAN;
    static size_t attr[64] = {0};
    if (dev.device >= 64 || attr[dev.device] < smem) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return cuda_status(e);
        if (dev.device < 64) attr[dev.device] = smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(dev.num_sms));
    cfg.blockDim = dim3(kSwThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, static_cast<unsigned char*>(ws), n, slots));
}

unsigned int stream_read_and_clear_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_stream_err, sizeof v) != cudaSuccess) return 0;
    if (v) cudaMemcpyToSymbol(g_stream_err, &zero, sizeof zero);
    return v;
}

}  // namespace qg
