// qg_stream.cu -- a whole int8 decode sweep as one persistent launch whose
// weight stream does not stop at stage boundaries.
//
// A decode step reads every decoder weight once ("Qwen3-VL 4B -- Core AI
// (.aimodel)", Measured: decode is the weight read), as an ordered chain of
// S=1 projections in which each stage needs the whole output of the stage
// before it ("Qwen3.8-27B ... -- Core AI", The vision path: prefill runs as
// pipelined S=1 steps).  Only the activation depends on the previous stage,
// never the weights; so every warp streams its own weight rows through a
// deep per-lane shared-memory ring whose copy cursor runs straight on into
// the next stages while the warp waits for the next activation.  With 8-11
// slots per lane and 15 streaming warps per SM, 110-150 KB of weights per SM
// are in flight across each stage boundary.
//
//  * One CTA per SM (cooperative launch): 15 streaming warps + 1 sync warp.
//  * Items: one or two weight rows (a row or row pair of a projection, or the
//    gate and up rows of one SwiGLU output).  Item j of a stage goes to CTA
//    j % G and to warp ((j / G) + rot) % 15 of it; rot turns from stage to
//    stage so that no warp always gets the extra item.
//  * Copy cursor: each lane copies 16 bytes of every row's 512-byte step with
//    cp.async into its warp's ring slot, four lanes copying the step's 16
//    scales; D - 1 steps stay in flight, across stage boundaries.
//  * Compute: lane l takes the 8-byte code pieces at 8 l and 256 + 8 l of a
//    step against x read raw (fp16, as the bulk copy left it) at 16 l and
//    512 + 16 l: conflict-free, so x needs no re-layout.  Codes become exact
//    fp16 q (byte permute into 1024 + (q + 128), packed subtraction of 1152)
//    and the sm_100 mixed-precision FMA accumulates the exact products q x
//    in fp32; the block scale multiplies each 8-code partial.
//  * Sync warp: when every warp of its CTA is done with stage s (an
//    mbarrier), it arrives on the grid counter of stage s (release), waits
//    for every CTA (acquire, bounded) and fetches x of stage s + 1 with one
//    bulk copy into the other half of a double buffer, on an mbarrier the
//    streaming warps wait on.  It also finishes a head stage's argmax for its
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

constexpr int kSwW = 15;                      // streaming warps per CTA
constexpr int kSwThreads = (kSwW + 1) * 32;   // + the sync warp
constexpr int kSwStep = 512;                  // code bytes of one warp step along a row
constexpr int kSwSlotRow = kSwStep + 32;      // codes + the step's 16 fp16 scales
constexpr int kSwSlot = 2 * kSwSlotRow;       // a slot holds up to two rows
constexpr int kSwMaxStages = 320;
constexpr uint32_t kStreamMagic = 0x32575351u;

enum StreamOp : int32_t { kOpGemv = 0, kOpSwiglu = 1, kOpHead = 2 };

// What the warps' cursors read of a stage (kept in shared memory).
struct StreamStage {
    const uint8_t* codes[2];    // gemv/head: [0]; swiglu: gate, up
    const uint16_t* scales[2];
    int32_t n, k;               // rows, columns (k % 512 == 0)
    int32_t items;              // work items of the stage
    int32_t op;                 // StreamOp
    int32_t rows;               // rows per item: 1 or 2
    int32_t rot;                // warp rotation of the item assignment
    int32_t nst;                // steps per row: k / 512
    int32_t xext;               // x is a run input: no stage of the plan writes it
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
    int32_t depth;              // ring slots per lane the plan was made for
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
__host__ __device__ constexpr size_t sw_smem(int n, int xmax, int depth) {
    return sw_desc_bytes(n) + 2 * sw_x_bytes(xmax) + static_cast<size_t>(kSwW) * depth * kSwSlot;
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

__device__ __forceinline__ void cp16(uint32_t dst, const void* src, uint64_t pol) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst),
                 "l"(src), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_g2s_u32(uint32_t dst, const void* src, uint32_t bytes,
                                             uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}
// Ask L2 to fetch [p, p + bytes) (16-byte aligned, a multiple of 16): a hint
// with no completion to track.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
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
// 8 int8 codes against their 8 fp16 x: sum q x with exact products.
__device__ __forceinline__ float dot8(uint2 c, uint4 x) {
    float a0 = 0.f, a1 = 0.f;
    const uint32_t u0 = c.x ^ 0x80808080u, u1 = c.y ^ 0x80808080u;
    fma_mixed(a0, a1, hsub2s(__byte_perm(u0, 0x64646464u, 0x4140), 0x64806480u), x.x);
    fma_mixed(a0, a1, hsub2s(__byte_perm(u0, 0x64646464u, 0x4342), 0x64806480u), x.y);
    fma_mixed(a0, a1, hsub2s(__byte_perm(u1, 0x64646464u, 0x4140), 0x64806480u), x.z);
    fma_mixed(a0, a1, hsub2s(__byte_perm(u1, 0x64646464u, 0x4342), 0x64806480u), x.w);
    return a0 + a1;
}

__device__ __forceinline__ unsigned long long key_of(float v, int idx) {
    uint32_t b = __float_as_uint(v);
    b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);  // order-preserving
    return (static_cast<unsigned long long>(b) << 32) |
           static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(idx));
}

// A warp's walk over the plan: stage s, its m-th item there (global item
// index `item`), and the step within the item's rows.
struct Cursor {
    int s, m, step;
    int64_t item;
};

// Item m of stage `st` for warp w of CTA cta (-1 if the warp has none).
__device__ __forceinline__ int64_t item_of(const StreamStage& st, int cta, int w, int G, int m) {
    const int wr = (w - st.rot + kSwW) % kSwW;  // rot < kSwW
    const int64_t j = static_cast<int64_t>(cta) +
                      static_cast<int64_t>(G) * (wr + static_cast<int64_t>(kSwW) * m);
    return j < st.items ? j : -1;
}

// Position c at the first existing item at or after (c.s, c.m); c.s == n
// when the plan is exhausted.
__device__ __forceinline__ void seek(Cursor& c, const StreamStage* st, int n, int cta, int w,
                                     int G) {
    c.step = 0;
    while (c.s < n) {
        c.item = item_of(st[c.s], cta, w, G, c.m);
        if (c.item >= 0) return;
        ++c.s;
        c.m = 0;
    }
}

// Row r (0 or 1) of item j of stage st, clamped into the matrix (a second
// row past the end is copied and discarded), and the matrix it lies in.
__device__ __forceinline__ int64_t item_row(const StreamStage& st, int64_t j, int r, int* mat) {
    if (st.op == kOpSwiglu) {
        *mat = r;
        return j;
    }
    *mat = 0;
    const int64_t row = j * st.rows + r;
    return row < st.n ? row : st.n - 1;
}

template <int D>
__global__ void __launch_bounds__(kSwThreads, 1) stream_sweep_kernel(unsigned char* ws, int n) {
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ __align__(8) uint64_t xfull[2];  // x of stage s landed (tx bytes)
    __shared__ __align__(8) uint64_t sdone[2];  // every streaming warp done with stage s
    __shared__ float best_v[2][kSwW];
    __shared__ int best_i[2][kSwW];
    __shared__ volatile int abort_sh;

    const StreamHeader* hdr = reinterpret_cast<const StreamHeader*>(ws);
    uint32_t dyn_smem;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_smem));
    if (hdr->magic != kStreamMagic || hdr->n_stages != n || hdr->depth != D ||
        hdr->xmax < kSwStep || sw_smem(n, hdr->xmax, D) > dyn_smem) {
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
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kSwW) {
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
    } else {
        // ---------------------------------------------------- streaming warp --
        const uint64_t pol = l2_policy_evict_first();
        const uint32_t ring = ring0 + static_cast<uint32_t>(warp) * D * kSwSlot;
        // copy cursor: the item it copies, with this lane's source pointers of
        // that item's rows (advanced by one step per copy)
        Cursor cc = {0, 0, 0, -1};
        seek(cc, st, n, cta, warp, G);
        int cslot = 0;
        const uint8_t* cp0 = nullptr;   // row 0 codes, this lane's 16 bytes
        const uint8_t* cp1 = nullptr;   // row 1 codes
        const uint16_t* cps = nullptr;  // side lanes 0-3: scales of row lane >> 1, piece lane & 1
        int cleft = 0;                  // steps of the item left to copy
        bool ctwo = false;              // the item has two rows
        auto load_item = [&]() {
            const StreamStage& S = st[cc.s];
            int m0, m1;
            const int64_t r0 = item_row(S, cc.item, 0, &m0);
            const int64_t r1 = item_row(S, cc.item, 1, &m1);
            ctwo = S.rows == 2 || S.op == kOpSwiglu;
            cp0 = S.codes[m0] + r0 * S.k + lane * 16;
            cp1 = S.codes[m1] + r1 * S.k + lane * 16;
            if (lane == 0) {
                // ask L2 for the whole item now: its later steps' copies then
                // hit L2 instead of waiting out HBM latency one step at a time
                const uint8_t* c0 = S.codes[m0] + r0 * S.k;
                const uint8_t* c1 = S.codes[m1] + r1 * S.k;
                const uint32_t sb = static_cast<uint32_t>(S.k / 16);  // scale bytes per row
                if (ctwo && m0 == m1 && r1 == r0 + 1) {
                    prefetch_l2_bulk(c0, static_cast<uint32_t>(2 * S.k));
                    prefetch_l2_bulk(S.scales[m0] + r0 * (S.k / 32), 2 * sb);
                } else {
                    prefetch_l2_bulk(c0, static_cast<uint32_t>(S.k));
                    prefetch_l2_bulk(S.scales[m0] + r0 * (S.k / 32), sb);
                    if (ctwo) {
                        prefetch_l2_bulk(c1, static_cast<uint32_t>(S.k));
                        prefetch_l2_bulk(S.scales[m1] + r1 * (S.k / 32), sb);
                    }
                }
            }
            const bool srow1 = (lane >> 1) & 1;
            cps = S.scales[srow1 ? m1 : m0] + (srow1 ? r1 : r0) * (S.k / 32) + (lane & 1) * 8;
            cleft = S.nst;
        };
        if (cc.s < n) load_item();
        const bool side_lane = lane < 4;
        const uint32_t side_off = static_cast<uint32_t>((lane >> 1) * kSwSlotRow + kSwStep + (lane & 1) * 16);
        auto issue = [&]() {
            if (cleft > 0) {
                const uint32_t dst = ring + cslot * kSwSlot + lane * 16;
                cp16(dst, cp0, pol);
                if (ctwo) cp16(dst + kSwSlotRow, cp1, pol);
                if (side_lane && (lane < 2 || ctwo))
                    cp16(ring + cslot * kSwSlot + side_off, cps, pol);
                cp0 += kSwStep;
                cp1 += kSwStep;
                cps += 16;
                if (--cleft == 0) {
                    ++cc.m;
                    seek(cc, st, n, cta, warp, G);
                    if (cc.s < n) load_item();
                }
            }
            cp_commit();
            if (++cslot == D) cslot = 0;
        };
#pragma unroll 1
        for (int d = 0; d < D - 1; ++d) issue();

        // compute cursor
        Cursor uc = {0, 0, 0, -1};
        int uslot = 0;
        int cur = -1;  // the stage whose x this warp has waited for
        float bv = -FLT_MAX;
        int bi = INT_MAX;
        bool aborted = false;
        // stages before (and including) `upto` that this warp has no more
        // items in: arrive on their completion barriers, in order
        int arrived = 0;  // stages 0 .. arrived-1 arrived
        auto arrive_until = [&](int upto) -> bool {
            for (; arrived < upto; ++arrived) {
                const int s = arrived;
                // Arrive for stage s only once x of stage s - 1 has landed: the
                // sync warp copies it after it has seen stage s - 2 complete,
                // so the barrier of parity s & 1 is then in stage s's phase
                // (a warp without items must not run two phases ahead).
                if (s >= 1 && !mbar_wait_bounded(&xfull[(s - 1) & 1], ((s - 1) >> 1) & 1))
                    return false;
                if (st[s].op == kOpHead) {
                    // best of this warp in stage s (its head rows), then arrive
                    if (lane == 0) {
                        best_v[s & 1][warp] = s == cur ? bv : -FLT_MAX;
                        best_i[s & 1][warp] = s == cur ? bi : INT_MAX;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sdone[s & 1]);
            }
            return true;
        };
        seek(uc, st, n, cta, warp, G);
        while (uc.s < n) {
            const StreamStage& S = st[uc.s];
            if (uc.s != cur) {
                // finish the stages before this one, then wait for its x
                if (!arrive_until(uc.s)) {
                    aborted = true;
                    break;
                }
                cur = uc.s;
                bv = -FLT_MAX;
                bi = INT_MAX;
                if (abort_sh || !mbar_wait_bounded(&xfull[cur & 1], (cur >> 1) & 1)) {
                    aborted = true;
                    break;
                }
            }
            uint32_t xp = xbuf0 + (cur & 1) * xstride + lane * 16;  // this lane's x pieces
            const bool two = S.op == kOpSwiglu || S.rows == 2;
            const int nst = S.nst;
            float acc0 = 0.f, acc1 = 0.f;
            for (int step = 0; step < nst; ++step) {
                issue();
                cp_wait<D - 1>();
                __syncwarp();  // every lane's copies of this slot are visible
                const uint32_t slot = ring + uslot * kSwSlot;
                const uint4 xa = lds128s(xp);
                const uint4 xb = lds128s(xp + kSwStep);
                xp += kSwStep * 2;
                {
                    const uint2 ca = lds64(slot + lane * 8);
                    const uint2 cb = lds64(slot + 256 + lane * 8);
                    const float sa = h2f(lds16s(slot + kSwStep + (lane >> 2) * 2));
                    const float sb = h2f(lds16s(slot + kSwStep + 16 + (lane >> 2) * 2));
                    acc0 = fmaf(sa, dot8(ca, xa), fmaf(sb, dot8(cb, xb), acc0));
                }
                if (two) {
                    const uint32_t s1 = slot + kSwSlotRow;
                    const uint2 ca = lds64(s1 + lane * 8);
                    const uint2 cb = lds64(s1 + 256 + lane * 8);
                    const float sa = h2f(lds16s(s1 + kSwStep + (lane >> 2) * 2));
                    const float sb = h2f(lds16s(s1 + kSwStep + 16 + (lane >> 2) * 2));
                    acc1 = fmaf(sa, dot8(ca, xa), fmaf(sb, dot8(cb, xb), acc1));
                }
                __syncwarp();  // every lane is done with the slot before it is refilled
                if (++uslot == D) uslot = 0;
            }
            acc0 = warp_sum(acc0);
            acc1 = warp_sum(acc1);
            if (lane == 0) {
                const StreamOut& o = outs[uc.s];
                if (S.op == kOpSwiglu) {
                    o.h[uc.item] = f2h_rn(acc0 / (1.0f + expf(-acc0)) * acc1);
                } else {
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const int64_t row = uc.item * S.rows + r;
                        if (r < S.rows && row < S.n) {
                            const float v = r == 0 ? acc0 : acc1;
                            if (S.op == kOpGemv) {
                                if (o.y) o.y[row] = v;
                                if (o.y16) o.y16[row] = f2h_rn(v);
                            } else {
                                if (o.logits) o.logits[row] = v;
                                if (v > bv) {  // rows arrive in increasing order
                                    bv = v;
                                    bi = static_cast<int>(row);
                                }
                            }
                        }
                    }
                }
            }
            ++uc.m;
            seek(uc, st, n, cta, warp, G);
        }
        if (!aborted && !arrive_until(n)) aborted = true;
        if (aborted) {
            if (lane == 0) {
                if (!abort_sh) atomicOr(&g_stream_err, kGemvErrTimeout);
                abort_sh = 1;
            }
        }
        cp_wait<0>();  // this lane's copies land before the CTA may exit
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

// Plan: every stage int8 block-32 with k % 512 == 0, at most kSwMaxStages
// stages, shared memory for the descriptors, x and the rings at depth 11 or
// at least 8.  Returns QG_ERR_FORMAT / QG_ERR_SHAPE when the plan does not
// qualify (the caller then plans the general persistent kernel).
qg_status plan_stream(const GemvLaunch* L, int n, void* ws, size_t ws_bytes, int* depth_out,
                      int* xmax_out) {
    DeviceInfo dev;
    qg_status st = device_info(&dev);
    if (st != QG_OK) return st;
    if (n > kSwMaxStages) return QG_ERR_SHAPE;
    if (ws_bytes < sw_bytes(n)) return QG_ERR_WORKSPACE;
    int xmax = 0;
    for (int i = 0; i < n; ++i) {
        if (L[i].fmt != QG_FMT_I8_B32) return QG_ERR_FORMAT;
        if (L[i].k % kSwStep != 0 || L[i].n > (1LL << 30)) return QG_ERR_SHAPE;
        if (L[i].k > xmax) xmax = static_cast<int>(L[i].k);
    }
    int depth = 0;
    for (int d : {11, 8})
        if (sw_smem(n, xmax, d) + 1024 <= static_cast<size_t>(dev.max_smem_optin)) {
            depth = d;
            break;
        }
    if (depth == 0) return QG_ERR_SHAPE;
    const int G = dev.num_sms;
    std::vector<unsigned char> host(sw_bytes(n), 0);
    StreamHeader* hdr = reinterpret_cast<StreamHeader*>(host.data());
    hdr->magic = kStreamMagic;
    hdr->n_stages = n;
    hdr->depth = depth;
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
        s.rot = static_cast<int32_t>((i * 7) % kSwW);
        const uintptr_t x0 = reinterpret_cast<uintptr_t>(l.x), x1 = x0 + static_cast<uintptr_t>(l.k) * 2;
        s.xext = 1;
        for (const auto& w : written)
            if (x0 < w.second && w.first < x1) s.xext = 0;
        if (l.epilogue == kEpiSwiglu) {
            s.op = kOpSwiglu;
            s.rows = 2;
            s.items = static_cast<int32_t>(l.n);
        } else {
            s.op = l.epilogue == kEpiHead ? kOpHead : kOpGemv;
            // two rows per item: every ring slot carries two rows' steps (a
            // warp without an item in a small stage streams ahead instead)
            s.rows = l.n >= 2 ? 2 : 1;
            s.items = static_cast<int32_t>((l.n + s.rows - 1) / s.rows);
        }
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
        *depth_out = depth;
        *xmax_out = xmax;
    }
    return st;
}

qg_status launch_stream(void* ws, int n, int depth, int xmax, cudaStream_t stream) {
    DeviceInfo dev;
    qg_status st = device_info(&dev);
    if (st != QG_OK) return st;
    if (n < 1 || n > kSwMaxStages || xmax < kSwStep) return QG_ERR_PLAN;
    void (*kern)(unsigned char*, int);
    if (depth == 11) {
        kern = stream_sweep_kernel<11>;
    } else if (depth == 8) {
        kern = stream_sweep_kernel<8>;
    } else {
        return QG_ERR_PLAN;
    }
    const size_t smem = sw_smem(n, xmax, depth);
    if (smem + 1024 > static_cast<size_t>(dev.max_smem_optin)) return QG_ERR_PLAN;
    static size_t attr[2][64] = {{0}};
    const int ki = depth == 11 ? 0 : 1;
    if (dev.device >= 64 || attr[ki][dev.device] < smem) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return cuda_status(e);
        if (dev.device < 64) attr[ki][dev.device] = smem;
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
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, static_cast<unsigned char*>(ws), n));
}

unsigned int stream_read_and_clear_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_stream_err, sizeof v) != cudaSuccess) return 0;
    if (v) cudaMemcpyToSymbol(g_stream_err, &zero, sizeof zero);
    return v;
}

}  // namespace qg
