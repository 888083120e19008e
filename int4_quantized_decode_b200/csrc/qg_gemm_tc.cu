// qg_gemm_tc.cu -- chunked prefill on the fifth-generation tensor cores: S <= 16
// tokens through int8 block-32 or int4 group-64 weights ("Qwen3.8-27B ... --
// Core AI", The vision path: a static 16-token 'prefill' function next to the
// one-token decode step; "Qwen3-VL 4B & 8B -- Core ML stateful", Architecture:
// the INT4 group-64 variant).
//
//   Y[s, r] = sum_k X[s, k] w_dq[r, k]      (plain, fp32 out)
//   H[s, r] = fp16( silu(g) u )             (fused gate/up SwiGLU)
//
// Sixteen tokens share every weight, so the path is a dense contraction and
// runs on tcgen05.mma; it stays bound by the weight stream (32 flop per
// 1.06 B of int8, per 0.56 B of int4), far below the tensor-core ridge.
//
// One CTA computes a 128-row weight tile (M = 128) for all 16 tokens (N = 16)
// over a K range; the CTAs of a thread-block cluster split K and reduce their
// fp32 partials through distributed shared memory in a fixed rank order
// (deterministic, no global workspace).  Warp roles:
//
//  * warp 0, one thread -- producer: TMA (cp.async.bulk.tensor.2d, this GPU's
//    memory only, no multicast) copies each stage's code tile (128 rows x 128
//    bytes, 128-byte swizzle) and the X chunk (16 rows x 64 fp16 per box,
//    128-byte swizzle, rows >= S filled with zeros by the copy) into a ring of
//    shared-memory stages on one mbarrier each.  Codes do not depend on the
//    previous kernel and are requested before griddepcontrol.wait; X after.
//  * warps 2..9 -- dequantize: thread = weight row (its warp's quarter of the
//    tensor-memory lanes), two warps per quarter taking alternate 16-k steps.
//    Each turns its row's 16 codes of a step into fp16(q s) (int8: byte
//    permute into 1024 + u, exact subtraction, one rounding by the block
//    scale) or fp16(q s + b) (int4: one fused rounding) and stores them into
//    tensor memory (tcgen05.st), where the MMA reads its A operand.
//  * warp 1 -- allocates tensor memory; one thread issues tcgen05.mma
//    kind::f16 (A from tensor memory, B = X from shared memory through a
//    128-byte-swizzle K-major descriptor, fp32 accumulator D in tensor
//    memory) and tcgen05.commit to release A slots and X stages.
//  * epilogue: tcgen05.ld of D (thread = row, 16 columns = tokens), split-K
//    reduction over the cluster, fp32 or SwiGLU fp16 store.
//
// Every wait is bounded: a wait that gives up sets the CTA's abort flag and
// the device error flag; the CTA then skips its remaining work, drains its
// own copies and MMAs (bounded), frees its tensor memory and still takes part
// in every cluster barrier, so no peer waits forever.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "qg_device.cuh"
#include "qg_internal.h"

namespace qg {

QG_DEFINE_ERROR_FLAG(g_tc_err);

namespace {

constexpr int kTcRows = 128;       // M of one MMA: weight rows of a tile
constexpr int kTcTokens = 16;      // N of one MMA: tokens (rows of X)
constexpr int kKStep = 16;         // K of one tcgen05.mma kind::f16
constexpr int kCodeBox = 128;      // bytes of codes per tile row per stage (swizzle span)
constexpr int kXBoxK = 64;         // k per X box (128 bytes of fp16)
constexpr int kXBoxBytes = kTcTokens * kXBoxK * 2;  // 2 KB
constexpr int kCodeTileBytes = kTcRows * kCodeBox;  // 16 KB
constexpr int kStages = 4;
constexpr int kDqWarps = 8;
constexpr int kThreadsTc = (2 + kDqWarps) * 32;
constexpr int kMaxClusterTc = 8;

template <int FMT>
struct TcFmt {
    static constexpr int kStageK = FMT == 0 ? 128 : 256;  // k per stage: one 128-byte box row
    static constexpr int kKSteps = kStageK / kKStep;       // 8 or 16
    static constexpr int kXBoxes = kStageK / kXBoxK;       // 2 or 4
    static constexpr int kGroup = FMT == 0 ? 32 : 64;      // k per scale (and bias)
};

template <int FMT, int NMAT>
struct TcLayout {
    using F = TcFmt<FMT>;
    static constexpr int kStageBytes = NMAT * kCodeTileBytes + F::kXBoxes * kXBoxBytes;
    static constexpr int kSmem = kStages * kStageBytes;          // + 1 KB alignment slack
    // Two single-weight CTAs fit on an SM (shared memory) and share its 512
    // tensor-memory columns; a gate/up CTA is alone on its SM and takes all.
    static constexpr uint32_t kTmemCols = NMAT == 1 ? 256 : 512;
    // tensor memory: D_m at columns [16 m, 16 m + 16); A slots after it, each
    // NMAT x 8 columns (16 fp16 of K per lane)
    static constexpr int kDCols = 16 * NMAT;
    static constexpr int kASlots = (static_cast<int>(kTmemCols) - kDCols) / (8 * NMAT) / 2 * 2;
    // a dequant warp writes all its A slots of a stage before it signals
    // them, so the ring must hold a whole stage beyond the one being read
    static_assert(kASlots >= F::kKSteps, "tensor memory holds too few A slots");
    static_assert(kStageBytes % 1024 == 0, "stages keep 1024-byte alignment");
    static_assert(NMAT == 1 || kSmem > 116 * 1024, "a gate/up CTA must be alone on its SM");
    static constexpr int kCtasPerSm = NMAT == 1 ? 2 : 1;
};

struct TcParams {
    const uint16_t* scales[2];
    const uint16_t* biases[2];
    float* Y;
    uint16_t* H;
    int64_t n, k;
    int S;
    int splits;  // CTAs of a cluster along K
};

// ----------------------------------------------------------- PTX helpers ---
__device__ __forceinline__ uint32_t cluster_ctarank_tc() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Every thread of the CTA arrives (release) and waits (acquire): the
// non-.aligned form, safe whatever the warp's convergence.
__device__ __forceinline__ void cluster_barrier() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ float ld_dsmem(uint32_t local_addr, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[d] (+)= A[a] (tensor memory) x B (shared memory descriptor)
__device__ __forceinline__ void tc_mma_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// arrive on `bar` once every tcgen05.mma this thread issued so far completed
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tc_st8(uint32_t taddr, const uint32_t (&v)[8]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
        : "memory");
}
__device__ __forceinline__ void tc_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Instruction descriptor of kind::f16: fp16 A and B, both K-major, fp32 D,
// M = 128 (bits 24-28: M >> 4), N = 16 (bits 17-22: N >> 3), D format f32
// (bits 4-5 = 1).
constexpr uint32_t kIdescF16M128N16 = (1u << 4) | (static_cast<uint32_t>(kTcTokens >> 3) << 17) |
                                      (static_cast<uint32_t>(kTcRows >> 4) << 24);

// Shared-memory descriptor of a K-major operand in the 128-byte swizzle
// layout that TMA writes for a box 128 bytes wide: 8-row groups 1024 bytes
// apart (stride byte offset), start address in 16-byte units, version 1,
// layout 2 (128-byte swizzle); the leading byte offset is unused (1).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (1ull << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ uint32_t hsub2_tc(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t hmul2_tc(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t hfma2_tc(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// 16 int8 codes (k order) -> 8 registers of fp16 pairs fp16(q s), one
// rounding: byte permute into 1024 + (q + 128), exact subtraction of 1152,
// multiply by the block scale s2 = (s, s).
__device__ __forceinline__ void dequant16_i8(uint4 c, uint32_t s2, uint32_t (&a)[8]) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t u = w[i] ^ 0x80808080u;
        a[2 * i] = hmul2_tc(hsub2_tc(__byte_perm(u, 0x64646464u, 0x4140), 0x64806480u), s2);
        a[2 * i + 1] = hmul2_tc(hsub2_tc(__byte_perm(u, 0x64646464u, 0x4342), 0x64806480u), s2);
    }
}

// 16 int4 codes (two words, even k in the low nibble) -> 8 registers of fp16
// pairs fp16(q s + b), one fused rounding per weight.  Masks give the pairs
// (k, k + 4) of a word; a byte permute restores the (k, k + 1) pairs.
__device__ __forceinline__ void dequant16_i4(uint2 c, uint32_t s2, uint32_t b2, uint32_t (&a)[8]) {
    const uint32_t w[2] = {c.x, c.y};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint32_t v = w[i];
        uint32_t p[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t m = ((v >> (4 * j)) & 0x000F000Fu) | 0x64006400u;  // (k_j, k_j+4) + 1024
            p[j] = hfma2_tc(hsub2_tc(m, 0x64006400u), s2, b2);
        }
        a[4 * i + 0] = __byte_perm(p[0], p[1], 0x5410);  // (k0, k1)
        a[4 * i + 1] = __byte_perm(p[2], p[3], 0x5410);  // (k2, k3)
        a[4 * i + 2] = __byte_perm(p[0], p[1], 0x7632);  // (k4, k5)
        a[4 * i + 3] = __byte_perm(p[2], p[3], 0x7632);  // (k6, k7)
    }
}

__device__ __forceinline__ uint32_t half2_bits(uint16_t h) {
    return static_cast<uint32_t>(h) | (static_cast<uint32_t>(h) << 16);
}

// Bounded mbarrier wait that gives up at once when the CTA already aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort) {
    if (*abort) return false;
    if (mbar_wait_bounded(bar, parity)) return true;
    *abort = 1;
    atomicOr(&g_tc_err, kGemvErrTimeout);
    return false;
}

// The same for a whole warp: every lane waits (so every lane has observed the
// phase), and the outcome is made warp-uniform, so that the warp-collective
// tcgen05 instructions that follow run converged or not at all.
__device__ __forceinline__ bool warp_wait_or_abort(uint64_t* bar, uint32_t parity,
                                                   volatile int* abort) {
    const bool ok = wait_or_abort(bar, parity, abort);
    return __all_sync(0xffffffffu, ok);
}

template <int FMT, int NMAT, int EPI>
__global__ void __launch_bounds__(kThreadsTc, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_codes0,
                   const __grid_constant__ CUtensorMap tm_codes1,
                   const __grid_constant__ CUtensorMap tm_x, const TcParams p) {
    using F = TcFmt<FMT>;
    using L = TcLayout<FMT, NMAT>;
    constexpr int KSTEPS = F::kKSteps;
    constexpr int NA = L::kASlots;
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kStages];
    __shared__ __align__(8) uint64_t empty_bar[kStages];
    __shared__ __align__(8) uint64_t afull_bar[NA];
    __shared__ __align__(8) uint64_t aempty_bar[NA];
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;

    // stages start on a 1024-byte boundary (the 128-byte swizzle atom)
    const uint32_t sraw = smem_u32(smem_raw);
    const uint32_t sbase = (sraw + 1023u) & ~1023u;
    unsigned char* sgen = smem_raw + (sbase - sraw);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = p.splits;
    const uint32_t rank = P > 1 ? cluster_ctarank_tc() : 0u;
    const int64_t tile = blockIdx.x / P;
    const int64_t row0 = tile * kTcRows;
    // this CTA's K range: stages [st0, st1) of the row, split as evenly as the
    // stage count allows
    const int total_st = static_cast<int>(p.k / F::kStageK);
    const int st0 = static_cast<int>(rank) * total_st / P;
    const int st1 = (static_cast<int>(rank) + 1) * total_st / P;
    const int64_t kbeg = static_cast<int64_t>(st0) * F::kStageK;
    const int nstages = st1 - st0;
    const int nsteps = nstages * KSTEPS;

    if (threadIdx.x == 0) {
        abort_sh = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], kDqWarps + 1);
        }
        for (int j = 0; j < NA; ++j) {
            mbar_init(&afull_bar[j], 4);
            mbar_init(&aempty_bar[j], 1);
        }
        mbar_init(&done_bar, 1);
        fence_mbar_init();
        prefetch_tmap(&tm_codes0);
        if (NMAT == 2) prefetch_tmap(&tm_codes1);
        prefetch_tmap(&tm_x);
    }
    if (warp == 1) {  // tensor memory for D and the A slots (whole warp)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&tmem_base_sh)),
                     "r"(L::kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    // the next kernel in the stream may start its own prologue now (its reads
    // of our outputs wait for our completion in griddepcontrol.wait)
    griddep_launch_dependents();

    auto stage_codes = [&](int slot, int m) -> uint32_t {
        return sbase + slot * L::kStageBytes + m * kCodeTileBytes;
    };
    auto stage_x = [&](int slot) -> uint32_t {
        return sbase + slot * L::kStageBytes + NMAT * kCodeTileBytes;
    };
    auto a_col = [&](int slot, int m) -> uint32_t {
        return static_cast<uint32_t>(L::kDCols + (slot * NMAT + m) * 8);
    };

    if (warp == 0) {
        // ------------------------------------------------------- producer ---
        if (lane == 0) {
            const uint64_t pol_w = l2_policy_evict_first();
            const uint64_t pol_x = l2_policy_evict_last();
            const int code_bytes_per_k = FMT == 0 ? 1 : 0;  // int8: 1 byte per k; int4: 1/2
            auto code_c0 = [&](int st) -> int {
                const int64_t k0 = kbeg + static_cast<int64_t>(st) * F::kStageK;
                return static_cast<int>(code_bytes_per_k ? k0 : k0 / 2);
            };
            auto issue_codes = [&](int st) {
                const int slot = st % kStages;
                mbar_arrive_expect_tx(&full_bar[slot], L::kStageBytes);
                tma_load_2d(stage_codes(slot, 0), &tm_codes0, code_c0(st), static_cast<int>(row0),
                            &full_bar[slot], pol_w);
                if (NMAT == 2)
                    tma_load_2d(stage_codes(slot, 1), &tm_codes1, code_c0(st),
                                static_cast<int>(row0), &full_bar[slot], pol_w);
            };
            auto issue_x = [&](int st) {
                const int slot = st % kStages;
                const int64_t k0 = kbeg + static_cast<int64_t>(st) * F::kStageK;
#pragma unroll
                for (int b = 0; b < F::kXBoxes; ++b)
                    tma_load_2d(stage_x(slot) + b * kXBoxBytes, &tm_x,
                                static_cast<int>(k0 + b * kXBoxK), 0, &full_bar[slot], pol_x);
            };
            // codes of the first stages before the wait on the previous kernel
            const int pre = nstages < kStages ? nstages : kStages;
            for (int st = 0; st < pre; ++st) issue_codes(st);
            griddep_wait();
            for (int st = 0; st < pre; ++st) issue_x(st);
            for (int st = kStages; st < nstages; ++st) {
                const int slot = st % kStages;
                if (!wait_or_abort(&empty_bar[slot], ((st / kStages) - 1) & 1, &abort_sh)) break;
                issue_codes(st);
                issue_x(st);
            }
            // drain: every issued copy lands before the CTA may exit (bounded)
            const int first = nstages > kStages ? nstages - kStages : 0;
            for (int st = first; st < nstages; ++st)
                mbar_wait_bounded(&full_bar[st % kStages], (st / kStages) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA ---
        if (lane == 0) {
            for (int t = 0; t < nsteps; ++t) {
                const int st = t / KSTEPS, kk = t % KSTEPS;
                const int slot = st % kStages;
                const int a = t % NA;
                if (kk == 0 && !wait_or_abort(&full_bar[slot], (st / kStages) & 1, &abort_sh)) break;
                if (!wait_or_abort(&afull_bar[a], (t / NA) & 1, &abort_sh)) break;
                tc_fence_after();
                const uint64_t bdesc = sw128_kmajor_desc(stage_x(slot) + (kk / 4) * kXBoxBytes +
                                                         (kk % 4) * (kKStep * 2));
#pragma unroll
                for (int m = 0; m < NMAT; ++m)
                    tc_mma_ts(tmem + 16 * m, tmem + a_col(a, m), bdesc, kIdescF16M128N16,
                              t > 0 ? 1u : 0u);
                tc_commit(&aempty_bar[a]);                     // A slot free once read
                if (kk == KSTEPS - 1) tc_commit(&empty_bar[slot]);  // X of this stage read
            }
            tc_commit(&done_bar);  // every MMA issued above has completed
        }
    } else {
        // ---------------------------------------------------- dequantize ---
        const int dq = warp - 2;              // 0..7
        const int quarter = warp & 3;         // tensor-memory lanes 32*quarter .. +31
        const int half = dq >> 2;             // this warp's parity of 16-k steps
        const int rl = quarter * 32 + lane;   // row within the tile
        const int64_t grow = row0 + rl < p.n ? row0 + rl : p.n - 1;  // tail rows: discard
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const int64_t sides_per_row = p.k / F::kGroup;
        const uint16_t* srow[NMAT];
        const uint16_t* brow[NMAT];
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
            srow[m] = p.scales[m] + grow * sides_per_row + kbeg / F::kGroup;
            brow[m] = FMT == 1 ? p.biases[m] + grow * sides_per_row + kbeg / F::kGroup : nullptr;
        }
        // the row's 4 scales (and biases) of a stage: 8 bytes each
        auto load_sides = [&](int st, uint2 (&sv)[NMAT], uint2 (&bv)[NMAT]) {
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
                sv[m] = __ldg(reinterpret_cast<const uint2*>(srow[m] + st * 4));
                if (FMT == 1) bv[m] = __ldg(reinterpret_cast<const uint2*>(brow[m] + st * 4));
            }
        };
        uint2 sv[NMAT], bv[NMAT], sv_next[NMAT], bv_next[NMAT];
        if (nstages > 0) load_sides(0, sv, bv);
        const int r7 = rl & 7;
        for (int st = 0; st < nstages; ++st) {
            const int slot = st % kStages;
            if (st + 1 < nstages) load_sides(st + 1, sv_next, bv_next);
            if (!warp_wait_or_abort(&full_bar[slot], (st / kStages) & 1, &abort_sh)) break;
            bool ok = true;
            // every A slot of this warp's steps of the stage is written, then
            // one wait for the stores signals them all
            for (int kk = half; kk < KSTEPS; kk += 2) {
                const int t = st * KSTEPS + kk;
                const int a = t % NA;
                if (t >= NA && !warp_wait_or_abort(&aempty_bar[a], ((t / NA) - 1) & 1, &abort_sh)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    uint32_t av[8];
                    const uint32_t tile_row = stage_codes(slot, m) + rl * kCodeBox;
                    if (FMT == 0) {
                        // 16 codes = 16-byte chunk kk of the row, swizzled by row % 8
                        const uint4 c = *reinterpret_cast<const uint4*>(
                            sgen + (tile_row - sbase) + ((kk ^ r7) << 4));
                        const uint32_t sw = (kk >> 1) < 2 ? sv[m].x : sv[m].y;
                        const uint16_t s = static_cast<uint16_t>(((kk >> 1) & 1) ? sw >> 16 : sw & 0xFFFFu);
                        dequant16_i8(c, half2_bits(s), av);
                    } else {
                        // 16 codes = 8 bytes: half (kk & 1) of chunk kk / 2
                        const uint2 c = *reinterpret_cast<const uint2*>(
                            sgen + (tile_row - sbase) + ((((kk >> 1) ^ r7) << 4) | ((kk & 1) << 3)));
                        const int g = kk >> 2;  // group of 64 within the stage
                        const uint32_t sw = g < 2 ? sv[m].x : sv[m].y;
                        const uint32_t bw = g < 2 ? bv[m].x : bv[m].y;
                        const uint16_t s = static_cast<uint16_t>((g & 1) ? sw >> 16 : sw & 0xFFFFu);
                        const uint16_t b = static_cast<uint16_t>((g & 1) ? bw >> 16 : bw & 0xFFFFu);
                        dequant16_i4(c, half2_bits(s), half2_bits(b), av);
                    }
                    tc_st8(tmem + lane_addr + a_col(a, m), av);
                }
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (ok)
                    for (int kk = half; kk < KSTEPS; kk += 2)
                        mbar_arrive(&afull_bar[(st * KSTEPS + kk) % NA]);
                mbar_arrive(&empty_bar[slot]);  // this warp is done with the codes
            }
            if (!ok) break;
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
                sv[m] = sv_next[m];
                bv[m] = bv_next[m];
            }
        }
    }

    // ------------------------------------------------------------ epilogue ---
    // Outputs may be read by the previous kernel in the stream: write them only
    // after it has completed.
    griddep_wait();
    float acc[NMAT][16];
    const bool epi_warp = warp >= 2 && warp < 6;  // one warp per tensor-memory quarter
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;
    if (epi_warp) {
        const bool done = wait_or_abort(&done_bar, 0, &abort_sh);
        tc_fence_after();
        __syncwarp();
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
            tc_ld16(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + 16 * m, acc[m]);
            if (!done)
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[m][i] = 0.f;
        }
    } else if (threadIdx.x == 32 && abort_sh) {
        mbar_wait_bounded(&done_bar, 0);  // MMAs in flight finish before the CTA exits
    }

    float* red = reinterpret_cast<float*>(sgen);  // stages are free: every copy landed and was read
    if (P > 1) {
        __syncthreads();
        if (epi_warp) {
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
                for (int i = 0; i < 16; ++i) red[(rl * NMAT + m) * 16 + i] = acc[m][i];
        }
        cluster_barrier();
        // rank r finishes rows [r * 128 / P, (r + 1) * 128 / P), summing the
        // ranks' partials in rank order
        const int r_lo = static_cast<int>(rank) * kTcRows / P;
        const int r_hi = (static_cast<int>(rank) + 1) * kTcRows / P;
        for (int e = threadIdx.x - 64; e >= 0 && e < (r_hi - r_lo) * 16; e += kThreadsTc - 64) {
            const int r = r_lo + e / 16, tok = e % 16;
            float v[NMAT];
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
                const uint32_t addr = smem_u32(&red[(r * NMAT + m) * 16 + tok]);
                float s = 0.f;
                for (int q = 0; q < P; ++q) s += ld_dsmem(addr, static_cast<uint32_t>(q));
                v[m] = s;
            }
            const int64_t grow = row0 + r;
            if (tok < p.S && grow < p.n) {
                if (EPI == kEpiPlain)
                    p.Y[static_cast<int64_t>(tok) * p.n + grow] = v[0];
                else
                    p.H[static_cast<int64_t>(tok) * p.n + grow] =
                        f2h_rn(v[0] / (1.0f + expf(-v[0])) * v[NMAT - 1]);
            }
        }
        cluster_barrier();  // peers keep their shared memory until it is read
    } else if (epi_warp) {
        const int64_t grow = row0 + rl;
        if (grow < p.n) {
#pragma unroll
            for (int tok = 0; tok < kTcTokens; ++tok) {
                if (tok >= p.S) break;
                if (EPI == kEpiPlain)
                    p.Y[static_cast<int64_t>(tok) * p.n + grow] = acc[0][tok];
                else
                    p.H[static_cast<int64_t>(tok) * p.n + grow] =
                        f2h_rn(acc[0][tok] / (1.0f + expf(-acc[0][tok])) * acc[NMAT - 1][tok]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(L::kTmemCols)
                     : "memory");
    }
}

// ------------------------------------------------------------------ host ---
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D tensor map, 128-byte swizzle: rows of `row_bytes` (elements of
// `elem` bytes), box `box_inner` elements x `box_rows` rows.
qg_status make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem,
                   uint64_t inner, uint64_t rows, uint32_t box_inner, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return QG_ERR_CUDA;
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {inner * static_cast<uint64_t>(elem)};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? QG_OK : QG_ERR_CUDA;
}

template <int FMT, int NMAT, int EPI>
qg_status launch_tc_t(const GemmS16Launch& Lc, const DeviceInfo& dev, cudaStream_t stream) {
    using F = TcFmt<FMT>;
    using L = TcLayout<FMT, NMAT>;
    auto kern = gemm_tc_kernel<FMT, NMAT, EPI>;
    const size_t smem = L::kSmem + 1024;
    if (smem + 2048 > static_cast<size_t>(dev.max_smem_optin)) return QG_ERR_SHAPE;
    static bool attr_done[64] = {false};
    if (dev.device >= 64 || !attr_done[dev.device]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return cuda_status(e);
        if (dev.device < 64) attr_done[dev.device] = true;
    }
    CUtensorMap mc[2], mx;
    const uint64_t row_bytes = FMT == 0 ? static_cast<uint64_t>(Lc.k) : static_cast<uint64_t>(Lc.k) / 2;
    for (int m = 0; m < NMAT; ++m) {
        qg_status st = make_map(&mc[m], Lc.codes[m], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, row_bytes,
                                static_cast<uint64_t>(Lc.n), kCodeBox, kTcRows);
        if (st != QG_OK) return st;
    }
    if (NMAT == 1) mc[1] = mc[0];
    qg_status st = make_map(&mx, Lc.X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                            static_cast<uint64_t>(Lc.k), static_cast<uint64_t>(Lc.S), kXBoxK,
                            kTcTokens);
    if (st != QG_OK) return st;

    TcParams p = {};
    for (int m = 0; m < 2; ++m) {
        const int src = m < NMAT ? m : 0;
        p.scales[m] = Lc.scales[src];
        p.biases[m] = Lc.biases[src];
    }
    p.Y = Lc.Y;
    p.H = Lc.H;
    p.n = Lc.n;
    p.k = Lc.k;
    p.S = Lc.S;
    // Split K over a cluster of P CTAs (1..8, at most one per stage): every SM
    // streams its CTAs' shares of the weight, so the time goes with the most
    // CTAs any SM holds times the share of one, ceil(tiles P / SMs) / P; take
    // the P that minimizes it, the smaller P on ties.
    const int64_t tiles = (Lc.n + kTcRows - 1) / kTcRows;
    const int64_t stages = Lc.k / F::kStageK;
    int P = 1;
    double best = 1e30;
    for (int c = 1; c <= kMaxClusterTc && c <= stages; ++c) {
        const int64_t per_sm = (tiles * c + dev.num_sms - 1) / dev.num_sms;
        const double t = static_cast<double>(per_sm) / c;
        if (t < best - 1e-9) {
            best = t;
            P = c;
        }
    }
    p.splits = P;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles * P));
    cfg.blockDim = dim3(kThreadsTc);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = static_cast<unsigned>(P);
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, mc[0], mc[1], mx, p));
}

}  // namespace

qg_status launch_gemm_tc(const GemmS16Launch& L, cudaStream_t stream) {
    if (L.S < 2 || L.S > kTcTokens) return QG_ERR_SHAPE;
    if (L.k % 512 != 0) return QG_ERR_SHAPE;  // whole stages for every split
    if (L.n > (1LL << 31) - kTcRows) return QG_ERR_SHAPE;
    DeviceInfo dev;
    qg_status st = device_info(&dev);
    if (st != QG_OK) return st;
    const bool swiglu = L.epilogue == kEpiSwiglu;
    if (L.fmt == QG_FMT_I8_B32)
        return swiglu ? launch_tc_t<0, 2, kEpiSwiglu>(L, dev, stream)
                      : launch_tc_t<0, 1, kEpiPlain>(L, dev, stream);
    if (L.fmt == QG_FMT_I4_G64)
        return swiglu ? launch_tc_t<1, 2, kEpiSwiglu>(L, dev, stream)
                      : launch_tc_t<1, 1, kEpiPlain>(L, dev, stream);
    return QG_ERR_FORMAT;
}

unsigned int gemm_tc_read_and_clear_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_err, sizeof v) != cudaSuccess) return 0;
    if (v) cudaMemcpyToSymbol(g_tc_err, &zero, sizeof zero);
    return v;
}

}  // namespace qg
