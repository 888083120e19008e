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
// over a K range; gate/up runs as pair tiles (64 gate rows in tensor-memory
// lanes 0-63, the same 64 rows of up in lanes 64-127), so every call runs with
// the same single-weight resources, two CTAs per SM.  The CTAs of a thread-block
// cluster split K; each pushes its fp32 partials into the shared memory of the
// CTA that finishes those rows, which sums them in rank order after one
// cluster barrier (deterministic, no global workspace).  Warp roles:
//
//  * warp 0 -- producer (warp-uniform loop, the elected lane issues): TMA
//    (cp.async.bulk.tensor.2d, this GPU's memory only, no multicast) copies
//    each stage's code tile (128 rows x 128 bytes, 128-byte swizzle) and the
//    X chunk (16 rows x 64 fp16 per box, rows >= S filled with zeros by the
//    copy) into a ring of shared-memory stages on one mbarrier each.  Codes do
//    not depend on the previous kernel and are requested before
//    griddepcontrol.wait; X after.
//  * warps 2..9 -- dequantize: thread = weight row (its warp's quarter of the
//    tensor-memory lanes); two sets of four warps take alternate A groups of
//    8 steps of 16 k, so one set dequantizes while the other's stores drain.
//    Each thread turns its row's 16 codes of a step into fp16(q s) (int8:
//    byte permute into 1024 + u, exact subtraction, one rounding by the block
//    scale) or fp16(q s + b) (int4: one fused rounding) and stores them into
//    tensor memory (tcgen05.st), where the MMA reads its A operand.
//  * warp 1 -- allocates tensor memory; in a warp-uniform loop its elected
//    lane issues tcgen05.mma kind::f16 (A from tensor memory, B = X from
//    shared memory through a 128-byte-swizzle K-major descriptor, fp32 D in
//    tensor memory, step j into accumulator j mod 4 so that consecutive MMAs
//    never wait on each other) and one tcgen05.commit per A group.
//  * epilogue (warps 2..5): tcgen05.ld of the four accumulators (thread =
//    row, 16 columns = tokens), the split-K reduction, fp32 or SwiGLU fp16
//    store; tensor memory is freed after they signal their reads are done.
//
// Every wait is bounded: a wait that gives up sets the CTA's abort flag and
// the device error flag; the CTA then skips its remaining work, drains its
// own copies and MMAs (bounded), frees its tensor memory and still takes part
// in every cluster barrier, so no peer waits forever.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
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
constexpr int kAcc = 4;            // accumulators per weight matrix: independent MMA chains
constexpr int kGroupSteps = 8;     // 16-k steps per A group (one commit releases a group)
constexpr int kMaxClusterTc = 8;
// Gate/up as pair tiles: one 128-row MMA tile holds 64 gate rows (tensor-memory
// lanes 0-63) and the same 64 rows of up (lanes 64-127), so a SwiGLU call runs
// with single-weight resources (two CTAs per SM, twice the tiles).
constexpr int kEpiPair = 100;
constexpr int kPairRows = kTcRows / 2;

template <int FMT>
struct TcFmt {
    static constexpr int kStageK = FMT == 0 ? 128 : 256;  // k per stage: one 128-byte box row
    static constexpr int kKSteps = kStageK / kKStep;       // 8 or 16
    static constexpr int kXBoxes = kStageK / kXBoxK;       // 2 or 4
    static constexpr int kGroup = FMT == 0 ? 32 : 64;      // k per scale (and bias)
};

template <int FMT, int NMAT, bool SPLIT, bool SK = false>
struct TcLayout {
    using F = TcFmt<FMT>;
    static constexpr int kStageBytes = NMAT * kCodeTileBytes + F::kXBoxes * kXBoxBytes;
    // ring depth: a single-weight CTA keeps two per SM within shared memory,
    // a split gate/up CTA leaves room for the receive buffer; with one A
    // group per stage (int8) the depth is even, so that each of the two
    // dequantizing sets always takes the same slots and waits every phase of
    // their barriers (a parity wait must not skip a phase)
    static constexpr int kStages = (NMAT == 1 || SPLIT) ? 4 : (FMT == 0 ? 6 : 5);
    // split K: the partials the CTAs of the cluster push for the rows this
    // CTA finishes, [source rank][matrix][token][row], ceil(128 / P) rows
    // per rank (P ceil(128 / P) < 128 + P)
    // (pair tiles: [source rank][gate|up][token][pair row], ceil(64 / P) pair rows)
    static constexpr int kRecvBytes =
        !SPLIT ? 0
               : (NMAT == 1 ? 2 * (kPairRows + kMaxClusterTc) * 16 * 4
                            : (kTcRows + kMaxClusterTc) * NMAT * 16 * 4);
    static constexpr int kSmem = kStages * kStageBytes + kRecvBytes;  // + 1 KB alignment slack
    // Two single-weight CTAs fit on an SM (shared memory) and share its 512
    // tensor-memory columns; a gate/up CTA is alone on its SM and takes all.
    static constexpr uint32_t kTmemCols = NMAT == 1 ? 256 : 512;
    // tensor memory: accumulator c of matrix m at columns 16 (m kAcc + c)
    // (stream-K: a second set of them, for the CTA's second tile, at + 16
    // kAcc NMAT); then the A groups, each kGroupSteps x NMAT x 8 columns (16
    // fp16 of K per lane and step)
    static constexpr int kDSetCols = 16 * kAcc * NMAT;
    static constexpr int kDCols = kDSetCols * (SK ? 2 : 1);
    static constexpr int kGroupCols = kGroupSteps * NMAT * 8;
    static constexpr int kAGroups = (static_cast<int>(kTmemCols) - kDCols) / kGroupCols;
    static constexpr int kGroupsPerStage = F::kKSteps / kGroupSteps;  // 1 or 2
    // gate/up CTAs are alone on their SM: twice the dequantizing warps
    static constexpr int kDqWarps = NMAT == 2 ? 16 : 8;
    static constexpr int kThreads = (2 + kDqWarps) * 32;
    static_assert(kAGroups >= 2, "tensor memory holds too few A groups to overlap");
    static_assert(F::kKSteps % kGroupSteps == 0, "stages hold whole A groups");
    static_assert(kGroupsPerStage != 1 || kStages % 2 == 0, "each set keeps its own slots");
    static_assert(kGroupSteps % kAcc == 0, "every accumulator takes the same steps of a group");
    static_assert(kStageBytes % 1024 == 0, "stages keep 1024-byte alignment");
    static_assert(NMAT == 1 || kSmem > 116 * 1024, "a gate/up CTA must be alone on its SM");
    static_assert(NMAT == 2 || kSmem + 2048 <= 113 * 1024, "two single-weight CTAs per SM");
    static_assert(!SK || (SPLIT && NMAT == 1), "stream-K runs pair tiles in clusters");
    static_assert(!SK || kRecvBytes >= kPairRows * 2 * 16 * 4, "one pair tile's partial");
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
// The two halves of a cluster barrier, every thread of every CTA once each.
__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}
// Copy `bytes` (a multiple of 16, both addresses 16-byte aligned) of this
// CTA's shared memory into a peer's (dst and its mbarrier as shared::cluster
// addresses); the bytes complete the peer's mbarrier transaction.
__device__ __forceinline__ void bulk_s2peer(uint32_t dst, uint32_t src, uint32_t bytes,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, "
        "[%3];" ::"r"(dst),
        "r"(src), "r"(bytes), "r"(bar)
        : "memory");
}
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
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
// One lane of a converged warp (the same lane every time): the warp runs the
// loop around an issuing instruction uniformly, so its operands stay
// warp-uniform, and only the elected lane issues.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b32 r;\n\telect.sync r|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(pred));
    return pred != 0;
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
// 16 columns of this warp's 32 lanes, without waiting (tc_wait_ld completes it)
__device__ __forceinline__ void tc_ld16_async(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tc_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
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

template <int FMT, int NMAT, int EPI, bool SPLIT, bool SK = false>
__global__ void __launch_bounds__(TcLayout<FMT, NMAT, SPLIT, SK>::kThreads, NMAT == 1 ? 2 : 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_codes0,
                   const __grid_constant__ CUtensorMap tm_codes1,
                   const __grid_constant__ CUtensorMap tm_x, const TcParams p) {
    using F = TcFmt<FMT>;
    using L = TcLayout<FMT, NMAT, SPLIT, SK>;
    constexpr int NSTG = L::kStages;
    constexpr int NG = L::kAGroups;
    constexpr int GPS = L::kGroupsPerStage;
    constexpr int NDQ = L::kDqWarps;
    constexpr int SUB = NDQ / 4;  // dequantizing warps per tensor-memory lane quarter
    constexpr int SETW = SUB / 2;  // of those, per set (the two sets take alternate A groups)
    // a stage's codes are read by one set (int8: one group per stage) or by both
    constexpr int kEmptyArrivals = (GPS == 1 ? NDQ / 2 : NDQ) + 1;
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[NSTG];   // a stage's codes have landed
    __shared__ __align__(8) uint64_t xfull_bar[NSTG];  // its X chunk has landed
    __shared__ __align__(8) uint64_t empty_bar[NSTG];
    __shared__ __align__(8) uint64_t afull_bar[NG];
    __shared__ __align__(8) uint64_t aempty_bar[NG];
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ __align__(8) uint64_t fin_bar;  // epilogue warps done with tensor memory
    __shared__ __align__(8) uint64_t recv_bar; // split K: the peers' partials have landed
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;

    // stages start on a 1024-byte boundary (the 128-byte swizzle atom)
    const uint32_t sraw = smem_u32(smem_raw);
    const uint32_t sbase = (sraw + 1023u) & ~1023u;
    unsigned char* sgen = smem_raw + (sbase - sraw);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = SPLIT ? p.splits : 1;
    const uint32_t rank = SPLIT ? cluster_ctarank_tc() : 0u;
    constexpr bool PAIR = EPI == kEpiPair;
    static_assert(!PAIR || NMAT == 1, "a pair tile holds both matrices in one MMA tile");
    static_assert(!SK || PAIR, "stream-K runs pair tiles");
    constexpr int kTileRows = PAIR ? kPairRows : kTcRows;  // output rows of a tile
    // This CTA's work: nA stages of tile tA from its stage sA, then (stream-K
    // only) nB stages of tile tA + 1 from its stage 0.  A split CTA takes the
    // stages [rank S / P, (rank + 1) S / P) of its tile's S, as evenly as the
    // stage count allows.  Stream-K: a cluster of P CTAs takes the (P - 1) S
    // stages of its P - 1 tiles in P equal shares, u = [rank (P - 1) S / P,
    // (rank + 1) (P - 1) S / P); with S >= P, rank 0 holds the head of the
    // first tile, rank P - 1 the tail of the last, and every rank r between
    // them the tail of tile r - 1 and the head of tile r.
    const int total_st = static_cast<int>(p.k / F::kStageK);
    int64_t tA;
    int sA, nA, nB = 0;
    if (SK) {
        const int U = (P - 1) * total_st;
        const int u0 = static_cast<int>(rank) * U / P;
        const int u1 = (static_cast<int>(rank) + 1) * U / P;
        const int t_in = u0 / total_st;  // tile of the cluster the share starts in
        const int endA = (t_in + 1) * total_st < u1 ? (t_in + 1) * total_st : u1;
        tA = static_cast<int64_t>(blockIdx.x / P) * (P - 1) + t_in;
        sA = u0 - t_in * total_st;
        nA = endA - u0;
        nB = u1 - endA;
    } else {
        tA = blockIdx.x / P;
        sA = static_cast<int>(rank) * total_st / P;
        nA = (static_cast<int>(rank) + 1) * total_st / P - sA;
    }
    const int64_t row0 = tA * kTileRows;         // first output row of tile tA
    const int64_t row0B = row0 + kTileRows;      // ... of tile tA + 1
    const int64_t kbeg = static_cast<int64_t>(sA) * F::kStageK;
    const int nstages = nA + nB;
    const int ngroups = nstages * GPS;
    const int gB = nA * GPS;  // first A group of tile tA + 1 (== ngroups without one)

    if (threadIdx.x == 0) {
        abort_sh = 0;
        for (int s = 0; s < NSTG; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&xfull_bar[s], 1);
            mbar_init(&empty_bar[s], kEmptyArrivals);
        }
        for (int j = 0; j < NG; ++j) {
            mbar_init(&afull_bar[j], NDQ / 2);
            mbar_init(&aempty_bar[j], 1);
        }
        mbar_init(&done_bar, 1);
        mbar_init(&fin_bar, 4);
        mbar_init(&recv_bar, 1);
        fence_mbar_init();
        prefetch_tmap(&tm_codes0);
        if (NMAT == 2) prefetch_tmap(&tm_codes1);
        prefetch_tmap(&tm_x);
    }
    if (warp == 1) {  // tensor memory for D and the A groups (whole warp)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&tmem_base_sh)),
                     "r"(L::kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // split K: every CTA's receive barrier is initialized before any peer may
    // copy into it (the matching wait comes just before the copies)
    if (SPLIT) cluster_arrive();
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
    // accumulator c of matrix m (of the second set: + kDSetCols); step j of A
    // group g for matrix m
    auto d_col = [](int m, int c) -> uint32_t { return static_cast<uint32_t>(16 * (m * kAcc + c)); };
    auto a_col = [](int g, int j, int m) -> uint32_t {
        return static_cast<uint32_t>(L::kDCols + g * L::kGroupCols + (j * NMAT + m) * 8);
    };

    if (warp == 0) {
        // ------------------------------------------------------- producer ---
        // The whole warp runs the loop and waits; the elected lane issues.
        const uint64_t pol_w = l2_policy_evict_first();
        const uint64_t pol_x = l2_policy_evict_last();
        const int code_bytes_per_k = FMT == 0 ? 1 : 0;  // int8: 1 byte per k; int4: 1/2
        // stage st of this CTA: k offset and first row of its tile
        auto stage_k0 = [&](int st) -> int64_t {
            return static_cast<int64_t>(st < nA ? sA + st : st - nA) * F::kStageK;
        };
        auto code_c0 = [&](int st) -> int {
            const int64_t k0 = stage_k0(st);
            return static_cast<int>(code_bytes_per_k ? k0 : k0 / 2);
        };
        auto issue_codes = [&](int st) {
            const int slot = st % NSTG;
            const int r0 = static_cast<int>(st < nA ? row0 : row0B);
            mbar_arrive_expect_tx(&full_bar[slot], NMAT * kCodeTileBytes);
            tma_load_2d(stage_codes(slot, 0), &tm_codes0, code_c0(st), r0, &full_bar[slot], pol_w);
            if (PAIR)  // up rows below the gate rows (64-row boxes)
                tma_load_2d(stage_codes(slot, 0) + kPairRows * kCodeBox, &tm_codes1, code_c0(st),
                            r0, &full_bar[slot], pol_w);
            if (NMAT == 2)
                tma_load_2d(stage_codes(slot, 1), &tm_codes1, code_c0(st), r0, &full_bar[slot],
                            pol_w);
        };
        auto issue_x = [&](int st) {
            const int slot = st % NSTG;
            const int64_t k0 = stage_k0(st);
            mbar_arrive_expect_tx(&xfull_bar[slot], F::kXBoxes * kXBoxBytes);
#pragma unroll
            for (int b = 0; b < F::kXBoxes; ++b)
                tma_load_2d(stage_x(slot) + b * kXBoxBytes, &tm_x, static_cast<int>(k0 + b * kXBoxK),
                            0, &xfull_bar[slot], pol_x);
        };
        // codes of the first stages before the wait on the previous kernel
        const int pre = nstages < NSTG ? nstages : NSTG;
        if (elect_one())
            for (int st = 0; st < pre; ++st) issue_codes(st);
        __syncwarp();
        griddep_wait();
        if (elect_one())
            for (int st = 0; st < pre; ++st) issue_x(st);
        __syncwarp();
        for (int st = NSTG; st < nstages; ++st) {
            const int slot = st % NSTG;
            if (!warp_wait_or_abort(&empty_bar[slot], ((st / NSTG) - 1) & 1, &abort_sh)) break;
            if (elect_one()) {
                issue_codes(st);
                issue_x(st);
            }
            __syncwarp();
        }
        // drain: every issued copy lands before the CTA may exit (bounded)
        const int first = nstages > NSTG ? nstages - NSTG : 0;
        for (int st = first; st < nstages; ++st) {
            mbar_wait_bounded(&full_bar[st % NSTG], (st / NSTG) & 1);
            mbar_wait_bounded(&xfull_bar[st % NSTG], (st / NSTG) & 1);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA ---
        // One A group (8 steps of 16 k) at a time, issued back to back: step j
        // accumulates into accumulator j % kAcc, so consecutive MMAs do not
        // wait for one another's result; one commit then releases the group.
        // The whole warp runs the loop and waits; the elected lane issues the
        // MMAs and their commits.  Stream-K: the groups of the second tile
        // accumulate into the second set, which they start afresh.
        for (int g = 0; g < ngroups; ++g) {
            const int st = g / GPS, gi = g % GPS;
            const int slot = st % NSTG;
            const int ag = g % NG;
            if (gi == 0 && !warp_wait_or_abort(&xfull_bar[slot], (st / NSTG) & 1, &abort_sh)) break;
            if (!warp_wait_or_abort(&afull_bar[ag], (g / NG) & 1, &abort_sh)) break;
            tc_fence_after();
            const uint32_t dset = g >= gB ? static_cast<uint32_t>(L::kDSetCols) : 0u;
            const bool fresh = g == 0 || g == gB;  // the first group of a tile
            if (elect_one()) {
#pragma unroll
                for (int j = 0; j < kGroupSteps; ++j) {
                    const int kk = gi * kGroupSteps + j;  // 16-k step within the stage
                    const uint64_t bdesc = sw128_kmajor_desc(stage_x(slot) + (kk / 4) * kXBoxBytes +
                                                             (kk % 4) * (kKStep * 2));
#pragma unroll
                    for (int m = 0; m < NMAT; ++m)
                        tc_mma_ts(tmem + dset + d_col(m, j % kAcc), tmem + a_col(ag, j, m), bdesc,
                                  kIdescF16M128N16, (!fresh || j >= kAcc) ? 1u : 0u);
                }
                tc_commit(&aempty_bar[ag]);                     // A group free once read
                if (gi == GPS - 1) tc_commit(&empty_bar[slot]);  // X of this stage read
            }
            __syncwarp();
        }
        if (elect_one()) tc_commit(&done_bar);  // every MMA issued above has completed
        __syncwarp();
    } else {
        // ---------------------------------------------------- dequantize ---
        // Two sets of warps take alternate A groups, so that one set's group
        // is dequantized while the other's stores drain; within a set, the
        // SETW warps of a lane quarter split the group's steps.
        const int dq = warp - 2;              // 0 .. NDQ - 1
        const int quarter = warp & 3;         // tensor-memory lanes 32*quarter .. +31
        const int sub = dq >> 2;              // 0 .. SUB - 1
        const int set = sub / SETW;           // groups g = set (mod 2)
        const int ssub = sub % SETW;          // steps j = ssub (mod SETW) of a group
        const int rl = quarter * 32 + lane;   // row within the tile
        const int64_t grow_raw = PAIR ? row0 + (rl & (kPairRows - 1)) : row0 + rl;
        const int64_t grow = grow_raw < p.n ? grow_raw : p.n - 1;  // tail rows: discard
        const int64_t growB = grow_raw + kTileRows < p.n ? grow_raw + kTileRows : p.n - 1;
        const int msrc = PAIR ? rl / kPairRows : 0;                 // pair tile: gate or up
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const int64_t sides_per_row = p.k / F::kGroup;
        // the row's scales (and biases) from this CTA's first stage of tile tA,
        // and (stream-K) from stage 0 of tile tA + 1
        const uint16_t* srow[NMAT];
        const uint16_t* brow[NMAT];
        const uint16_t* srowB[NMAT];
        const uint16_t* browB[NMAT];
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
            // (a select, not an index: a parameter array indexed at run time
            // would be copied to local memory)
            const uint16_t* sbase = (m + msrc) == 0 ? p.scales[0] : p.scales[1];
            const uint16_t* bbase = (m + msrc) == 0 ? p.biases[0] : p.biases[1];
            srow[m] = sbase + grow * sides_per_row + kbeg / F::kGroup;
            brow[m] = FMT == 1 ? bbase + grow * sides_per_row + kbeg / F::kGroup : nullptr;
            srowB[m] = sbase + growB * sides_per_row;
            browB[m] = FMT == 1 ? bbase + growB * sides_per_row : nullptr;
        }
        // the row's 4 scales (and biases) of a stage: 8 bytes each
        auto load_sides = [&](int st, uint2 (&sv)[NMAT], uint2 (&bv)[NMAT]) {
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
                const bool b = SK && st >= nA;
                const int o = (b ? st - nA : st) * 4;
                sv[m] = __ldg(reinterpret_cast<const uint2*>((b ? srowB[m] : srow[m]) + o));
                if (FMT == 1)
                    bv[m] = __ldg(reinterpret_cast<const uint2*>((b ? browB[m] : brow[m]) + o));
            }
        };
        uint2 sv[NMAT], bv[NMAT], sv_next[NMAT], bv_next[NMAT];
        if (set < ngroups) load_sides(set / GPS, sv, bv);
        const int r7 = rl & 7;
        // every group a warp takes is its only group of that stage (int8: one
        // group per stage; int4: two, one per set)
        for (int g = set; g < ngroups; g += 2) {
            const int st = g / GPS, gi = g % GPS;
            const int slot = st % NSTG;
            const int ag = g % NG;
            if (g + 2 < ngroups) load_sides((g + 2) / GPS, sv_next, bv_next);
            if (!warp_wait_or_abort(&full_bar[slot], (st / NSTG) & 1, &abort_sh)) break;
            if (g >= NG && !warp_wait_or_abort(&aempty_bar[ag], ((g / NG) - 1) & 1, &abort_sh))
                break;
            tc_fence_after();
#pragma unroll
            for (int jj = 0; jj < kGroupSteps / SETW; ++jj) {
                const int j = ssub + jj * SETW;
                const int kk = gi * kGroupSteps + j;  // 16-k step within the stage
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
                        const int q = kk >> 2;  // group of 64 within the stage
                        const uint32_t sw = q < 2 ? sv[m].x : sv[m].y;
                        const uint32_t bw = q < 2 ? bv[m].x : bv[m].y;
                        const uint16_t s = static_cast<uint16_t>((q & 1) ? sw >> 16 : sw & 0xFFFFu);
                        const uint16_t b = static_cast<uint16_t>((q & 1) ? bw >> 16 : bw & 0xFFFFu);
                        dequant16_i4(c, half2_bits(s), half2_bits(b), av);
                    }
                    tc_st8(tmem + lane_addr + a_col(ag, j, m), av);
                }
            }
            // one wait for the group's stores, then the group and the codes
            // are signalled
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&afull_bar[ag]);
                mbar_arrive(&empty_bar[slot]);  // done with the codes
            }
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
    float accB[16];  // stream-K: the second tile's partial (rank 1)
    const bool epi_warp = warp >= 2 && warp < 6;  // one warp per tensor-memory quarter
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;
    if (epi_warp) {
        const bool done = wait_or_abort(&done_bar, 0, &abort_sh);
        tc_fence_after();
        __syncwarp();
        // the kAcc partial sums of each matrix, added in accumulator order
        auto load_acc = [&](uint32_t col0, float (&out)[16]) {
            const uint32_t base = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + col0;
            uint32_t r[kAcc][16];  // every accumulator's load in flight, one wait
#pragma unroll
            for (int c = 0; c < kAcc; ++c) tc_ld16_async(base + d_col(0, c), r[c]);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float v = __uint_as_float(r[0][i]);
#pragma unroll
                for (int c = 1; c < kAcc; ++c) v += __uint_as_float(r[c][i]);
                out[i] = done ? v : 0.f;
            }
        };
#pragma unroll
        for (int m = 0; m < NMAT; ++m) load_acc(d_col(m, 0), acc[m]);
        if (SK && nB > 0) load_acc(static_cast<uint32_t>(L::kDSetCols), accB);
        // this warp's tensor-memory reads are complete (tcgen05.wait::ld)
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&fin_bar);
    }

    if (SK) {
        // Stream-K.  Every rank but the first stages the partial of its first
        // tile as [pair row][gate|up][token] and sends it with one bulk copy
        // into the receive buffer, onto the receive barrier, of rank - 1, which
        // owns that tile; every rank but the last owns the tile of its last
        // stages, adds the partial it receives to its own and stores the tile.
        constexpr int kPartialFloats = kPairRows * 2 * 16;
        float* stage = reinterpret_cast<float*>(sgen);       // the stages are free now
        float* xch = stage + kPartialFloats;                  // the owner's gate/up exchange
        float* recv = reinterpret_cast<float*>(sgen + NSTG * L::kStageBytes);
        const bool sends = rank > 0;
        const bool owns = static_cast<int>(rank) < P - 1;
        const int ri = rl & (kPairRows - 1), vm = rl / kPairRows;
        if (epi_warp && sends) {
            float4* dst = reinterpret_cast<float4*>(stage + (ri * 2 + vm) * 16);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                dst[i] = make_float4(acc[0][4 * i], acc[0][4 * i + 1], acc[0][4 * i + 2],
                                     acc[0][4 * i + 3]);
            // the bulk copy (async proxy) reads what these stores wrote
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        __syncwarp();
        if (warp >= 2)  // warps 2.. : the staged partial is visible to the sending warp
            asm volatile("barrier.sync 2, %0;" ::"r"(L::kThreads - 64) : "memory");
        if (owns && threadIdx.x == 64)
            mbar_arrive_expect_tx(&recv_bar, static_cast<uint32_t>(kPartialFloats * 4));
        cluster_wait();  // every peer's receive barrier is initialized
        if (sends && warp == 2) {
            if (lane == 0) {
                const uint32_t q = rank - 1;
                bulk_s2peer(peer_addr(smem_u32(recv), q), smem_u32(stage),
                            static_cast<uint32_t>(kPartialFloats * 4),
                            peer_addr(smem_u32(&recv_bar), q));
            }
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
        if (owns && epi_warp) {
            if (!mbar_wait_bounded(&recv_bar, 0) && lane == 0) atomicOr(&g_tc_err, kGemvErrTimeout);
            // own partial (of the last stages: the second set when there are
            // two tiles) + the received one, then the pair tile's gate/up
            // exchange as in the whole-tile path below
            const float* own = nB > 0 ? accB : acc[0];
            const int64_t orow0 = nB > 0 ? row0B : row0;
#pragma unroll
            for (int i = 0; i < 16; ++i) xch[i * kTcRows + rl] = own[i] + recv[(ri * 2 + vm) * 16 + i];
            __syncwarp();
            asm volatile("barrier.sync 1, 128;" ::: "memory");
            for (int e = (warp - 2) * 32 + lane; e < kPairRows * 16; e += 128) {
                const int tok = e / kPairRows, r = e % kPairRows;
                const float g = xch[tok * kTcRows + r], u = xch[tok * kTcRows + kPairRows + r];
                const int64_t grow = orow0 + r;
                if (tok < p.S && grow < p.n)
                    p.H[static_cast<int64_t>(tok) * p.n + grow] = f2h_rn(g / (1.0f + expf(-g)) * u);
            }
        }
        // this CTA's copy has read its staged partial before it may exit
        if (sends && warp == 2) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    } else if (SPLIT) {
        // Split K.  Rank q finishes rows [q RT / P, (q + 1) RT / P) of the
        // tile's RT rows (output rows; pair rows for a pair tile, each with
        // the gate and up vectors).  Every CTA stages its partials in its own
        // shared memory as [row][vector][token], then sends each finishing
        // CTA its block with one bulk copy into that CTA's receive buffer
        // ([source rank][row][vector][token]), completing on its receive
        // barrier; each CTA sums its rows' partials in rank order.
        constexpr int RT = PAIR ? kPairRows : kTcRows;
        constexpr int VM = PAIR ? 2 : NMAT;
        constexpr int kRowFloats = VM * 16;
        float* stage = reinterpret_cast<float*>(sgen);  // the stages are free now
        float* recv = reinterpret_cast<float*>(sgen + NSTG * L::kStageBytes);
        auto lo_of = [&](int q) { return q * RT / P; };
        if (epi_warp) {
            const int ri = PAIR ? (rl & (kPairRows - 1)) : rl;
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
                const int vm = PAIR ? rl / kPairRows : m;
                float4* dst = reinterpret_cast<float4*>(stage + (ri * VM + vm) * 16);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_float4(acc[m][4 * i], acc[m][4 * i + 1], acc[m][4 * i + 2],
                                         acc[m][4 * i + 3]);
            }
            // the bulk copies (async proxy) read what these stores wrote
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        __syncwarp();
        if (warp >= 2)  // warps 2.. : every staged row is visible to the senders and reducers
            asm volatile("barrier.sync 2, %0;" ::"r"(L::kThreads - 64) : "memory");
        const int r_lo = lo_of(static_cast<int>(rank));
        const int R = lo_of(static_cast<int>(rank) + 1) - r_lo;
        if (threadIdx.x == 64)
            mbar_arrive_expect_tx(&recv_bar, static_cast<uint32_t>((P - 1) * R * kRowFloats * 4));
        cluster_wait();  // every peer's receive barrier is initialized
        if (warp == 2) {
            if (lane < P && lane != static_cast<int>(rank)) {
                const int q = lane, qlo = lo_of(q), qR = lo_of(q + 1) - qlo;
                const uint32_t src = smem_u32(stage + qlo * kRowFloats);
                const uint32_t dst = peer_addr(
                    smem_u32(recv + static_cast<int>(rank) * qR * kRowFloats), static_cast<uint32_t>(q));
                bulk_s2peer(dst, src, static_cast<uint32_t>(qR * kRowFloats * 4),
                            peer_addr(smem_u32(&recv_bar), static_cast<uint32_t>(q)));
            }
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
        if (threadIdx.x >= 64) {
            if (!mbar_wait_bounded(&recv_bar, 0) && threadIdx.x == 64)
                atomicOr(&g_tc_err, kGemvErrTimeout);
            for (int e = threadIdx.x - 64; e < R * 16; e += L::kThreads - 64) {
                const int r = e / 16, tok = e % 16;  // consecutive threads, consecutive words
                float v[VM];
#pragma unroll
                for (int vm = 0; vm < VM; ++vm) {
                    float sum = 0.f;
                    for (int q = 0; q < P; ++q)
                        sum += q == static_cast<int>(rank)
                                   ? stage[((r_lo + r) * VM + vm) * 16 + tok]
                                   : recv[((q * R + r) * VM + vm) * 16 + tok];
                    v[vm] = sum;
                }
                const int64_t grow = row0 + r_lo + r;
                if (tok < p.S && grow < p.n) {
                    if (EPI == kEpiPlain)
                        p.Y[static_cast<int64_t>(tok) * p.n + grow] = v[0];
                    else
                        p.H[static_cast<int64_t>(tok) * p.n + grow] =
                            f2h_rn(v[0] / (1.0f + expf(-v[0])) * v[VM - 1]);
                }
            }
        }
        // this CTA's copies have read its staged partials before it may exit
        if (warp == 2) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    } else if (PAIR) {
        if (epi_warp) {
            // the four epilogue warps exchange their rows through shared memory
            // (the stages are free: every copy landed and was read): lane r
            // holds gate row r, lane 64 + r the same row of up
            float* xch = reinterpret_cast<float*>(sgen);
#pragma unroll
            for (int i = 0; i < 16; ++i) xch[i * kTcRows + rl] = acc[0][i];
            __syncwarp();
            asm volatile("barrier.sync 1, 128;" ::: "memory");
            for (int e = (warp - 2) * 32 + lane; e < kPairRows * 16; e += 128) {
                const int tok = e / kPairRows, r = e % kPairRows;
                const float g = xch[tok * kTcRows + r], u = xch[tok * kTcRows + kPairRows + r];
                const int64_t grow = row0 + r;
                if (tok < p.S && grow < p.n)
                    p.H[static_cast<int64_t>(tok) * p.n + grow] = f2h_rn(g / (1.0f + expf(-g)) * u);
            }
        }
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
    __syncwarp();
    if (warp == 1) {
        // free tensor memory once no MMA is in flight and the epilogue warps
        // have read their accumulators (bounded waits; the epilogue warps
        // arrive even when the CTA gave up)
        mbar_wait_bounded(&done_bar, 0);
        mbar_wait_bounded(&fin_bar, 0);
        __syncwarp();
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

// Shared memory of the kernel variant, and its attributes set once per device.
template <int FMT, int NMAT, int EPI, bool SPLIT, bool SK = false>
qg_status prepare_tc(const DeviceInfo& dev, size_t* smem_out) {
    using L = TcLayout<FMT, NMAT, SPLIT, SK>;
    auto kern = gemm_tc_kernel<FMT, NMAT, EPI, SPLIT, SK>;
    const size_t smem = L::kSmem + 1024;
    if (smem + 2048 > static_cast<size_t>(dev.max_smem_optin)) return QG_ERR_SHAPE;
    static bool attr_done[64] = {false};
    if (dev.device >= 64 || !attr_done[dev.device]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return cuda_status(e);
        // all of the unified L1 as shared memory: two single-weight CTAs per SM
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return cuda_status(e);
        if (dev.device < 64) attr_done[dev.device] = true;
    }
    *smem_out = smem;
    return QG_OK;
}

// Clusters of P CTAs the device holds at once for this kernel (cached per
// device and P); 0 if the query fails.
template <int FMT, int NMAT, int EPI, bool SPLIT, bool SK = false>
int clusters_per_wave(const DeviceInfo& dev, size_t smem, int P) {
    static int cache[64][kMaxClusterTc + 1] = {{0}};
    if (dev.device < 64 && cache[dev.device][P] != 0) return cache[dev.device][P];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(P * dev.num_sms));
    cfg.blockDim = dim3(TcLayout<FMT, NMAT, SPLIT>::kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(P);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<FMT, NMAT, EPI, SPLIT, SK>, &cfg) !=
        cudaSuccess) {
        cudaGetLastError();  // clear the query's error
        return 0;
    }
    if (dev.device < 64) cache[dev.device][P] = n > 0 ? n : -1;
    return n;
}

// The split P of a launch and the time the model expects for it (us).
template <int FMT, int NMAT, int EPI>
double choose_split(const GemmS16Launch& Lc, const DeviceInfo& dev, size_t smem1, size_t smemP,
                    int* P_out) {
    using F = TcFmt<FMT>;
    // Split K over a cluster of P CTAs (1..8, at most one per stage).  The
    // clusters run in rounds of as many as the GPU holds at once; a round
    // costs the busiest SM's bytes over its rate plus a fixed cost (launch,
    // pipeline fill, epilogue).  Rates and costs were measured on B200 by
    // timing every P on the int8 and int4 projections of 2B-8B decoders: an
    // int8 CTA alone on its SM streams ~29 KB/us, an SM holding two ~54 KB/us
    // (int4, bound by its dequantization, about half of that); fixed cost
    // ~4.4 us, ~4.6 us with the split's bulk-copy reduction.  The occupancy query counts
    // a kernel that allocates tensor memory as one CTA per SM although two
    // single-weight CTAs co-reside, so their capacity is taken as twice the
    // query's, and at least 90% of the slots for clusters of P (GPC packing).
    // Take the P that minimizes rounds x round cost, the smaller P on ties.
    constexpr bool PAIR = EPI == kEpiPair;
    const int64_t tiles = (Lc.n + (PAIR ? kPairRows : kTcRows) - 1) / (PAIR ? kPairRows : kTcRows);
    const int64_t stages = Lc.k / F::kStageK;
    const double bytes_per_k = FMT == 0 ? 1.0625 : 0.5625;
    // a tile streams 128 weight rows per matrix (a pair tile: 64 of each)
    const double tile_kb = kTcRows * static_cast<double>(Lc.k) * bytes_per_k * NMAT / 1e3;
    int P = 1;
    double best = 1e30;
    for (int c = 1; c <= kMaxClusterTc && c <= stages; ++c) {
        int cpw = c == 1 ? clusters_per_wave<FMT, NMAT, EPI, false>(dev, smem1, c)
                         : clusters_per_wave<FMT, NMAT, EPI, true>(dev, smemP, c);
        if (cpw <= 0) continue;
        if (NMAT == 1)
            cpw = std::max(2 * cpw, static_cast<int>(0.9 * 2 * dev.num_sms / c));
        const int64_t rounds = (tiles + cpw - 1) / cpw;
        const int64_t per_round = (tiles + rounds - 1) / rounds;
        const int64_t per_sm = (per_round * c + dev.num_sms - 1) / dev.num_sms;
        const double fmt_rate = FMT == 0 ? 1.0 : 0.5;
        const double rate = fmt_rate * (NMAT == 2 ? 45.0 : (per_sm >= 2 ? 54.0 : 29.0));
        const double fixed_us = c > 1 ? 4.6 : 4.4;
        const double t = static_cast<double>(rounds) *
                         (static_cast<double>(per_sm) * tile_kb / c / rate + fixed_us);
        if (t < best * (1 - 1e-9)) {
            best = t;
            P = c;
        }
    }
    *P_out = P;
    return best;
}

// Stream-K for pair tiles: clusters of C CTAs over C - 1 tiles, each CTA
// (C - 1) / C of a tile, every tile finished by one CTA.  The same model as
// the split: returns the time it expects for the best C (3..8, C - 1 dividing
// the tile count, at least C stages per tile), or infinity if none applies.
template <int FMT>
double stream_k_time(const GemmS16Launch& Lc, const DeviceInfo& dev, size_t smemSK, int* C_out) {
    using F = TcFmt<FMT>;
    const int64_t tiles = (Lc.n + kPairRows - 1) / kPairRows;
    const int64_t stages = Lc.k / F::kStageK;
    const double bytes_per_k = FMT == 0 ? 1.0625 : 0.5625;
    const double tile_kb = kTcRows * static_cast<double>(Lc.k) * bytes_per_k / 1e3;
    double best = 1e30;
    *C_out = 0;
    for (int c = 3; c <= kMaxClusterTc; ++c) {
        if (tiles % (c - 1) != 0 || stages < c) continue;
        int cpw = clusters_per_wave<FMT, 1, kEpiPair, true, true>(dev, smemSK, c);
        if (cpw <= 0) continue;
        cpw = std::max(2 * cpw, static_cast<int>(0.9 * 2 * dev.num_sms / c));
        const int64_t clusters = tiles / (c - 1);
        const int64_t rounds = (clusters + cpw - 1) / cpw;
        const int64_t per_round = (clusters + rounds - 1) / rounds;
        const int64_t per_sm = (per_round * c + dev.num_sms - 1) / dev.num_sms;
        const double rate = (FMT == 0 ? 1.0 : 0.5) * (per_sm >= 2 ? 54.0 : 29.0);
        const double t = static_cast<double>(rounds) *
                         (static_cast<double>(per_sm) * tile_kb * (c - 1) / c / rate + 4.6);
        if (t < best * (1 - 1e-9)) {
            best = t;
            *C_out = c;
        }
    }
    return best;
}

template <int FMT, int NMAT, int EPI>
qg_status prepare_both(const DeviceInfo& dev, size_t* smem1, size_t* smemP) {
    qg_status st = prepare_tc<FMT, NMAT, EPI, false>(dev, smem1);
    if (st != QG_OK) return st;
    return prepare_tc<FMT, NMAT, EPI, true>(dev, smemP);
}

template <int FMT, int NMAT, int EPI>
qg_status launch_tc_t(const GemmS16Launch& Lc, const DeviceInfo& dev, cudaStream_t stream,
                      int P, size_t smem1, size_t smemP, bool sk = false) {
    constexpr bool PAIR = EPI == kEpiPair;
    constexpr int kMats = PAIR ? 2 : NMAT;
    CUtensorMap mc[2], mx;
    const uint64_t row_bytes = FMT == 0 ? static_cast<uint64_t>(Lc.k) : static_cast<uint64_t>(Lc.k) / 2;
    for (int m = 0; m < kMats; ++m) {
        qg_status st = make_map(&mc[m], Lc.codes[m], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, row_bytes,
                                static_cast<uint64_t>(Lc.n), kCodeBox, PAIR ? kPairRows : kTcRows);
        if (st != QG_OK) return st;
    }
    if (kMats == 1) mc[1] = mc[0];
    qg_status st = make_map(&mx, Lc.X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                            static_cast<uint64_t>(Lc.k), static_cast<uint64_t>(Lc.S), kXBoxK,
                            kTcTokens);
    if (st != QG_OK) return st;

    TcParams p = {};
    for (int m = 0; m < 2; ++m) {
        const int src = m < kMats ? m : 0;
        p.scales[m] = Lc.scales[src];
        p.biases[m] = Lc.biases[src];
    }
    p.Y = Lc.Y;
    p.H = Lc.H;
    p.n = Lc.n;
    p.k = Lc.k;
    p.S = Lc.S;
    const int64_t tiles = (Lc.n + (PAIR ? kPairRows : kTcRows) - 1) / (PAIR ? kPairRows : kTcRows);
    p.splits = P;  // stream-K: P CTAs per P - 1 tiles (smemP is the stream-K kernel's)

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(sk ? tiles / (P - 1) * P : tiles * P));
    cfg.blockDim = dim3(TcLayout<FMT, NMAT, false>::kThreads);
    cfg.dynamicSmemBytes = P > 1 ? smemP : smem1;
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
    if (PAIR && sk)
        return cuda_status(cudaLaunchKernelEx(&cfg, gemm_tc_kernel<FMT, NMAT, EPI, true, PAIR>,
                                              mc[0], mc[1], mx, p));
    if (P > 1)
        return cuda_status(cudaLaunchKernelEx(&cfg, gemm_tc_kernel<FMT, NMAT, EPI, true>, mc[0],
                                              mc[1], mx, p));
    return cuda_status(cudaLaunchKernelEx(&cfg, gemm_tc_kernel<FMT, NMAT, EPI, false>, mc[0],
                                          mc[1], mx, p));
}

// One S <= 16 call, with the split from the model.  Gate/up runs as pair
// tiles: on every shape of the 2B-27B decoders (and the test shapes) the model
// expects them to finish before two-matrix tiles of 128 rows (one CTA per SM
// by its 512 tensor-memory columns), and on the 8B gate/up they measured 24.4
// against 27.2 us.
template <int FMT>
qg_status launch_fmt(const GemmS16Launch& L, const DeviceInfo& dev, cudaStream_t stream) {
    size_t s1 = 0, sP = 0;
    int P = 1;
    if (L.epilogue != kEpiSwiglu) {
        qg_status st = prepare_both<FMT, 1, kEpiPlain>(dev, &s1, &sP);
        if (st != QG_OK) return st;
        choose_split<FMT, 1, kEpiPlain>(L, dev, s1, sP, &P);
        return launch_tc_t<FMT, 1, kEpiPlain>(L, dev, stream, P, s1, sP);
    }
    qg_status st = prepare_both<FMT, 1, kEpiPair>(dev, &s1, &sP);
    if (st != QG_OK) return st;
    const double t_split = choose_split<FMT, 1, kEpiPair>(L, dev, s1, sP, &P);
    size_t sSK = 0;
    st = prepare_tc<FMT, 1, kEpiPair, true, true>(dev, &sSK);
    if (st != QG_OK) return st;
    int C = 0;
    if (stream_k_time<FMT>(L, dev, sSK, &C) < t_split)
        return launch_tc_t<FMT, 1, kEpiPair>(L, dev, stream, C, s1, sSK, true);
    return launch_tc_t<FMT, 1, kEpiPair>(L, dev, stream, P, s1, sP);
}

}  // namespace

qg_status launch_gemm_tc(const GemmS16Launch& L, cudaStream_t stream) {
    if (L.S < 2 || L.S > kTcTokens) return QG_ERR_SHAPE;
    if (L.k % 512 != 0) return QG_ERR_SHAPE;  // whole stages for every split
    if (L.n > (1LL << 31) - kTcRows) return QG_ERR_SHAPE;
    DeviceInfo dev;
    qg_status st = device_info(&dev);
    if (st != QG_OK) return st;
    if (L.fmt == QG_FMT_I8_B32) return launch_fmt<0>(L, dev, stream);
    if (L.fmt == QG_FMT_I4_G64) return launch_fmt<1>(L, dev, stream);
    return QG_ERR_FORMAT;
}

unsigned int gemm_tc_read_and_clear_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_err, sizeof v) != cudaSuccess) return 0;
    if (v) cudaMemcpyToSymbol(g_tc_err, &zero, sizeof zero);
    return v;
}

}  // namespace qg
