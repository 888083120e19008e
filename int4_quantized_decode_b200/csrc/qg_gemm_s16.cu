// qg_gemm_s16.cu -- chunked prefill: S <= 16 tokens through int8 block-32
// weights on the tensor cores ("Qwen3.8-27B ... -- Core AI", The vision
// path: a static S=16 'prefill' function next to the S=1 decode step).
//
//   Y[s, r] = sum_k X[s, k] w_dq[r, k]    (plain, fp32 out)
//   H[s, r] = fp16( silu(g) u )           (fused gate/up SwiGLU)
//
// The contraction is dense (16 tokens share every weight), so it runs on the
// tensor cores; it stays bound by the weight stream (32 flop per 1.06 B).
//
//  * A CTA owns a 64-row tile (per weight) and a K range; the CTAs of a
//    thread-block cluster split K and reduce their fp32 partials through
//    distributed shared memory in a fixed order (deterministic, no global
//    workspace, no atomics).  The split is chosen so the grid covers the SMs.
//  * Four warps, each owning 16 rows (plus the matching 16 rows of the up
//    projection for SwiGLU).  Every lane copies the bytes its A fragments need
//    -- 16 consecutive codes of rows g and g+8 per 64-k chunk -- with cp.async
//    into its own shared-memory ring, RING-1 chunks ahead.  The mma's k index is permuted within every 64-k chunk so
//    that those 16 bytes are exactly the lane's fragment slots; the B (X)
//    fragments use the same permutation.  No cross-lane synchronization is
//    needed for A.
//  * X streams through two shared-memory panels of 512 k (16 token rows,
//    pitch padded by 16 B so every 8-lane phase of a 16-byte read hits
//    distinct banks), together with the panel's scales for the tile's rows
//    (each 16-byte piece copied by one thread: copies of one source by many
//    lanes serialize in shared memory); panel p+1 is copied while panel p is
//    used, in the same per-thread cp.async groups as A.
//  * Codes become fp16 in registers (byte permute into the mantissa of 1024,
//    subtract 1152, multiply by the block scale: one fp16 rounding of q*s),
//    then mma.sync m16n8k16 (f16 x f16 -> f32).
//  * The first A chunks are copied before griddepcontrol.wait (programmatic
//    dependent launch); X, produced by the previous kernel, after it.
#include "qg_device.cuh"
#include "qg_internal.h"

namespace qg {

QG_DEFINE_ERROR_FLAG(g_s16_err);

namespace {

constexpr int kWarpsS16 = 4;
constexpr int kThreadsS16 = kWarpsS16 * 32;
constexpr int kTileRows = kWarpsS16 * 16;
constexpr int kChunk = 64;                    // k per ring slot (one lane: 16 codes of 2 rows)
constexpr int kPanel = 512;                   // k per X panel
constexpr int kChunksPerPanel = kPanel / kChunk;
constexpr int kXPitch = kPanel * 2 + 16;      // bytes per token row of an X panel
constexpr int kXPanelBytes = 16 * kXPitch;
constexpr int kMaxCluster = 8;

// Scales of one X panel for the tile's rows: 16 fp16 per row, row pitch
// padded to 48 B so the 8 rows of a lane phase hit distinct banks.
constexpr int kSPitch = 48;

template <int NMAT>
struct S16Layout {
    static constexpr int kRing = NMAT == 1 ? 8 : 6;
    // per warp, per slot, per matrix, per row-half (g / g+8): 32 lanes x 16 B of codes
    static constexpr int kSlotRow = 32 * 16;
    static constexpr int kSlot = NMAT * 2 * kSlotRow;
    static constexpr int kRingBytes = kWarpsS16 * kRing * kSlot;
    static constexpr int kScalePanel = NMAT * kTileRows * kSPitch;
    static constexpr int kRed = kThreadsS16 * NMAT * 8 * 4;
    static constexpr int kSmem = kRingBytes + 2 * kXPanelBytes + 2 * kScalePanel + kRed;
};

struct S16Params {
    const int8_t* codes[2];
    const uint16_t* scales[2];
    const uint16_t* X;
    float* Y;
    uint16_t* H;
    int64_t n, k;
    int S;
    int splits;  // CTAs per cluster along K
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t local_addr, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint64_t pol) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst),
                 "l"(src), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp_async16_keep(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
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

// 4 int8 codes (one word) of one row -> two fp16x2 A-fragment registers
// holding q*s (one fp16 rounding).
__device__ __forceinline__ void dequant4(uint32_t word, __half2 s2, uint32_t& lo, uint32_t& hi) {
    const uint32_t u = word ^ 0x80808080u;  // q + 128 per byte
    const __half2 bias = __half2half2(__ushort_as_half(0x6480));  // 1152
    const uint32_t hl = __byte_perm(u, 0x64646464u, 0x4140);      // 1024 + u0, 1024 + u1
    const uint32_t hh = __byte_perm(u, 0x64646464u, 0x4342);      // 1024 + u2, 1024 + u3
    __half2 ql = __hsub2(*reinterpret_cast<const __half2*>(&hl), bias);
    __half2 qh = __hsub2(*reinterpret_cast<const __half2*>(&hh), bias);
    ql = __hmul2(ql, s2);
    qh = __hmul2(qh, s2);
    lo = *reinterpret_cast<uint32_t*>(&ql);
    hi = *reinterpret_cast<uint32_t*>(&qh);
}

__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int EPI>
__global__ void __launch_bounds__(kThreadsS16, 2) gemm_s16_kernel(const S16Params p) {
    constexpr int NMAT = EPI == kEpiSwiglu ? 2 : 1;
    using L = S16Layout<NMAT>;
    constexpr int RING = L::kRing;
    extern __shared__ __align__(128) unsigned char smem[];
    const uint32_t sbase = smem_u32(smem);
    const uint32_t xpanel0 = sbase + L::kRingBytes;
    const uint32_t spanel0 = xpanel0 + 2 * kXPanelBytes;
    float* red = reinterpret_cast<float*>(smem + L::kRingBytes + 2 * kXPanelBytes +
                                          2 * L::kScalePanel);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;
    const int P = p.splits;
    const uint32_t rank = P > 1 ? cluster_ctarank() : 0u;
    const int64_t tile = blockIdx.x / P;
    const int64_t N = p.n, K = p.k;
    const int kc = static_cast<int>(K / P);  // this CTA's K range (multiple of kPanel)
    const int64_t kbeg = static_cast<int64_t>(rank) * kc;
    const int nch = kc / kChunk;
    const uint64_t pol = l2_policy_evict_first();

    // Zero both X panels once: token rows >= S are never copied.
    for (int i = threadIdx.x; i < 2 * kXPanelBytes / 16; i += kThreadsS16)
        reinterpret_cast<uint4*>(smem + L::kRingBytes)[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();

    // ---- A copies: rows g and g+8 of this warp's 16 rows, 16 codes at
    // 16*tq within each 64-k chunk.
    const int64_t rowA = tile * kTileRows + warp * 16 + g;
    const int64_t r_lo = rowA < N ? rowA : N - 1;          // tail rows: copy, discard
    const int64_t r_hi = rowA + 8 < N ? rowA + 8 : N - 1;
    const int8_t* ca[NMAT][2];
#pragma unroll
    for (int m = 0; m < NMAT; ++m) {
        const int8_t* cm = m == 0 ? p.codes[0] : p.codes[1];
        ca[m][0] = cm + r_lo * K + kbeg + 16 * tq;
        ca[m][1] = cm + r_hi * K + kbeg + 16 * tq;
    }
    const uint32_t ring = sbase + warp * RING * L::kSlot;
    auto slot_codes = [&](int s, int m, int h) -> uint32_t {
        return ring + s * L::kSlot + (m * 2 + h) * L::kSlotRow + lane * 16;
    };
    auto issue_a = [&](int c) {  // chunk c of this CTA's K range into slot c % RING
        const int s = c % RING;
#pragma unroll
        for (int m = 0; m < NMAT; ++m)
#pragma unroll
            for (int h = 0; h < 2; ++h) cp_async16(slot_codes(s, m, h), ca[m][h] + c * kChunk, pol);
    };
    // Panel q -> buffers q & 1: X (16 token rows x 1024 bytes) and the 16
    // scales of every tile row (two 16-byte pieces per row); every piece is
    // copied by exactly one thread.
    auto issue_x = [&](int q) {
        const uint32_t buf = xpanel0 + (q & 1) * kXPanelBytes;
        for (int i = threadIdx.x; i < 16 * (kPanel * 2 / 16); i += kThreadsS16) {
            const int tok = i / (kPanel * 2 / 16), v = i % (kPanel * 2 / 16);
            if (tok < p.S)
                cp_async16_keep(buf + tok * kXPitch + v * 16,
                                p.X + static_cast<int64_t>(tok) * K + kbeg + q * kPanel + v * 8);
        }
        const uint32_t sbuf = spanel0 + (q & 1) * L::kScalePanel;
        for (int i = threadIdx.x; i < NMAT * kTileRows * 2; i += kThreadsS16) {
            const int m = i / (kTileRows * 2), rr = (i / 2) % kTileRows, piece = i & 1;
            const int64_t r0 = tile * kTileRows + rr;
            const int64_t r = r0 < N ? r0 : N - 1;
            const uint16_t* sm = m == 0 ? p.scales[0] : p.scales[1];
            cp_async16_keep(sbuf + (m * kTileRows + rr) * kSPitch + piece * 16,
                            sm + r * (K / 32) + (kbeg + q * kPanel) / 32 + piece * 8);
        }
    };

    // 1) prologue: A chunks 0..RING-2 (independent of the previous kernel)
#pragma unroll
    for (int c = 0; c < RING - 1; ++c) {
        if (c < nch) issue_a(c);
        cp_async_commit();
    }
    // 2) X depends on the previous kernel
    griddep_wait();
    issue_x(0);
    if (kc > kPanel) issue_x(1);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    griddep_launch_dependents();

    float acc[NMAT][2][4];
#pragma unroll
    for (int m = 0; m < NMAT; ++m)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[m][nt][e] = 0.f;
    const int rl = warp * 16 + g;  // this lane's row g inside the tile

    for (int c = 0; c < nch; ++c) {
        const int q = c / kChunksPerPanel;
        if (c % kChunksPerPanel == 0 && c > 0) {
            // panel q was copied during panel q-1 (issued kChunksPerPanel
            // groups ago); make every thread's copies visible, then start the
            // copy of panel q+1 into the buffer panel q-1 used.
            cp_async_wait<RING - 1>();
            __syncthreads();
        }
        if (c + RING - 1 < nch) issue_a(c + RING - 1);
        if (c % kChunksPerPanel == 0 && c > 0 && (q + 1) * kPanel < kc) issue_x(q + 1);
        cp_async_commit();
        cp_async_wait<RING - 1>();

        // B fragments: tokens g and g + 8, halves 16 tq .. 16 tq + 15 of the chunk
        const uint32_t xb = xpanel0 + (q & 1) * kXPanelBytes + g * kXPitch +
                            ((c % kChunksPerPanel) * kChunk + 16 * tq) * 2;
        const uint4 x0a = lds128(xb), x0b = lds128(xb + 16);
        const uint4 x1a = lds128(xb + 8 * kXPitch), x1b = lds128(xb + 8 * kXPitch + 16);
        const uint32_t bx0[8] = {x0a.x, x0a.y, x0a.z, x0a.w, x0b.x, x0b.y, x0b.z, x0b.w};
        const uint32_t bx1[8] = {x1a.x, x1a.y, x1a.z, x1a.w, x1b.x, x1b.y, x1b.z, x1b.w};
        const int s = c % RING;
        // block of this lane's 16 codes inside the panel: 2 per chunk
        const uint32_t sb = spanel0 + (q & 1) * L::kScalePanel +
                            ((c % kChunksPerPanel) * 2 + (tq >> 1)) * 2;
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
            const uint4 cg = lds128(slot_codes(s, m, 0));
            const uint4 cg8 = lds128(slot_codes(s, m, 1));
            const __half2 s0 = __half2half2(__ushort_as_half(
                lds16(sb + (m * kTileRows + rl) * kSPitch)));
            const __half2 s8 = __half2half2(__ushort_as_half(
                lds16(sb + (m * kTileRows + rl + 8) * kSPitch)));
            const uint32_t wg[4] = {cg.x, cg.y, cg.z, cg.w};
            const uint32_t wg8[4] = {cg8.x, cg8.y, cg8.z, cg8.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t a[4];
                dequant4(wg[j], s0, a[0], a[2]);
                dequant4(wg8[j], s8, a[1], a[3]);
                mma16816(acc[m][0], a, bx0[2 * j], bx0[2 * j + 1]);
                mma16816(acc[m][1], a, bx1[2 * j], bx1[2 * j + 1]);
            }
        }
    }
    cp_async_wait<0>();

    // ------------------------------------------- split-K reduction (DSMEM) ---
    float* my_red = red + threadIdx.x * NMAT * 8;
    if (P > 1) {
#pragma unroll
        for (int m = 0; m < NMAT; ++m)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) my_red[(m * 2 + nt) * 4 + e] = acc[m][nt][e];
        cluster_sync_all();
        if (rank == 0) {
            const uint32_t base = smem_u32(my_red);
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int idx = (m * 2 + nt) * 4 + e;
                        float v = my_red[idx];
                        for (int r = 1; r < P; ++r) v += ld_dsmem_f32(base + idx * 4, r);
                        acc[m][nt][e] = v;
                    }
        }
        cluster_sync_all();  // peers keep their shared memory until it is read
    }

    // --------------------------------------------------------------- epilogue
    if (rank == 0) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int s = nt * 8 + 2 * tq + (e & 1);
                const int64_t r = rowA + (e >= 2 ? 8 : 0);
                if (s < p.S && r < N) {
                    if (EPI == kEpiPlain) {
                        p.Y[static_cast<int64_t>(s) * N + r] = acc[0][nt][e];
                    } else {
                        const float gv = acc[0][nt][e];
                        const float uv = acc[NMAT - 1][nt][e];
                        p.H[static_cast<int64_t>(s) * N + r] = f2h_rn(gv / (1.0f + expf(-gv)) * uv);
                    }
                }
            }
    }
}

template <int EPI>
qg_status launch_s16_t(const S16Params& p0, const DeviceInfo& dev, cudaStream_t stream) {
    constexpr int NMAT = EPI == kEpiSwiglu ? 2 : 1;
    using L = S16Layout<NMAT>;
    auto kern = gemm_s16_kernel<EPI>;
    if (L::kSmem + 1024 > dev.max_smem_optin) return QG_ERR_SHAPE;
    static int attr_done[64] = {0};
    if (dev.device >= 64 || !attr_done[dev.device]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
        if (e != cudaSuccess) return cuda_status(e);
        if (dev.device < 64) attr_done[dev.device] = 1;
    }
    S16Params p = p0;
    const int64_t tiles = (p.n + kTileRows - 1) / kTileRows;
    // Split K across a cluster of P CTAs (a power of two that keeps each CTA's
    // range a whole number of X panels), choosing the P whose grid fills the
    // two-CTAs-per-SM waves best; ties go to the smaller P.
    const int64_t slots = 2LL * dev.num_sms;
    int P = 1;
    double best = -1.0;
    for (int c = 1; c <= kMaxCluster; c *= 2) {
        if (p.k % (static_cast<int64_t>(c) * kPanel) != 0) break;
        const int64_t ctas = tiles * c;
        const double eff = static_cast<double>(ctas) / (((ctas + slots - 1) / slots) * slots);
        if (eff > best + 1e-9) {
            best = eff;
            P = c;
        }
    }
    p.splits = P;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles * P));
    cfg.blockDim = dim3(kThreadsS16);
    cfg.dynamicSmemBytes = L::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (P > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = P;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, p));
}

}  // namespace

qg_status launch_gemm_s16(const GemmS16Launch& L, cudaStream_t stream) {
    // Every CTA's K range is a whole number of 512-k X panels.
    if (L.k % kPanel != 0) return QG_ERR_SHAPE;
    DeviceInfo dev;
    qg_status st = device_info(&dev);
    if (st != QG_OK) return st;
    S16Params p = {};
    p.codes[0] = L.codes[0];
    p.codes[1] = L.codes[1];
    p.scales[0] = L.scales[0];
    p.scales[1] = L.scales[1];
    p.X = L.X;
    p.Y = L.Y;
    p.H = L.H;
    p.n = L.n;
    p.k = L.k;
    p.S = L.S;
    if (L.epilogue == kEpiSwiglu) return launch_s16_t<kEpiSwiglu>(p, dev, stream);
    return launch_s16_t<kEpiPlain>(p, dev, stream);
}

unsigned int gemm_s16_read_and_clear_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_s16_err, sizeof v) != cudaSuccess) return 0;
    if (v) cudaMemcpyToSymbol(g_s16_err, &zero, sizeof zero);
    return v;
}

}  // namespace qg
