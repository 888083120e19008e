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
// Layout of the work:
//  * A CTA owns a 64-row tile (per weight) and a contiguous range of K; the
//    CTAs of a thread-block cluster split K and reduce their fp32 partials
//    through distributed shared memory in a fixed order (deterministic, no
//    global workspace, no atomics).
//  * One producer warp streams stages of 256 k through a 1-D bulk-copy ring
//    (no multicast): the X chunk [16 x 256] fp16 shared by all rows, and per
//    row 256 code bytes + 8 fp16 scales.  The code prologue is issued before
//    griddepcontrol.wait (programmatic dependent launch); X, produced by the
//    previous kernel, after it.
//  * Four consumer warps each own 16 rows (and the matching 16 rows of the
//    up projection for SwiGLU).  Each lane reads 16 consecutive codes of a
//    row; the mma's k index is permuted within every 64-k chunk so that those
//    bytes are exactly the lane's A-fragment slots, and the B (X) fragments
//    use the same permutation.  Codes become fp16 in registers (byte permute
//    into the mantissa of 1024, subtract 1152, multiply by the block scale:
//    one fp16 rounding of q*s), then mma.sync m16n8k16 (f16 x f16 -> f32).
//  * Row pitches are padded by 16 B so every 16-byte shared load of a warp
//    phase hits distinct banks.
#include "qg_device.cuh"
#include "qg_internal.h"

namespace qg {

QG_DEFINE_ERROR_FLAG(g_s16_err);

namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kKC = 256;                   // k per stage
constexpr int kTileRows = kConsumerWarps * 16;
constexpr int kXPitch = kKC * 2 + 16;      // bytes per token row of X
constexpr int kCPitch = kKC + 16;          // bytes per weight row of codes
constexpr int kSPitch = kKC / 32 * 2;      // bytes per weight row of scales (16)
constexpr int kMaxCluster = 8;

template <int NMAT>
struct S16Layout {
    static constexpr int kRows = kTileRows * NMAT;
    static constexpr int kX = 16 * kXPitch;
    static constexpr int kCodes = kRows * kCPitch;
    static constexpr int kScales = kRows * kSPitch;
    static constexpr int kStage = kX + kCodes + kScales;
    static constexpr int kStages = NMAT == 1 ? 4 : 2;
    static constexpr int kBars = 128;  // full[kStages] + empty[kStages], padded
    static constexpr int kRed = kConsumerWarps * 32 * NMAT * 8 * 4;
    static constexpr int kSmem = kBars + kStages * kStage + kRed;
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
__global__ void __launch_bounds__(kThreads, 1) gemm_s16_kernel(const S16Params p) {
    constexpr int NMAT = EPI == kEpiSwiglu ? 2 : 1;
    using L = S16Layout<NMAT>;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + L::kStages;
    unsigned char* stages = smem + L::kBars;
    float* red = reinterpret_cast<float*>(stages + L::kStages * L::kStage);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = p.splits;
    const uint32_t rank = P > 1 ? cluster_ctarank() : 0u;
    const int64_t tile = blockIdx.x / P;
    const int64_t row0 = tile * kTileRows;
    const int64_t N = p.n, K = p.k;
    const int nst_all = static_cast<int>(K / kKC + (K % kKC ? 1 : 0));
    const int sb = static_cast<int>((static_cast<int64_t>(nst_all) * rank) / P);
    const int se = static_cast<int>((static_cast<int64_t>(nst_all) * (rank + 1)) / P);
    const int nst = se - sb;
    const int rows_valid = static_cast<int>(N - row0 < kTileRows ? N - row0 : kTileRows);

    // Zero the ring (token rows >= S and rows >= N are never copied), set up
    // the barriers, and order both before the first bulk copy.
    for (int i = threadIdx.x; i < L::kStages * L::kStage / 16; i += kThreads)
        reinterpret_cast<uint4*>(stages)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (threadIdx.x == 0) {
        for (int s = 0; s < L::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_mbar_init();
    }
    fence_proxy_async_smem();
    __syncthreads();

    bool failed = false;
    __shared__ int s_failed;
    __shared__ int s_issued;  // stages the producer has issued
    if (threadIdx.x == 0) {
        s_failed = 0;
        s_issued = 0;
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------ producer ---
        const uint64_t pol = l2_policy_evict_first();
        const uint64_t pol_x = l2_policy_evict_last();
        auto stage_tx = [&](int st) -> uint32_t {
            const int64_t k0 = static_cast<int64_t>(st) * kKC;
            const int kc = static_cast<int>(K - k0 < kKC ? K - k0 : kKC);
            return static_cast<uint32_t>(p.S) * kc * 2u +
                   static_cast<uint32_t>(NMAT * rows_valid) * (kc + kc / 16);
        };
        auto issue_weights = [&](int t) {
            const int st = sb + t;
            const int64_t k0 = static_cast<int64_t>(st) * kKC;
            const int kc = static_cast<int>(K - k0 < kKC ? K - k0 : kKC);
            unsigned char* stg = stages + (t % L::kStages) * L::kStage;
            uint64_t* bar = &full[t % L::kStages];
            for (int i = lane; i < NMAT * rows_valid; i += 32) {
                const int m = i / rows_valid, j = i - m * rows_valid;
                const int64_t r = row0 + j;
                const int srow = m * kTileRows + j;
                // select (not index) the weight: a runtime index into the
                // parameter arrays would move them to local memory
                const int8_t* cm = m == 0 ? p.codes[0] : p.codes[1];
                const uint16_t* sm = m == 0 ? p.scales[0] : p.scales[1];
                bulk_g2s(stg + L::kX + srow * kCPitch, cm + r * K + k0, static_cast<uint32_t>(kc),
                         bar, pol);
                bulk_g2s(stg + L::kX + L::kCodes + srow * kSPitch, sm + r * (K / 32) + k0 / 32,
                         static_cast<uint32_t>(kc / 16), bar, pol);
            }
        };
        auto issue_x = [&](int t) {
            const int st = sb + t;
            const int64_t k0 = static_cast<int64_t>(st) * kKC;
            const int kc = static_cast<int>(K - k0 < kKC ? K - k0 : kKC);
            unsigned char* stg = stages + (t % L::kStages) * L::kStage;
            if (lane < p.S)
                bulk_g2s(stg + lane * kXPitch, p.X + lane * K + k0, static_cast<uint32_t>(kc * 2),
                         &full[t % L::kStages], pol_x);
        };
        const int pre = nst < L::kStages ? nst : L::kStages;
        for (int t = 0; t < pre; ++t) {
            if (lane == 0) mbar_arrive_expect_tx(&full[t], stage_tx(sb + t));
            __syncwarp();
            issue_weights(t);
        }
        griddep_wait();
        for (int t = 0; t < pre; ++t) issue_x(t);
        int issued = pre;
        for (int t = L::kStages; t < nst && !failed; ++t) {
            const uint32_t par = static_cast<uint32_t>(((t / L::kStages) - 1) & 1);
            const bool ok = mbar_wait_bounded(&empty[t % L::kStages], par);
            if (!__all_sync(0xffffffffu, ok)) {
                failed = true;
                break;
            }
            if (lane == 0) mbar_arrive_expect_tx(&full[t % L::kStages], stage_tx(sb + t));
            __syncwarp();
            issue_weights(t);
            issue_x(t);
            issued = t + 1;
        }
        if (lane == 0) s_issued = issued;
        if (failed && lane == 0) {
            atomicOr(&g_s16_err, 1u);
            atomicExch(&s_failed, 1);
        }
    } else {
        griddep_wait();
    }
    griddep_launch_dependents();

    // ------------------------------------------------------------ consumers ---
    const int g = lane >> 2, tq = lane & 3;
    float acc[NMAT][2][4];
#pragma unroll
    for (int m = 0; m < NMAT; ++m)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[m][nt][e] = 0.f;

    int consumed = 0;
    if (warp < kConsumerWarps) {
        for (int t = 0; t < nst; ++t) {
            const int slot = t % L::kStages;
            const bool ok = mbar_wait_bounded(&full[slot], static_cast<uint32_t>((t / L::kStages) & 1));
            if (!__all_sync(0xffffffffu, ok)) {
                failed = true;
                break;
            }
            const unsigned char* stg = stages + slot * L::kStage;
            const int64_t k0 = static_cast<int64_t>(sb + t) * kKC;
            const int kc = static_cast<int>(K - k0 < kKC ? K - k0 : kKC);
            for (int sc = 0; sc < kc / 64; ++sc) {
                // B fragments: tokens g and g + 8, halves 16 tq .. 16 tq + 15 of
                // this 64-k chunk.
                const unsigned char* xg = stg + g * kXPitch + (64 * sc + 16 * tq) * 2;
                const uint4 x0a = *reinterpret_cast<const uint4*>(xg);
                const uint4 x0b = *reinterpret_cast<const uint4*>(xg + 16);
                const uint4 x1a = *reinterpret_cast<const uint4*>(xg + 8 * kXPitch);
                const uint4 x1b = *reinterpret_cast<const uint4*>(xg + 8 * kXPitch + 16);
                const uint32_t bx0[8] = {x0a.x, x0a.y, x0a.z, x0a.w, x0b.x, x0b.y, x0b.z, x0b.w};
                const uint32_t bx1[8] = {x1a.x, x1a.y, x1a.z, x1a.w, x1b.x, x1b.y, x1b.z, x1b.w};
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    const int srow = m * kTileRows + warp * 16 + g;
                    const unsigned char* cr = stg + L::kX + srow * kCPitch + 64 * sc + 16 * tq;
                    const uint4 cg = *reinterpret_cast<const uint4*>(cr);
                    const uint4 cg8 = *reinterpret_cast<const uint4*>(cr + 8 * kCPitch);
                    const unsigned char* sr = stg + L::kX + L::kCodes + srow * kSPitch +
                                              (2 * sc + (tq >> 1)) * 2;
                    const __half2 s0 = __half2half2(*reinterpret_cast<const __half*>(sr));
                    const __half2 s8 = __half2half2(*reinterpret_cast<const __half*>(sr + 8 * kSPitch));
                    const uint32_t wg[4] = {cg.x, cg.y, cg.z, cg.w};
                    const uint32_t wg8[4] = {cg8.x, cg8.y, cg8.z, cg8.w};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t a[4];
                        dequant4(wg[c], s0, a[0], a[2]);
                        dequant4(wg8[c], s8, a[1], a[3]);
                        mma16816(acc[m][0], a, bx0[2 * c], bx0[2 * c + 1]);
                        mma16816(acc[m][1], a, bx1[2 * c], bx1[2 * c + 1]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
            ++consumed;
        }
        if (failed && lane == 0) {
            atomicOr(&g_s16_err, 1u);
            atomicExch(&s_failed, 1);
        }
    }
    __syncthreads();
    if (s_failed && threadIdx.x == 0) {
        // Drain copies still in flight (bounded) before the CTA can exit: the
        // latest use of every slot is among the last kStages issued stages.
        const int first = s_issued > L::kStages ? s_issued - L::kStages : 0;
        for (int t = first; t < s_issued; ++t)
            mbar_wait_bounded(&full[t % L::kStages], static_cast<uint32_t>((t / L::kStages) & 1));
    }

    // ------------------------------------------- split-K reduction (DSMEM) ---
    float* my_red = red + (static_cast<int>(threadIdx.x) * NMAT * 8);
    if (P > 1) {
        if (warp < kConsumerWarps) {
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) my_red[(m * 2 + nt) * 4 + e] = acc[m][nt][e];
        }
        cluster_sync_all();
        if (rank == 0 && warp < kConsumerWarps) {
            const uint32_t base = smem_u32(my_red);
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int idx = (m * 2 + nt) * 4 + e;
                        float v = my_red[idx];
                        for (int q = 1; q < P; ++q) v += ld_dsmem_f32(base + idx * 4, q);
                        acc[m][nt][e] = v;
                    }
        }
        cluster_sync_all();  // peers keep their shared memory until read
    }

    // --------------------------------------------------------------- epilogue
    if (rank == 0 && warp < kConsumerWarps) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int s = nt * 8 + 2 * tq + (e & 1);
                const int64_t r = row0 + warp * 16 + g + (e >= 2 ? 8 : 0);
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
    (void)consumed;
}

template <int EPI>
qg_status launch_s16_t(const S16Params& p0, const DeviceInfo& dev, cudaStream_t stream) {
    constexpr int NMAT = EPI == kEpiSwiglu ? 2 : 1;
    using L = S16Layout<NMAT>;
    auto kern = gemm_s16_kernel<EPI>;
    if (L::kSmem > dev.max_smem_optin) return QG_ERR_SHAPE;
    static int attr_done[64] = {0};
    if (dev.device < 64 && !attr_done[dev.device]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
        if (e != cudaSuccess) return cuda_status(e);
        attr_done[dev.device] = 1;
    }
    S16Params p = p0;
    const int64_t tiles = (p.n + kTileRows - 1) / kTileRows;
    const int nst = static_cast<int>(p.k / kKC);
    // Split K across a cluster until the grid covers the SMs twice over.
    int P = 1;
    while (P < kMaxCluster && tiles * P < 2LL * dev.num_sms && 2 * P <= nst) P *= 2;
    p.splits = P;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles * P));
    cfg.blockDim = dim3(kThreads);
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
    if (L.k % kKC != 0) return QG_ERR_SHAPE;  // 16-byte aligned scale windows
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
