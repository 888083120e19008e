// qg_gemv.cu -- the S=1 entry points: plain GEMV, fused gate/up SwiGLU and
// fused head argmax launches (kernel templates in qg_gemv_impl.cuh), the
// persistent sweep that runs a decode step's stages in one launch, and the
// device-side embedding gather.
#include <vector>

#include "qg_device.cuh"
#include "qg_internal.h"

namespace qg {
QG_DEFINE_ERROR_FLAG(g_gemv_err);
}  // namespace qg

#include "qg_gemv_impl.cuh"

namespace qg {
namespace {

// ----------------------------------------------------------------------- //
// Persistent sweep: every stage of a decode step in one launch.            //
// ----------------------------------------------------------------------- //
// A stage's variant within the kernel that runs its plan.  Each kernel holds
// only as many ring variants as fit its 128 registers per thread without
// spilling: kernel 0 runs int8 plans (every epilogue, 1/2/4 rows per warp
// item), kernel 1 runs int4 plans (int4 projections at 1-2 rows, SwiGLU at
// 1 row, and the int8 head the pages pair with an int4 body).
enum : int32_t {
    kVarPlain1, kVarPlain2, kVarPlain4, kVarSwiglu1, kVarSwiglu2,
    kVarHead1, kVarHead2, kVarHead4
};
enum : int32_t { kI4Plain1, kI4Plain2, kI4Swiglu1, kI4Head8x1, kI4Head8x2, kI4Head8x4 };

constexpr uint32_t kSweepMagic = 0x57534751u;  // "QGSW"

struct SweepHeader {
    uint32_t magic;
    int32_t n_stages;
    int32_t kernel;
    uint32_t reserved[61];
};
static_assert(sizeof(SweepHeader) == 256, "header is 256 bytes");

struct SweepStage {
    Params p;
    int32_t variant;
    int32_t reserved[5];
};

__host__ __device__ constexpr size_t align256(size_t v) { return (v + 255) / 256 * 256; }

// Workspace: [header][arrival counters: one per stage + one exit counter]
//            [16 bytes of argmax scratch per stage][stage descriptors]
__host__ __device__ constexpr size_t sweep_counters_offset() { return sizeof(SweepHeader); }
__host__ __device__ constexpr size_t sweep_scratch_offset(int n) {
    return sweep_counters_offset() + align256(static_cast<size_t>(n + 1) * 4);
}
__host__ __device__ constexpr size_t sweep_stages_offset(int n) {
    return sweep_scratch_offset(n) + align256(static_cast<size_t>(n) * 16);
}

// The stage's parameters are read from shared memory where they are needed
// (per item, not per step), as a launch of its own reads its constant bank.
template <int FMT, int NMAT, int RG, int EPI>
__device__ __forceinline__ bool sweep_stage(const SweepStage* st, unsigned char* smem,
                                            GridSync& sync, float* red_v, int* red_i) {
    return ring_stage<FMT, NMAT, RG, EPI>(st->p, smem, sync, red_v, red_i);
}

template <int KERNEL>
__device__ __forceinline__ bool sweep_dispatch(int v, const SweepStage* st, unsigned char* smem,
                                               GridSync& sync, float* red_v, int* red_i) {
#define QG_STAGE(F, M, R, E) return sweep_stage<F, M, R, E>(st, smem, sync, red_v, red_i)
    if (KERNEL == 0) {
        switch (v) {
            case kVarPlain1: QG_STAGE(0, 1, 1, kEpiPlain);
            case kVarPlain2: QG_STAGE(0, 1, 2, kEpiPlain);
            case kVarPlain4: QG_STAGE(0, 1, 4, kEpiPlain);
            case kVarSwiglu1: QG_STAGE(0, 2, 1, kEpiSwiglu);
            case kVarSwiglu2: QG_STAGE(0, 2, 2, kEpiSwiglu);
            case kVarHead1: QG_STAGE(0, 1, 1, kEpiHead);
            case kVarHead2: QG_STAGE(0, 1, 2, kEpiHead);
            default: QG_STAGE(0, 1, 4, kEpiHead);
        }
    } else {
        switch (v) {
            case kI4Plain1: QG_STAGE(1, 1, 1, kEpiPlain);
            case kI4Plain2: QG_STAGE(1, 1, 2, kEpiPlain);
            case kI4Swiglu1: QG_STAGE(1, 2, 1, kEpiSwiglu);
            case kI4Head8x1: QG_STAGE(0, 1, 1, kEpiHead);
            case kI4Head8x2: QG_STAGE(0, 1, 2, kEpiHead);
            default: QG_STAGE(0, 1, 4, kEpiHead);
        }
    }
#undef QG_STAGE
}

// One CTA per (SM, slot) for the whole sweep.  Stage s + 1 streams its first
// weights while the grid waits for the last CTAs of stage s; x of stage s + 1
// is read only after every CTA has finished stage s, the order a stream of
// separate launches gives.  Requires every CTA to be resident at once (a
// cooperative launch).
template <int KERNEL>
__global__ void __launch_bounds__(kThreads, 2) sweep_kernel(unsigned char* ws, int n_stages) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ float red_v[kWarps];
    __shared__ int red_i[kWarps];
    __shared__ int go;
    __shared__ __align__(16) SweepStage desc[2];  // this stage's and the next one's
    const SweepHeader* hdr = reinterpret_cast<const SweepHeader*>(ws);
    if (hdr->magic != kSweepMagic || hdr->n_stages != n_stages || hdr->kernel != KERNEL) {
        if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(&g_gemv_err, kGemvErrBadPlan);
        return;
    }
    unsigned int* ctr = reinterpret_cast<unsigned int*>(ws + sweep_counters_offset());
    const SweepStage* stages = reinterpret_cast<const SweepStage*>(ws + sweep_stages_offset(n_stages));
    static_assert(sizeof(SweepStage) % 16 == 0, "stage descriptors copy as 16-byte pieces");
    constexpr int kPieces = static_cast<int>(sizeof(SweepStage) / 16);
    if (threadIdx.x < kPieces)
        reinterpret_cast<uint4*>(&desc[0])[threadIdx.x] =
            ldg_nc_v4(reinterpret_cast<const uint4*>(stages) + threadIdx.x);
    for (int s = 0; s < n_stages; ++s) {
        __syncthreads();  // every warp is done with the previous stage; desc[s & 1] is in
        const SweepStage* cur = &desc[s & 1];
        GridSync sync{s > 0 ? ctr + (s - 1) : nullptr, &go,
                      s + 1 < n_stages ? reinterpret_cast<const uint4*>(stages + s + 1) : nullptr,
                      reinterpret_cast<uint4*>(&desc[(s + 1) & 1]), kPieces};
        const bool ok = sweep_dispatch<KERNEL>(cur->variant, cur, smem, sync, red_v, red_i);
        if (!ok) {
            if (threadIdx.x == 0) atomicOr(&g_gemv_err, kGemvErrTimeout);
            return;
        }
    }
    // The last CTA to finish re-zeroes every counter for the next run (no CTA
    // reads a counter after it has arrived here).
    __syncthreads();
    if (threadIdx.x == 0) {
        if (atomicAdd(ctr + n_stages, 1u) == gridDim.x - 1) {
            for (int s = 0; s <= n_stages; ++s) ctr[s] = 0u;
            __threadfence();
        }
    }
}


// The variant of a sweep stage in kernel `kernel`: the standalone launch's
// choice of rows per item, lowered to what the kernel holds and until the
// stage's rings and x fit the per-CTA budget.  Returns -1 (with *status set)
// if the kernel has no variant for the stage.
int sweep_variant(int kernel, const GemvLaunch& L, Params* p, int total_warps, int* rg_out,
                  qg_status* status) {
    if (L.fmt == QG_FMT_F16) {  // the persistent kernels hold no fp16-weight variant
        *status = QG_ERR_FORMAT;
        return -1;
    }
    const int block = L.fmt == QG_FMT_I8_B32 ? 32 : 64;
    *status = QG_ERR_SHAPE;
    if ((L.k / block) % 8 != 0) return -1;
    const bool swiglu = L.epilogue == kEpiSwiglu, head = L.epilogue == kEpiHead;
    int max_rg = swiglu ? 2 : 4;
    if (kernel == 1) {
        if (head ? L.fmt != QG_FMT_I8_B32 : L.fmt != QG_FMT_I4_G64) {
            *status = QG_ERR_FORMAT;
            return -1;
        }
        if (!head) max_rg = swiglu ? 1 : 2;
    }
    const int nmat = swiglu ? 2 : 1;
    for (int rg = pick_rg(L.n, max_rg, total_warps); rg >= 1; rg /= 2) {
        p->x_bulk = p->h_in ? 0 : 1;  // x by bulk copy if its raw buffer fits too
        if (x_smem_bytes(L.fmt, *p) + ring_bytes(L.fmt, nmat * rg) > kSmemPerCtaBudget)
            p->x_bulk = 0;
        if (x_smem_bytes(L.fmt, *p) + ring_bytes(L.fmt, nmat * rg) > kSmemPerCtaBudget) continue;
        *rg_out = rg;
        *status = QG_OK;
        if (kernel == 0) {
            if (swiglu) return rg == 2 ? kVarSwiglu2 : kVarSwiglu1;
            if (head) return rg == 4 ? kVarHead4 : (rg == 2 ? kVarHead2 : kVarHead1);
            return rg == 4 ? kVarPlain4 : (rg == 2 ? kVarPlain2 : kVarPlain1);
        }
        if (swiglu) return kI4Swiglu1;
        if (head) return rg == 4 ? kI4Head8x4 : (rg == 2 ? kI4Head8x2 : kI4Head8x1);
        return rg == 2 ? kI4Plain2 : kI4Plain1;
    }
    return -1;
}

}  // namespace

size_t sweep_workspace_bytes(int n_stages) {
    return sweep_stages_offset(n_stages) + static_cast<size_t>(n_stages) * sizeof(SweepStage);
}

qg_status plan_sweep(const GemvLaunch* L, int n_stages, void* ws, size_t ws_bytes,
                     int* kernel_out) {
    DeviceInfo dev;
    qg_status st = device_info(&dev);
    if (st != QG_OK) return st;
    const size_t bytes = sweep_workspace_bytes(n_stages);
    if (ws_bytes < bytes) return QG_ERR_WORKSPACE;
    int kernel = 0;
    for (int i = 0; i < n_stages; ++i)
        if (L[i].fmt == QG_FMT_I4_G64) kernel = 1;
    std::vector<unsigned char> host(bytes, 0);
    SweepHeader* hdr = reinterpret_cast<SweepHeader*>(host.data());
    hdr->magic = kSweepMagic;
    hdr->n_stages = n_stages;
    hdr->kernel = kernel;
    SweepStage* stages = reinterpret_cast<SweepStage*>(host.data() + sweep_stages_offset(n_stages));
    unsigned char* dev_base = static_cast<unsigned char*>(ws);
    const int total_warps = dev.num_sms * kCtasPerSm * kWarps;
    for (int i = 0; i < n_stages; ++i) {
        GemvLaunch Li = L[i];
        if (Li.epilogue == kEpiHead) Li.workspace = dev_base + sweep_scratch_offset(n_stages) + 16 * i;
        Params p = make_params(Li);
        int rg = 1;
        const int v = sweep_variant(kernel, Li, &p, total_warps, &rg, &st);
        if (v < 0) return st;
        const int nmat = Li.epilogue == kEpiSwiglu ? 2 : 1;
        const int64_t item_bytes = static_cast<int64_t>(nmat) * rg * (Li.fmt == 0 ? Li.k : Li.k / 2);
        p.prefetch_items = static_cast<int>(kPrefetchBytesPerWarp / item_bytes);
        if (p.prefetch_items < 1) p.prefetch_items = 1;
        stages[i].p = p;
        stages[i].variant = v;
    }
    st = cuda_status(cudaMemcpy(ws, host.data(), bytes, cudaMemcpyHostToDevice));
    if (st == QG_OK) *kernel_out = kernel;
    return st;
}

qg_status launch_sweep(int kernel, void* ws, int n_stages, cudaStream_t stream) {
    DeviceInfo dev;
    qg_status st = device_info(&dev);
    if (st != QG_OK) return st;
    if (kernel != 0 && kernel != 1) return QG_ERR_PLAN;
    auto kern = kernel == 0 ? sweep_kernel<0> : sweep_kernel<1>;
    static bool attr_set[2][64] = {{false}};
    if (dev.device >= 64 || !attr_set[kernel][dev.device]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kSmemPerCtaBudget));
        if (e != cudaSuccess) return cuda_status(e);
        if (dev.device < 64) attr_set[kernel][dev.device] = true;
    }
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads,
                                                                  kSmemPerCtaBudget);
    if (e != cudaSuccess) return cuda_status(e);
    if (per_sm < 1) return QG_ERR_SHAPE;
    if (per_sm > kCtasPerSm) per_sm = kCtasPerSm;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(dev.num_sms * per_sm));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemPerCtaBudget;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, static_cast<unsigned char*>(ws), n_stages));
}

qg_status launch_gemv_s1(const GemvLaunch& L, cudaStream_t stream) {
    DeviceInfo dev;
    qg_status st = device_info(&dev);
    if (st != QG_OK) return st;
    if (L.h_in || L.h_res) return launch_gemv_s1_decode(L, stream);
    const Params p = make_params(L);
    if (L.fmt == QG_FMT_I8_B32) return dispatch_fmt<0>(L, p, dev, stream);
    if (L.fmt == QG_FMT_I4_G64) return dispatch_fmt<1>(L, p, dev, stream);
    return dispatch_fmt<2>(L, p, dev, stream);
}

// h[i] = fp32(table[token][i]): the embedding row of the token the previous
// step chose ("Qwen3.8-27B ... -- Core AI", The vision path: the host gathers
// text rows from the fp16 embedding table; here the row is gathered on the
// device from the device-side argmax, so a decode loop never leaves the GPU).
__global__ void __launch_bounds__(256) embedding_gather_kernel(const uint16_t* table, int64_t V,
                                                               int64_t H, const int32_t* token,
                                                               float* h) {
    griddep_wait();  // the token may be the previous kernel's argmax
    const int32_t t = *token;
    if (t < 0 || t >= V) {
        if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(&g_gemv_err, kGemvErrToken);
        return;
    }
    const uint16_t* row = table + static_cast<int64_t>(t) * H;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < H;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        h[i] = h2f(row[i]);
    griddep_launch_dependents();
}

qg_status launch_embedding_gather(const uint16_t* table, int64_t V, int64_t H,
                                  const int32_t* token, float* h, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((H + 1023) / 1024));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, embedding_gather_kernel, table, V, H, token, h));
}

unsigned int gemv_read_and_clear_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_gemv_err, sizeof v) != cudaSuccess) return 0;
    if (v) cudaMemcpyToSymbol(g_gemv_err, &zero, sizeof zero);
    return v;
}

}  // namespace qg
