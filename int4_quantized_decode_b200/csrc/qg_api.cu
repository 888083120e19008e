// qg_api.cu -- the extern "C" entry points of libqgemv: argument validation
// (synchronous, before any launch) and dispatch to the kernel launchers.
#include <cstdint>
#include <vector>

#include "qg_internal.h"

namespace qg {

namespace {
thread_local cudaError_t t_last_cuda_error = cudaSuccess;
}

qg_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return QG_OK;
    t_last_cuda_error = e;
    (void)cudaGetLastError();  // clear a non-sticky error
    return QG_ERR_CUDA;
}

const char* last_cuda_error_name() { return cudaGetErrorName(t_last_cuda_error); }

qg_status device_info(DeviceInfo* out) {
    static DeviceInfo cache[64];
    static bool valid[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cuda_status(cudaErrorInvalidDevice);
    if (dev >= 0 && dev < 64 && valid[dev]) {
        *out = cache[dev];
        return QG_OK;
    }
    DeviceInfo d;
    d.device = dev;
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&d.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
            cudaSuccess)
        return cuda_status(cudaErrorInvalidDevice);
    if (dev >= 0 && dev < 64) {
        cache[dev] = d;
        valid[dev] = true;
    }
    *out = d;
    return QG_OK;
}

}  // namespace qg

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int64_t block_of(int fmt) { return fmt == QG_FMT_I8_B32 ? 32 : 64; }

// Shape, format and alignment of one weight descriptor.
qg_status check_weight(const qg_weight* W) {
    if (!W) return QG_ERR_NULL;
    if (W->fmt == QG_FMT_F16) {  // plain fp16 weights: rows of whole 16-byte vectors
        if (!W->codes) return QG_ERR_NULL;
        if (W->n < 1 || W->k < 8 || W->k % 8 != 0) return QG_ERR_SHAPE;
        if (W->n > (int64_t(1) << 31) - 1) return QG_ERR_SHAPE;
        if (!aligned(W->codes, 16)) return QG_ERR_ALIGN;
        return QG_OK;
    }
    if (W->fmt != QG_FMT_I8_B32 && W->fmt != QG_FMT_I4_G64) return QG_ERR_FORMAT;
    if (!W->codes || !W->scales) return QG_ERR_NULL;
    if (W->fmt == QG_FMT_I4_G64 && !W->biases) return QG_ERR_NULL;
    if (W->n < 1 || W->k < 1 || W->k % block_of(W->fmt) != 0) return QG_ERR_SHAPE;
    if (W->n > (int64_t(1) << 31) - 1) return QG_ERR_SHAPE;  // row indices are int32 in argmax
    if (!aligned(W->codes, 16) || !aligned(W->scales, 16)) return QG_ERR_ALIGN;
    if (W->fmt == QG_FMT_I4_G64 && !aligned(W->biases, 16)) return QG_ERR_ALIGN;
    return QG_OK;
}

constexpr int kMaxSweepStages = 65536;

// The fp32 hidden state and fp16 gains of an RMSNorm input (read as 16-byte
// vectors), and its epsilon.
qg_status check_norm(const float* h, const uint16_t* gamma, float eps) {
    if (!h || !gamma) return QG_ERR_NULL;
    if (!(eps >= 0.0f) || eps > 1.0f) return QG_ERR_SHAPE;
    if (!aligned(h, 16) || !aligned(gamma, 16)) return QG_ERR_ALIGN;
    return QG_OK;
}

// The launch description of one weight with the plain epilogue.
qg::GemvLaunch plain_launch(const qg_weight& W) {
    qg::GemvLaunch L = {};
    L.fmt = W.fmt;
    L.epilogue = qg::kEpiPlain;
    L.nmat = 1;
    L.n = W.n;
    L.k = W.k;
    L.codes[0] = W.codes;
    L.scales[0] = W.scales;
    L.biases[0] = W.biases;
    return L;
}

// Workspace of a sweep plan: room for either persistent kernel's layout.
size_t sweep_ws_bytes(int n_stages) {
    const size_t a = qg::sweep_workspace_bytes(n_stages), b = qg::stream_workspace_bytes(n_stages);
    return a > b ? a : b;
}

// One sweep stage -> the launch description of the S=1 call it stands for,
// with that call's checks.
qg_status stage_launch(const qg_stage& S, qg::GemvLaunch* out) {
    qg::GemvLaunch L = {};
    qg_status st = check_weight(&S.w);
    if (st != QG_OK) return st;
    if (!S.x) return QG_ERR_NULL;
    if (!aligned(S.x, 16)) return QG_ERR_ALIGN;
    L.fmt = S.w.fmt;
    L.nmat = 1;
    L.n = S.w.n;
    L.k = S.w.k;
    L.codes[0] = S.w.codes;
    L.scales[0] = S.w.scales;
    L.biases[0] = S.w.biases;
    L.x = S.x;
    switch (S.op) {
        case QG_STAGE_GEMV:
            if (!S.y && !S.y16) return QG_ERR_NULL;
            if ((S.y && !aligned(S.y, 4)) || (S.y16 && !aligned(S.y16, 2))) return QG_ERR_ALIGN;
            L.epilogue = qg::kEpiPlain;
            L.y = S.y;
            L.y16 = S.y16;
            break;
        case QG_STAGE_SWIGLU:
            st = check_weight(&S.w_up);
            if (st != QG_OK) return st;
            if (S.w_up.fmt != S.w.fmt) return QG_ERR_FORMAT;
            if (S.w_up.n != S.w.n || S.w_up.k != S.w.k) return QG_ERR_SHAPE;
            if (!S.h) return QG_ERR_NULL;
            if (!aligned(S.h, 2)) return QG_ERR_ALIGN;
            L.epilogue = qg::kEpiSwiglu;
            L.nmat = 2;
            L.codes[1] = S.w_up.codes;
            L.scales[1] = S.w_up.scales;
            L.biases[1] = S.w_up.biases;
            L.h = S.h;
            break;
        case QG_STAGE_HEAD_ARGMAX:
            if (!S.idx) return QG_ERR_NULL;
            if ((S.logits && !aligned(S.logits, 4)) || !aligned(S.idx, 4)) return QG_ERR_ALIGN;
            L.epilogue = qg::kEpiHead;
            L.logits = S.logits;
            L.idx = S.idx;
            break;
        default:
            return QG_ERR_FORMAT;
    }
    *out = L;
    return QG_OK;
}

}  // namespace

extern "C" {

int qg_abi_version(void) { return 103; }

const char* qg_last_cuda_error(void) { return qg::last_cuda_error_name(); }

const char* qg_status_string(qg_status s) {
    switch (s) {
        case QG_OK: return "QG_OK";
        case QG_ERR_NULL: return "QG_ERR_NULL: a required pointer is NULL";
        case QG_ERR_SHAPE: return "QG_ERR_SHAPE: unsupported n, k or S";
        case QG_ERR_ALIGN: return "QG_ERR_ALIGN: pointer not aligned as documented";
        case QG_ERR_FORMAT: return "QG_ERR_FORMAT: unknown or mismatched weight format";
        case QG_ERR_WORKSPACE: return "QG_ERR_WORKSPACE: workspace NULL or too small";
        case QG_ERR_CUDA: return "QG_ERR_CUDA: CUDA runtime error";
        case QG_ERR_TIMEOUT: return "QG_ERR_TIMEOUT: a device-side bounded wait expired";
        case QG_ERR_PLAN: return "QG_ERR_PLAN: the workspace holds no sweep plan of that size";
    }
    return "QG_ERR_UNKNOWN";
}

qg_status qg_quantize_block32(const float* w, int64_t n, int64_t k, int8_t* codes,
                              uint16_t* scales, cudaStream_t stream) {
    if (!w || !codes || !scales) return QG_ERR_NULL;
    if (n < 1 || k < 32 || k % 32 != 0) return QG_ERR_SHAPE;
    if (!aligned(w, 16) || !aligned(codes, 16) || !aligned(scales, 2)) return QG_ERR_ALIGN;
    return qg::launch_quantize_block32(w, n, k, codes, scales, stream);
}

qg_status qg_quantize_int4_g64(const float* w, int64_t n, int64_t k, uint8_t* codes,
                               uint16_t* scales, uint16_t* biases, cudaStream_t stream) {
    if (!w || !codes || !scales || !biases) return QG_ERR_NULL;
    if (n < 1 || k < 64 || k % 64 != 0) return QG_ERR_SHAPE;
    if (!aligned(w, 16) || !aligned(codes, 16) || !aligned(scales, 2) || !aligned(biases, 2))
        return QG_ERR_ALIGN;
    return qg::launch_quantize_int4_g64(w, n, k, codes, scales, biases, stream);
}

qg_status qg_gemv_s1(const qg_weight* W, const uint16_t* x, float* y, uint16_t* y16,
                     cudaStream_t stream) {
    qg_status st = check_weight(W);
    if (st != QG_OK) return st;
    if (!x || (!y && !y16)) return QG_ERR_NULL;
    if (!aligned(x, 16) || (y && !aligned(y, 4)) || (y16 && !aligned(y16, 2))) return QG_ERR_ALIGN;
    qg::GemvLaunch L = {};
    L.fmt = W->fmt;
    L.epilogue = qg::kEpiPlain;
    L.nmat = 1;
    L.n = W->n;
    L.k = W->k;
    L.codes[0] = W->codes;
    L.scales[0] = W->scales;
    L.biases[0] = W->biases;
    L.x = x;
    L.y = y;
    L.y16 = y16;
    return qg::launch_gemv_s1(L, stream);
}

qg_status qg_gemm_s16(const qg_weight* W, const uint16_t* X, int S, float* Y,
                      cudaStream_t stream) {
    qg_status st = check_weight(W);
    if (st != QG_OK) return st;
    if (!X || !Y) return QG_ERR_NULL;
    if (S < 1 || S > 16) return QG_ERR_SHAPE;
    if (!aligned(X, 16) || !aligned(Y, 4)) return QG_ERR_ALIGN;
    if (S == 1) return qg_gemv_s1(W, X, Y, nullptr, stream);
    if (W->fmt == QG_FMT_F16) return QG_ERR_FORMAT;
    qg::GemmS16Launch L = {};
    L.fmt = W->fmt;
    L.epilogue = qg::kEpiPlain;
    L.S = S;
    L.n = W->n;
    L.k = W->k;
    L.codes[0] = L.codes[1] = W->codes;
    L.scales[0] = L.scales[1] = W->scales;
    L.biases[0] = L.biases[1] = W->biases;
    L.X = X;
    L.Y = Y;
    return qg::launch_gemm_tc(L, stream);
}

qg_status qg_gate_up_swiglu(const qg_weight* Wg, const qg_weight* Wu, const uint16_t* X, int S,
                            uint16_t* H, cudaStream_t stream) {
    qg_status st = check_weight(Wg);
    if (st != QG_OK) return st;
    st = check_weight(Wu);
    if (st != QG_OK) return st;
    if (Wg->fmt != Wu->fmt || Wg->fmt == QG_FMT_F16) return QG_ERR_FORMAT;
    if (Wg->n != Wu->n || Wg->k != Wu->k) return QG_ERR_SHAPE;
    if (!X || !H) return QG_ERR_NULL;
    if (S < 1 || S > 16) return QG_ERR_SHAPE;
    if (!aligned(X, 16) || !aligned(H, 2)) return QG_ERR_ALIGN;
    if (S == 1) {
        qg::GemvLaunch L = {};
        L.fmt = Wg->fmt;
        L.epilogue = qg::kEpiSwiglu;
        L.nmat = 2;
        L.n = Wg->n;
        L.k = Wg->k;
        L.codes[0] = Wg->codes;
        L.scales[0] = Wg->scales;
        L.biases[0] = Wg->biases;
        L.codes[1] = Wu->codes;
        L.scales[1] = Wu->scales;
        L.biases[1] = Wu->biases;
        L.x = X;
        L.h = H;
        return qg::launch_gemv_s1(L, stream);
    }
    qg::GemmS16Launch L = {};
    L.fmt = Wg->fmt;
    L.epilogue = qg::kEpiSwiglu;
    L.S = S;
    L.n = Wg->n;
    L.k = Wg->k;
    L.codes[0] = Wg->codes;
    L.scales[0] = Wg->scales;
    L.biases[0] = Wg->biases;
    L.codes[1] = Wu->codes;
    L.scales[1] = Wu->scales;
    L.biases[1] = Wu->biases;
    L.X = X;
    L.H = H;
    return qg::launch_gemm_tc(L, stream);
}

size_t qg_head_argmax_workspace_bytes(int64_t n) {
    (void)n;
    return qg::kHeadWorkspaceBytes;
}

qg_status qg_head_argmax(const qg_weight* W, const uint16_t* x, float* logits, int32_t* idx,
                         void* workspace, size_t ws_bytes, cudaStream_t stream) {
    qg_status st = check_weight(W);
    if (st != QG_OK) return st;
    if (!x || !idx) return QG_ERR_NULL;
    if (!workspace || ws_bytes < qg::kHeadWorkspaceBytes) return QG_ERR_WORKSPACE;
    if (!aligned(x, 16) || (logits && !aligned(logits, 4)) || !aligned(idx, 4) ||
        !aligned(workspace, 16))
        return QG_ERR_ALIGN;
    qg::GemvLaunch L = {};
    L.fmt = W->fmt;
    L.epilogue = qg::kEpiHead;
    L.nmat = 1;
    L.n = W->n;
    L.k = W->k;
    L.codes[0] = W->codes;
    L.scales[0] = W->scales;
    L.biases[0] = W->biases;
    L.x = x;
    L.logits = logits;
    L.idx = idx;
    L.workspace = workspace;
    return qg::launch_gemv_s1(L, stream);
}

size_t qg_sweep_workspace_bytes(int n_stages) {
    if (n_stages < 1 || n_stages > kMaxSweepStages) return 0;
    return sweep_ws_bytes(n_stages);
}

qg_status qg_sweep_plan(const qg_stage* stages, int n_stages, void* workspace, size_t ws_bytes,
                        qg_sweep* sweep) {
    if (!stages || !sweep) return QG_ERR_NULL;
    if (n_stages < 1 || n_stages > kMaxSweepStages) return QG_ERR_SHAPE;
    if (!workspace || ws_bytes < sweep_ws_bytes(n_stages)) return QG_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return QG_ERR_ALIGN;
    std::vector<qg::GemvLaunch> L(static_cast<size_t>(n_stages));
    for (int i = 0; i < n_stages; ++i) {
        qg_status st = stage_launch(stages[i], &L[i]);
        if (st != QG_OK) return st;
    }
    qg_sweep out = {};
    out.n_stages = n_stages;
    // the stream sweep when the plan qualifies (all int8, rows of whole
    // 512-code steps), else the general persistent kernels
    int slots = 0, xmax = 0;
    qg_status st = qg::plan_stream(L.data(), n_stages, workspace, ws_bytes, &slots, &xmax);
    if (st == QG_OK) {
        out.kernel = qg::kSweepKernelStream;
        out.reserved[0] = slots;
        out.reserved[1] = xmax;
        *sweep = out;
        return QG_OK;
    }
    if (st != QG_ERR_FORMAT && st != QG_ERR_SHAPE) return st;
    int kernel = -1;
    st = qg::plan_sweep(L.data(), n_stages, workspace, ws_bytes, &kernel);
    if (st != QG_OK) return st;
    out.kernel = kernel;
    *sweep = out;
    return QG_OK;
}

qg_status qg_sweep_run(const qg_sweep* sweep, void* workspace, cudaStream_t stream) {
    if (!sweep || !workspace) return QG_ERR_NULL;
    if (sweep->n_stages < 1 || sweep->n_stages > kMaxSweepStages) return QG_ERR_SHAPE;
    if (!aligned(workspace, 256)) return QG_ERR_ALIGN;
    if (sweep->kernel == qg::kSweepKernelStream)
        return qg::launch_stream(workspace, sweep->n_stages, static_cast<int>(sweep->reserved[0]),
                                 static_cast<int>(sweep->reserved[1]), stream);
    return qg::launch_sweep(sweep->kernel, workspace, sweep->n_stages, stream);
}

// ---------------------------------------------------- decode-step fusions ---

qg_status qg_embedding_gather(const uint16_t* table, int64_t V, int64_t H, const int32_t* token,
                              float* h, cudaStream_t stream) {
    if (!table || !token || !h) return QG_ERR_NULL;
    if (V < 1 || H < 1 || V > (int64_t(1) << 31) - 1) return QG_ERR_SHAPE;
    if (!aligned(table, 2) || !aligned(token, 4) || !aligned(h, 4)) return QG_ERR_ALIGN;
    return qg::launch_embedding_gather(table, V, H, token, h, stream);
}

size_t qg_decode_attention_workspace_bytes(int hq, int hkv) {
    if (hq < 1 || hkv < 1 || hq % hkv != 0) return 0;
    return qg::decode_attention_workspace_bytes(hq, hkv);
}

qg_status qg_decode_attention(const float* qkv, int hq, int hkv, int d, uint16_t* kcache,
                              uint16_t* vcache, int64_t l_max, const int32_t* pos, double theta,
                              uint16_t* o, void* workspace, size_t ws_bytes, cudaStream_t stream) {
    if (!qkv || !kcache || !vcache || !pos || !o || !workspace) return QG_ERR_NULL;
    if (hkv < 1 || hq < hkv || hq % hkv != 0 || l_max < 1 || l_max > (int64_t(1) << 31) - 1)
        return QG_ERR_SHAPE;
    const int group = hq / hkv;
    if (d != 128 || (group != 1 && group != 2 && group != 4)) return QG_ERR_SHAPE;
    if (!(theta > 0.0)) return QG_ERR_SHAPE;
    if (!aligned(qkv, 16) || !aligned(kcache, 16) || !aligned(vcache, 16) || !aligned(pos, 4) ||
        !aligned(o, 16) || !aligned(workspace, 256))
        return QG_ERR_ALIGN;
    if (ws_bytes < qg::decode_attention_workspace_bytes(hq, hkv)) return QG_ERR_WORKSPACE;
    qg::AttentionLaunch L = {};
    L.qkv = qkv;
    L.kcache = kcache;
    L.vcache = vcache;
    L.l_max = l_max;
    L.hq = hq;
    L.hkv = hkv;
    L.d = d;
    L.pos = pos;
    L.theta = theta;
    L.o = o;
    L.workspace = workspace;
    L.ws_bytes = ws_bytes;
    return qg::launch_decode_attention(L, stream);
}

qg_status qg_rmsnorm_gemv_s1(const qg_weight* W, const float* h, const uint16_t* gamma, float eps,
                             float* y, uint16_t* y16, cudaStream_t stream) {
    qg_status st = check_weight(W);
    if (st != QG_OK) return st;
    st = check_norm(h, gamma, eps);
    if (st != QG_OK) return st;
    if (!y && !y16) return QG_ERR_NULL;
    if ((y && !aligned(y, 4)) || (y16 && !aligned(y16, 2))) return QG_ERR_ALIGN;
    qg::GemvLaunch L = plain_launch(*W);
    L.h_in = h;
    L.gamma = gamma;
    L.eps = eps;
    L.y = y;
    L.y16 = y16;
    return qg::launch_gemv_s1(L, stream);
}

qg_status qg_rmsnorm_f16(const float* h, const uint16_t* gamma, int64_t k, float eps,
                         uint16_t* x16, cudaStream_t stream) {
    qg_status st = check_norm(h, gamma, eps);
    if (st != QG_OK) return st;
    if (!x16) return QG_ERR_NULL;
    if (k < 8 || k % 8 != 0) return QG_ERR_SHAPE;
    if (!aligned(x16, 16)) return QG_ERR_ALIGN;
    return qg::launch_rmsnorm_f16(h, gamma, k, eps, x16, stream);
}

qg_status qg_gemv_s1_residual(const qg_weight* W, const uint16_t* x, float* h,
                              cudaStream_t stream) {
    qg_status st = check_weight(W);
    if (st != QG_OK) return st;
    if (!x || !h) return QG_ERR_NULL;
    if (!aligned(x, 16) || !aligned(h, 4)) return QG_ERR_ALIGN;
    qg::GemvLaunch L = plain_launch(*W);
    L.x = x;
    L.h_res = h;
    return qg::launch_gemv_s1(L, stream);
}

qg_status qg_rmsnorm_gate_up_swiglu(const qg_weight* Wg, const qg_weight* Wu, const float* h,
                                    const uint16_t* gamma, float eps, uint16_t* H,
                                    cudaStream_t stream) {
    qg_status st = check_weight(Wg);
    if (st != QG_OK) return st;
    st = check_weight(Wu);
    if (st != QG_OK) return st;
    if (Wg->fmt != Wu->fmt || Wg->fmt == QG_FMT_F16) return QG_ERR_FORMAT;
    if (Wg->n != Wu->n || Wg->k != Wu->k) return QG_ERR_SHAPE;
    st = check_norm(h, gamma, eps);
    if (st != QG_OK) return st;
    if (!H) return QG_ERR_NULL;
    if (!aligned(H, 2)) return QG_ERR_ALIGN;
    qg::GemvLaunch L = plain_launch(*Wg);
    L.epilogue = qg::kEpiSwiglu;
    L.nmat = 2;
    L.codes[1] = Wu->codes;
    L.scales[1] = Wu->scales;
    L.biases[1] = Wu->biases;
    L.h_in = h;
    L.gamma = gamma;
    L.eps = eps;
    L.h = H;
    return qg::launch_gemv_s1(L, stream);
}

qg_status qg_rmsnorm_head_argmax(const qg_weight* W, const float* h, const uint16_t* gamma,
                                 float eps, float* logits, int32_t* idx, void* workspace,
                                 size_t ws_bytes, cudaStream_t stream) {
    qg_status st = check_weight(W);
    if (st != QG_OK) return st;
    st = check_norm(h, gamma, eps);
    if (st != QG_OK) return st;
    if (!idx) return QG_ERR_NULL;
    if (!workspace || ws_bytes < qg::kHeadWorkspaceBytes) return QG_ERR_WORKSPACE;
    if ((logits && !aligned(logits, 4)) || !aligned(idx, 4) || !aligned(workspace, 16))
        return QG_ERR_ALIGN;
    qg::GemvLaunch L = plain_launch(*W);
    L.epilogue = qg::kEpiHead;
    L.h_in = h;
    L.gamma = gamma;
    L.eps = eps;
    L.logits = logits;
    L.idx = idx;
    L.workspace = workspace;
    return qg::launch_gemv_s1(L, stream);
}

qg_status qg_stream_check(cudaStream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return qg::cuda_status(e);
    const unsigned int g = qg::gemv_read_and_clear_error() | qg::gemv_decode_read_and_clear_error() |
                           qg::stream_read_and_clear_error();
    const unsigned int f = g | qg::gemm_tc_read_and_clear_error();
    const unsigned int a = qg::attention_read_and_clear_error();
    if (g & qg::kGemvErrBadPlan) return QG_ERR_PLAN;
    if ((g & qg::kGemvErrToken) || (a & 1u)) return QG_ERR_SHAPE;  // a position out of range
    return (f || (a & 2u)) ? QG_ERR_TIMEOUT : QG_OK;
}

}  // extern "C"
