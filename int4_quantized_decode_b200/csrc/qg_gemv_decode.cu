// qg_gemv_decode.cu -- the S=1 kernels of a decode step's fused calls: the
// pre-norm RMSNorm and the residual adds of the Qwen3-architecture decoder
// layers the pages port (the norm itself is not spelled out on the pages),
// compiled apart from the plain kernels so that neither carries the other's
// code:
//  * kEpiNormIn: x = fp16(h * rstd * gamma), the pre-norm RMSNorm of the fp32
//    hidden state, computed by every CTA while it stages x (qkv, gate/up and
//    the head take this input);
//  * kEpiResidual: h[r] = h[r] + y[r], the residual update after o and down.
#include "qg_device.cuh"
#include "qg_internal.h"

namespace qg {
QG_DEFINE_ERROR_FLAG(g_gemv_err);
}  // namespace qg

#include "qg_gemv_impl.cuh"

namespace qg {

qg_status launch_gemv_s1_decode(const GemvLaunch& L, cudaStream_t stream) {
    DeviceInfo dev;
    qg_status st = device_info(&dev);
    if (st != QG_OK) return st;
    const Params p = make_params(L);
    if (L.h_res) {  // the residual update takes an fp16 x (the attention or MLP output)
        if (L.h_in || L.epilogue != kEpiPlain) return QG_ERR_FORMAT;
        if (L.fmt == QG_FMT_I8_B32) return dispatch_fmt<0, kEpiResidual>(L, p, dev, stream);
        if (L.fmt == QG_FMT_I4_G64) return dispatch_fmt<1, kEpiResidual>(L, p, dev, stream);
        return dispatch_fmt<2, kEpiResidual>(L, p, dev, stream);
    }
    if (L.fmt == QG_FMT_I8_B32) return dispatch_fmt<0, kEpiPlain, kEpiNormIn>(L, p, dev, stream);
    if (L.fmt == QG_FMT_I4_G64) return dispatch_fmt<1, kEpiPlain, kEpiNormIn>(L, p, dev, stream);
    return dispatch_fmt<2, kEpiPlain, kEpiNormIn>(L, p, dev, stream);
}

// x = fp16(RMSNorm(h)) as the fused calls stage it: the same per-CTA
// reduction (one 256-thread CTA, the same fixed order) and the same per-piece
// arithmetic, so the values are the ones those calls multiply by.
__global__ void __launch_bounds__(kThreads) rmsnorm_f16_kernel(const float* h, const uint16_t* gamma,
                                                                int64_t k, float eps, uint16_t* x16) {
    __shared__ float red[kWarps];
    griddep_wait();
    const float rstd = rmsnorm_rstd(h, gamma, k, eps, red);
    for (int64_t i = threadIdx.x; i < k / 8; i += kThreads)
        *reinterpret_cast<uint4*>(x16 + 8 * i) = norm_piece(h + 8 * i, gamma + 8 * i, rstd);
    griddep_launch_dependents();
}

qg_status launch_rmsnorm_f16(const float* h, const uint16_t* gamma, int64_t k, float eps,
                             uint16_t* x16, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, rmsnorm_f16_kernel, h, gamma, k, eps, x16));
}

unsigned int gemv_decode_read_and_clear_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_gemv_err, sizeof v) != cudaSuccess) return 0;
    if (v) cudaMemcpyToSymbol(g_gemv_err, &zero, sizeof zero);
    return v;
}

}  // namespace qg
