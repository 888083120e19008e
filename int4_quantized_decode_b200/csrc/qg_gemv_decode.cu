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

unsigned int gemv_decode_read_and_clear_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_gemv_err, sizeof v) != cudaSuccess) return 0;
    if (v) cudaMemcpyToSymbol(g_gemv_err, &zero, sizeof zero);
    return v;
}

}  // namespace qg
