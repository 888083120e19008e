// qg_internal.h -- host-side interfaces between the C-ABI layer (qg_api.cu)
// and the kernel translation units.  Not part of the public ABI.
#pragma once

#include <cstdint>

#include "qgemv.h"

namespace qg {

// Cached per-device properties.
struct DeviceInfo {
    int device;
    int num_sms;
    int max_smem_optin;  // bytes of dynamic shared memory a CTA may opt into
    int smem_per_sm;     // bytes of shared memory per SM
};
qg_status device_info(DeviceInfo* out);

// Map a CUDA error (if any) to a status, clearing it and remembering its name
// for qg_last_cuda_error().
qg_status cuda_status(cudaError_t e);
const char* last_cuda_error_name();

// Epilogues of the S=1 streaming kernel.  kEpiResidual (h_res += y) and the
// flag kEpiNormIn (x = RMSNorm of an fp32 hidden state) are chosen by the
// launcher from h_res / h_in; callers set one of the first three.
enum GemvEpilogue : int { kEpiPlain = 0, kEpiSwiglu = 1, kEpiHead = 2, kEpiResidual = 3 };
constexpr int kEpiNormIn = 8;
__host__ __device__ constexpr int epi_kind(int epi) { return epi & 7; }

// One S=1 streaming launch: NMAT (1 or 2) weights of identical format and
// shape, one fp16 activation, one of three epilogues.
struct GemvLaunch {
    int fmt;  // qg_format
    int epilogue;
    int nmat;
    int64_t n, k;
    const void* codes[2];
    const uint16_t* scales[2];
    const uint16_t* biases[2];
    const uint16_t* x;
    float* y;             // plain: fp32 out or NULL
    uint16_t* y16;        // plain: fp16 out or NULL
    uint16_t* h;          // swiglu: fp16 out
    float* logits;        // head: fp32 out or NULL
    int32_t* idx;         // head: argmax out
    void* workspace;      // head: zeroed scratch (key + ticket)
    const float* h_in;    // if set: x = RMSNorm(h_in; gamma, eps) (x ignored)
    const uint16_t* gamma;
    float eps;
    float* h_res;         // plain: if set, h_res += y (the residual stream)
};
qg_status launch_gemv_s1(const GemvLaunch& L, cudaStream_t stream);
// The decode-step variants (h_in or h_res set), compiled on their own.
qg_status launch_gemv_s1_decode(const GemvLaunch& L, cudaStream_t stream);
// x16 = fp16(RMSNorm(h; gamma, eps)) exactly as the RMSNorm-input calls stage it.
qg_status launch_rmsnorm_f16(const float* h, const uint16_t* gamma, int64_t k, float eps,
                             uint16_t* x16, cudaStream_t stream);

// Persistent sweep: n S=1 stages (validated GemvLaunch descriptions, head
// workspaces ignored) planned into a device workspace, then run as one
// cooperative launch.
size_t sweep_workspace_bytes(int n_stages);
qg_status plan_sweep(const GemvLaunch* L, int n_stages, void* ws, size_t ws_bytes, int* kernel);
qg_status launch_sweep(int kernel, void* ws, int n_stages, cudaStream_t stream);
// The stream sweep (qg_stream.cu): all-int8 plans whose rows hold whole
// 512-code steps run as one launch whose weight stream spans the stages.
size_t stream_workspace_bytes(int n_stages);
qg_status plan_stream(const GemvLaunch* L, int n, void* ws, size_t ws_bytes, int* slots,
                      int* xmax);
qg_status launch_stream(void* ws, int n, int slots, int xmax, cudaStream_t stream);
unsigned int stream_read_and_clear_error();
constexpr int kSweepKernelStream = 2;

// Device error bits of the S=1 kernels (read and cleared by qg_stream_check):
// bit 0 a bounded wait gave up, bit 1 a sweep ran on a workspace that holds
// no plan of that many stages.
constexpr unsigned int kGemvErrTimeout = 1u;
constexpr unsigned int kGemvErrBadPlan = 2u;
constexpr unsigned int kGemvErrToken = 4u;  // embedding gather: token id out of range
unsigned int gemv_read_and_clear_error();
unsigned int gemv_decode_read_and_clear_error();

// h[i] = fp32(table[token][i]) for the device-side token id.
qg_status launch_embedding_gather(const uint16_t* table, int64_t V, int64_t H,
                                  const int32_t* token, float* h, cudaStream_t stream);

// Quantizers.
qg_status launch_quantize_block32(const float* w, int64_t n, int64_t k, int8_t* codes,
                                  uint16_t* scales, cudaStream_t stream);
qg_status launch_quantize_int4_g64(const float* w, int64_t n, int64_t k, uint8_t* codes,
                                   uint16_t* scales, uint16_t* biases, cudaStream_t stream);

// One decode step's attention core (qg_attention.cu).
struct AttentionLaunch {
    const float* qkv;       // fp32 [hq*d | hkv*d | hkv*d]
    uint16_t* kcache;       // fp16 [hkv][l_max][d]
    uint16_t* vcache;
    int64_t l_max;
    int hq, hkv, d;
    const int32_t* pos;     // device
    double theta;
    uint16_t* o;            // fp16 [hq*d]
    void* workspace;
    size_t ws_bytes;
};
size_t decode_attention_workspace_bytes(int hq, int hkv);
qg_status launch_decode_attention(const AttentionLaunch& L, cudaStream_t stream);
unsigned int attention_read_and_clear_error();  // bit 0: position outside [0, l_max); bit 1: a wait expired

// S <= 16 tokens on the tensor cores (qg_gemm_tc.cu): int8 block-32 or int4
// group-64 weights, plain (Y fp32) or SwiGLU (H fp16).
struct GemmS16Launch {
    int fmt;       // QG_FMT_I8_B32 or QG_FMT_I4_G64
    int epilogue;  // kEpiPlain or kEpiSwiglu
    int S;         // 2..16
    int64_t n, k;
    const void* codes[2];
    const uint16_t* scales[2];
    const uint16_t* biases[2];  // int4 only
    const uint16_t* X;
    float* Y;
    uint16_t* H;
};
qg_status launch_gemm_tc(const GemmS16Launch& L, cudaStream_t stream);
unsigned int gemm_tc_read_and_clear_error();

// Head-argmax workspace layout (bytes).
constexpr size_t kHeadWorkspaceBytes = 256;

}  // namespace qg
