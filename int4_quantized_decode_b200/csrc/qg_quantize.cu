// qg_quantize.cu -- offline quantizers (fp32 weights -> codes + fp16 side data).
//
// int8 per-block-32 symmetric absmax ("Qwen3-VL 4B -- Core AI (.aimodel)",
// Files; "Qwen3.8-27B ... -- Core AI", Verified: absmax, no clipping) and
// int4 group-64 affine ("Qwen3-VL 4B & 8B -- Core ML stateful", Architecture).
// Every floating-point step is one IEEE fp32 operation rounded to nearest
// even (explicit __fdiv_rn / __fsub_rn, no contraction), followed by an RNE
// conversion to fp16, so the codes and scales are bit-identical to the CPU
// oracle's.  Both kernels are streaming (4 B read + ~1.06 / 0.56 B written
// per weight): lanes cooperate on one block so every access is coalesced.
#include "qg_device.cuh"
#include "qg_internal.h"

namespace qg {
namespace {

constexpr int kThreads = 256;

// 8 lanes per block of 32 weights; each lane holds one float4.  Blocks are
// contiguous in memory (row-major, k % 32 == 0), so block b covers weights
// [32 b, 32 b + 32), codes [32 b, ...) and scale b.
__global__ void __launch_bounds__(kThreads) quantize_block32_kernel(const float* __restrict__ w,
                                                                    int64_t nblocks,
                                                                    int8_t* __restrict__ codes,
                                                                    uint16_t* __restrict__ scales) {
    const int lane = threadIdx.x & 31;
    const int sub = lane & 7;  // position inside the block
    const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t warps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
    for (int64_t b0 = warp_global * 4; b0 < nblocks; b0 += warps * 4) {
        const int64_t b = b0 + (lane >> 3);
        const bool valid = b < nblocks;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (valid) v = reinterpret_cast<const float4*>(w + b * 32)[sub];
        float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        const uint16_t s16 = f2h_rn(__fdiv_rn(a, 127.0f));
        const float s = h2f(s16);
        auto code = [&](float x) -> uint32_t {
            if (s == 0.0f) return 0u;
            int q = __float2int_rn(__fdiv_rn(x, s));
            q = q > 127 ? 127 : (q < -127 ? -127 : q);
            return static_cast<uint32_t>(q) & 0xFFu;
        };
        if (valid) {
            const uint32_t packed = code(v.x) | (code(v.y) << 8) | (code(v.z) << 16) | (code(v.w) << 24);
            reinterpret_cast<uint32_t*>(codes + b * 32)[sub] = packed;
            if (sub == 0) scales[b] = s16;
        }
    }
}

// 16 lanes per group of 64 weights; each lane holds one float4 and writes the
// two bytes of its four codes (even k in the low nibble).
__global__ void __launch_bounds__(kThreads) quantize_int4_kernel(const float* __restrict__ w,
                                                                 int64_t ngroups,
                                                                 uint8_t* __restrict__ codes,
                                                                 uint16_t* __restrict__ scales,
                                                                 uint16_t* __restrict__ biases) {
    const int lane = threadIdx.x & 31;
    const int sub = lane & 15;
    const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t warps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
    for (int64_t g0 = warp_global * 2; g0 < ngroups; g0 += warps * 2) {
        const int64_t g = g0 + (lane >> 4);
        const bool valid = g < ngroups;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (valid) v = reinterpret_cast<const float4*>(w + g * 64)[sub];
        float mx = fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w));
        float mn = fminf(fminf(v.x, v.y), fminf(v.z, v.w));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        }
        mx = __fadd_rn(mx, 0.0f);  // a signed-zero extreme counts as +0
        mn = __fadd_rn(mn, 0.0f);
        const uint16_t s16 = f2h_rn(__fdiv_rn(__fsub_rn(mx, mn), 15.0f));
        const uint16_t b16 = f2h_rn(mn);
        const float s = h2f(s16);
        const float bias = h2f(b16);
        auto code = [&](float x) -> uint32_t {
            if (s == 0.0f) return 0u;
            int q = __float2int_rn(__fdiv_rn(__fsub_rn(x, bias), s));
            q = q > 15 ? 15 : (q < 0 ? 0 : q);
            return static_cast<uint32_t>(q);
        };
        if (valid) {
            const uint32_t lo = code(v.x) | (code(v.y) << 4);
            const uint32_t hi = code(v.z) | (code(v.w) << 4);
            reinterpret_cast<uint16_t*>(codes + g * 32)[sub] = static_cast<uint16_t>(lo | (hi << 8));
            if (sub == 0) {
                scales[g] = s16;
                biases[g] = b16;
            }
        }
    }
}

int64_t grid_for(int64_t units_per_warp_iter, int64_t total_units, int num_sms) {
    const int64_t warps_needed = (total_units + units_per_warp_iter - 1) / units_per_warp_iter;
    int64_t grid = (warps_needed * 32 + kThreads - 1) / kThreads;
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    return grid;
}

}  // namespace

qg_status launch_quantize_block32(const float* w, int64_t n, int64_t k, int8_t* codes,
                                  uint16_t* scales, cudaStream_t stream) {
    DeviceInfo dev;
    qg_status st = device_info(&dev);
    if (st != QG_OK) return st;
    const int64_t nblocks = n * (k / 32);
    const int64_t grid = grid_for(4, nblocks, dev.num_sms);
    quantize_block32_kernel<<<static_cast<unsigned>(grid), kThreads, 0, stream>>>(w, nblocks, codes,
                                                                                 scales);
    return cuda_status(cudaGetLastError());
}

qg_status launch_quantize_int4_g64(const float* w, int64_t n, int64_t k, uint8_t* codes,
                                   uint16_t* scales, uint16_t* biases, cudaStream_t stream) {
    DeviceInfo dev;
    qg_status st = device_info(&dev);
    if (st != QG_OK) return st;
    const int64_t ngroups = n * (k / 64);
    const int64_t grid = grid_for(2, ngroups, dev.num_sms);
    quantize_int4_kernel<<<static_cast<unsigned>(grid), kThreads, 0, stream>>>(w, ngroups, codes,
                                                                              scales, biases);
    return cuda_status(cudaGetLastError());
}

}  // namespace qg
