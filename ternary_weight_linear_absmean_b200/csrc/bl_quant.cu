// bl_quant.cu -- per-token absmax int8 activation quantisation
// (BitNet b1.58, aratech.ae "BitLinear: the building block": activations are
// quantised to INT8 per token with absmax, the row's largest |x| landing on
// 127).
//
//   amax_m = max(max_k |x_mk|, 1e-5);  s_m = 127 / amax_m  (IEEE fp32 divide)
//   q_mk   = clamp(rint(x_mk * s_m), -127, 127)          (fp32 multiply)
//
// One block per token row: pass 1 reduces the max (order-independent, so
// exact), pass 2 re-reads the row (L1/L2 resident) and writes q with a
// zero-filled tail up to Kp = ceil(K/64)*64, the row stride the product
// kernels read with 16-byte loads.  Built without FMA contraction for this
// file's float math (-fmad=false) so x*s rounds exactly once.
#include "bl_internal.cuh"

namespace bl {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float load_x(const float* x, int64_t i) { return x[i]; }
__device__ __forceinline__ float load_x(const __nv_bfloat16* x, int64_t i)
{
    return __bfloat162float(x[i]);
}

__device__ __forceinline__ int8_t quant_one(float v, float s)
{
    float r = rintf(__fmul_rn(v, s));
    r = fminf(fmaxf(r, -127.0f), 127.0f);
    return (int8_t)(int)r;
}

template <typename XT>
__global__ void __launch_bounds__(kThreads)
quant_kernel(const XT* __restrict__ x, int64_t K, int64_t Kp, int8_t* __restrict__ q,
             float* __restrict__ s_out, unsigned* status)
{
    __shared__ float red[kThreads / 32];
    const int64_t m = blockIdx.x;
    const XT* row = x + m * K;
    int8_t* qrow = q + m * Kp;

    float amax = 0.0f;
    bool bad = false;
    for (int64_t k = threadIdx.x; k < K; k += kThreads) {
        const float v = load_x(row, k);
        bad |= !isfinite(v);
        amax = fmaxf(amax, fabsf(v));
    }
    if (bad) atomicOr(status, kStatusNonfiniteX);
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = red[0];
    for (int w = 1; w < kThreads / 32; ++w) amax = fmaxf(amax, red[w]);
    amax = fmaxf(amax, 1e-5f);
    const float s = 127.0f / amax;
    if (threadIdx.x == 0) s_out[m] = s;

    // pass 2: 4 consecutive codes per thread per step -> one 32-bit store
    for (int64_t k4 = (int64_t)threadIdx.x * 4; k4 < Kp; k4 += kThreads * 4) {
        uint32_t packed = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int64_t k = k4 + b;
            const int8_t v = (k < K) ? quant_one(load_x(row, k), s) : (int8_t)0;
            packed |= (uint32_t)(uint8_t)v << (8 * b);
        }
        *reinterpret_cast<uint32_t*>(qrow + k4) = packed;
    }
}

}  // namespace

cudaError_t launch_quant(const void* x, bl_dtype xt, int64_t M, int64_t K, int8_t* q, float* s,
                         unsigned* status, cudaStream_t st)
{
    const int64_t Kp = padded_k(K);
    if (xt == BL_F32)
        quant_kernel<float><<<(unsigned)M, kThreads, 0, st>>>(static_cast<const float*>(x), K, Kp, q,
                                                              s, status);
    else
        quant_kernel<__nv_bfloat16><<<(unsigned)M, kThreads, 0, st>>>(
            static_cast<const __nv_bfloat16*>(x), K, Kp, q, s, status);
    return cudaGetLastError();
}

}  // namespace bl
