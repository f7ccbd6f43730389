// bl_quant.cu -- per-token absmax int8 activation quantisation
// (BitNet b1.58, aratech.ae "BitLinear: the building block": activations are
// quantised to INT8 per token with absmax, the row's largest |x| landing on
// 127), optionally preceded by the sub-layer normalisation that the same
// section places before the quantiser (SubLN, read as RMS normalisation
// with a per-channel gain):
//
//   [norm]  ms = sum_k x_k^2 / K (fp64), r = fp32(1 / sqrt(ms + eps)),
//           x_k <- (x_k * r) * g_k        (fp32, rounded in that order)
//   amax_m = max(max_k |x_mk|, 1e-5);  s_m = 127 / amax_m  (IEEE fp32 divide)
//   q_mk   = clamp(rint(x_mk * s_m), -127, 127)          (fp32 multiply)
//
// One block per token row, over the rows of up to 16 problems (x, K, gain,
// q, s each) in one launch.  The row is read from memory once with 16-byte
// loads and kept in registers (up to 4 vectors per thread; longer rows are
// re-read from L2).  Two exact shortcuts: max |x| is an unsigned max over
// the bit patterns with the sign cleared (integer order is numeric order for
// non-negative IEEE values, and NaN/Inf sort above every finite value, so
// the same max flags non-finite input), and rint + clamp + convert is one
// round-to-nearest-even addition (rint_low_byte, bl_internal.cuh), since
// |x * s| < 127.5 for finite x.
// q rows have stride Kp = ceil(K/64)*64, zero-filled beyond K.  Built without
// FMA contraction (-fmad=false) so every product rounds exactly once.
#include "bl_internal.cuh"

namespace bl {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kKeep = 4;   // 16-byte vectors a thread keeps in registers

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d)
{
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

template <typename XT>
struct Vec;
template <>
struct Vec<float> {
    static constexpr int E = 4;
    __device__ static float get(const uint4& u, int i)
    {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        return __uint_as_float(w[i]);
    }
};
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int E = 8;
    __device__ static float get(const uint4& u, int i)
    {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        const uint32_t h = w[i >> 1];
        return __uint_as_float((i & 1) ? (h & 0xFFFF0000u) : (h << 16));
    }
};

__device__ __forceinline__ float load_x(const float* x, int64_t i) { return x[i]; }
__device__ __forceinline__ float load_x(const __nv_bfloat16* x, int64_t i) { return __bfloat162float(x[i]); }

template <typename T>
__device__ __forceinline__ T block_reduce_sum(T v, T* red)
{
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    T t = red[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) t += red[w];
    __syncthreads();
    return t;
}

__device__ __forceinline__ uint32_t block_reduce_max(uint32_t v, uint32_t* red)
{
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    uint32_t t = red[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) t = max(t, red[w]);
    __syncthreads();
    return t;
}

// A memory-bound kernel wants many warps per SM: bf16 rows without
// normalisation fit 8 blocks (64 warps, 32 registers per thread); the other
// forms need more registers and take 6 or 5 blocks without spilling.
template <typename XT, bool NORM>
__global__ void __launch_bounds__(kThreads, NORM ? 5 : sizeof(XT) == 2 ? 8 : 6)
quant_kernel(const __grid_constant__ QuantBatch b, unsigned* status)
{
    __shared__ double redd[kWarps];
    __shared__ uint32_t redu[kWarps];
    using V = Vec<XT>;
    constexpr int E = V::E;
    int pi = 0;
#pragma unroll 1
    for (int i = 1; i < b.count; ++i)
        if ((int)blockIdx.x >= b.row_begin[i]) pi = i;
    const QuantProblem& P = b.p[pi];
    const int64_t K = P.K, Kp = padded_k(P.K);
    const float* __restrict__ gain = P.gain;
    const double eps = b.eps;
    const int64_t m = (int64_t)blockIdx.x - P.row_begin;
    float* __restrict__ s_out = P.s;
    // Programmatic dependent launch: a kernel launched after this one may
    // start its own set-up now (it reads what this one writes only after
    // its griddepcontrol.wait); this one reads nothing before its own wait.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const XT* row = static_cast<const XT*>(P.x) + m * K;
    int8_t* qrow = P.q + m * Kp;
    const int t = threadIdx.x;
    const bool vec = (K % E) == 0;
    const int64_t nv = K / E;
    const bool held = vec && nv <= (int64_t)kKeep * kThreads;
    const uint4* rv = reinterpret_cast<const uint4*>(row);

    uint4 keep[kKeep];
    if (held) {
#pragma unroll
        for (int j = 0; j < kKeep; ++j) {
            const int64_t v = t + (int64_t)j * kThreads;
            keep[j] = v < nv ? __ldg(rv + v) : make_uint4(0, 0, 0, 0);
        }
    }
    // calls f(vector, index) for each of this thread's 16-byte vectors, from
    // registers when the row is held (static indices: no local memory)
    auto each = [&](auto&& f) {
        if (held) {
#pragma unroll
            for (int j = 0; j < kKeep; ++j) {
                const int64_t v = t + (int64_t)j * kThreads;
                if (v < nv) f(keep[j], v);
            }
        } else {
            for (int64_t v = t; v < nv; v += kThreads) f(__ldg(rv + v), v);
        }
    };

    // ---- normalisation factor r32 (SubLN)
    float r32 = 1.0f;
    if constexpr (NORM) {
        double ss = 0.0;
        if (vec) {
            each([&](const uint4& u, int64_t) {
#pragma unroll
                for (int i = 0; i < E; ++i) {
                    const double d = (double)V::get(u, i);
                    ss += d * d;
                }
            });
        } else {
            for (int64_t k = t; k < K; k += kThreads) {
                const double d = (double)load_x(row, k);
                ss += d * d;
            }
        }
        ss = block_reduce_sum(ss, redd);
        r32 = (float)(1.0 / sqrt(ss / (double)K + eps));
    }
    auto xn = [&](float v, int64_t k) -> float {
        if constexpr (NORM) return __fmul_rn(__fmul_rn(v, r32), __ldg(gain + k));
        return v;
    };

    // ---- amax (bit patterns, sign cleared)
    uint32_t mb = 0;
    if (vec) {
        each([&](const uint4& u, int64_t v) {
#pragma unroll
            for (int i = 0; i < E; ++i) mb = max(mb, __float_as_uint(xn(V::get(u, i), v * E + i)) & 0x7FFFFFFFu);
        });
    } else {
        for (int64_t k = t; k < K; k += kThreads) mb = max(mb, __float_as_uint(xn(load_x(row, k), k)) & 0x7FFFFFFFu);
    }
    mb = block_reduce_max(mb, redu);
    if (mb >= 0x7F800000u && t == 0) atomicOr(status, kStatusNonfiniteX);
    const float amax = fmaxf(__uint_as_float(mb), 1e-5f);
    const float s = 127.0f / amax;
    if (t == 0) s_out[m] = s;

    // ---- codes: E per vector -> E/4 packed words
    if (vec) {
        each([&](const uint4& u, int64_t v) {
                uint32_t w[E / 4];
#pragma unroll
                for (int p = 0; p < E / 4; ++p) {
                    int c[4];
#pragma unroll
                    for (int b = 0; b < 4; ++b)
                        c[b] = (int)rint_low_byte(__fmul_rn(xn(V::get(u, 4 * p + b), v * E + 4 * p + b), s));
                    w[p] = pack4(c[0], c[1], c[2], c[3]);
                }
                if constexpr (E == 8)
                    *reinterpret_cast<uint2*>(qrow + v * 8) = make_uint2(w[0], w[1]);
                else
                    *reinterpret_cast<uint32_t*>(qrow + v * 4) = w[0];
        });
        for (int64_t k4 = K + 4 * (int64_t)t; k4 < Kp; k4 += 4 * kThreads) *reinterpret_cast<uint32_t*>(qrow + k4) = 0u;
    } else {
        for (int64_t k4 = (int64_t)t * 4; k4 < Kp; k4 += kThreads * 4) {
            int c[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int64_t k = k4 + b;
                c[b] = (k < K) ? (int)rint_low_byte(__fmul_rn(xn(load_x(row, k), k), s)) : 0;
            }
            *reinterpret_cast<uint32_t*>(qrow + k4) = pack4(c[0], c[1], c[2], c[3]);
        }
    }
}

template <typename XT, bool NORM>
cudaError_t launch_k(const QuantBatch& b, unsigned* status, cudaStream_t st)
{
    // launched with programmatic stream serialisation: the kernel waits
    // (griddepcontrol.wait) before it reads or writes anything
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)b.rows);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, quant_kernel<XT, NORM>, b, status);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <typename XT>
cudaError_t launch_typed(const QuantBatch& b, unsigned* status, cudaStream_t st)
{
    if (b.p[0].gain) return launch_k<XT, true>(b, status, st);
    return launch_k<XT, false>(b, status, st);
}

QuantBatch single(const void* x, const float* gain, double eps, int64_t M, int64_t K, int8_t* q, float* s)
{
    QuantBatch b = {};
    b.count = 1;
    b.rows = (int)M;
    b.eps = eps;
    b.p[0].x = x;
    b.p[0].gain = gain;
    b.p[0].q = q;
    b.p[0].s = s;
    b.p[0].K = K;
    b.p[0].row_begin = 0;
    b.row_begin[0] = 0;
    return b;
}

}  // namespace

cudaError_t launch_quant(const void* x, bl_dtype xt, int64_t M, int64_t K, int8_t* q, float* s,
                         unsigned* status, cudaStream_t st)
{
    return launch_quant_grouped(single(x, nullptr, 0.0, M, K, q, s), xt, status, st);
}

cudaError_t launch_rmsnorm_quant(const void* x, bl_dtype xt, const float* gain, double eps, int64_t M, int64_t K,
                                 int8_t* q, float* s, unsigned* status, cudaStream_t st)
{
    return launch_quant_grouped(single(x, gain, eps, M, K, q, s), xt, status, st);
}

// Every problem of a batch either has a gain (SubLN) or none.
cudaError_t launch_quant_grouped(const QuantBatch& b, bl_dtype xt, unsigned* status, cudaStream_t st)
{
    if (b.rows <= 0) return cudaSuccess;
    if (xt == BL_F32) return launch_typed<float>(b, status, st);
    return launch_typed<__nv_bfloat16>(b, status, st);
}

}  // namespace bl
