// bl_pack.cu -- absmean ternary quantisation of a weight tensor and the
// 2-bit packed layout (BitNet b1.58, aratech.ae "Ternary weights {-1, 0, +1}":
// scale = 1/mean|W|, W_q = clip(-1, 1)(round(W * scale)); 2 bits per weight
// as in bhfrc.com/news/56965 sec. 4.1, stored as code + 1 -- see
// include/bitlinear.h).
//
// Three launches, all HBM-bound streaming passes:
//   1. absmean_partial: each block sums |W| over a fixed grid-stride slice
//      in fp64 and writes one partial (fixed block count and fixed tree
//      order, so gamma is deterministic run to run).  Plain cached loads, so
//      a tensor that fits in L2 is still there for pass 3.
//   2. absmean_finalize: one block sums the partials in fixed order ->
//      gamma64, gamma32 = (float)gamma64, and the code threshold.
//   3. pack: one thread per (8-row tile, 64-weight chunk, row) writes the
//      16 packed bytes of that chunk; consecutive threads write consecutive
//      16-byte pieces of the output.
//
// Code decision.  With d = gamma64 + eps (fp64), round-half-even of W/d
// clipped to [-1, 1] is non-zero exactly when |W|/d > 1/2, i.e. when the
// real number |W| exceeds d/2 (d/2 is exact in fp64).  For fp32 |W| that is
// the same as |W| > thr, thr = d/2 rounded DOWN to fp32, since no fp32 value
// lies in (thr, d/2].  So the kernel compares in fp32 against thr and the
// decision equals the exact fp64 one.  (A divide-then-round implementation
// can differ only where W/d rounds to exactly 0.5, inside the 1e-6 band.)
#include "bl_internal.cuh"

namespace bl {
namespace {

constexpr int kReduceThreads = 256;

__device__ __forceinline__ double block_sum_fixed(double v, double* smem)
{
    // warp tree (xor butterfly, fixed order), then warps summed in order.
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) smem[warp] = v;
    __syncthreads();
    double t = 0.0;
    if (threadIdx.x == 0)
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += smem[w];
    return t;   // valid in thread 0
}

__global__ void __launch_bounds__(kReduceThreads)
absmean_partial_kernel(const float* __restrict__ W, int64_t count, double* __restrict__ partial,
                       unsigned* status)
{
    __shared__ double red[kReduceThreads / 32];
    const int64_t nvec = count >> 2;
    const float4* W4 = reinterpret_cast<const float4*>(W);
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    double acc = 0.0;
    bool bad = false;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    // two independent 16-byte loads in flight per iteration
    for (; i + stride < nvec; i += 2 * stride) {
        const float4 a = W4[i];
        const float4 b = W4[i + stride];
        bad |= !(isfinite(a.x) && isfinite(a.y) && isfinite(a.z) && isfinite(a.w) &&
                 isfinite(b.x) && isfinite(b.y) && isfinite(b.z) && isfinite(b.w));
        acc += (double)fabsf(a.x) + (double)fabsf(a.y) + (double)fabsf(a.z) + (double)fabsf(a.w);
        acc += (double)fabsf(b.x) + (double)fabsf(b.y) + (double)fabsf(b.z) + (double)fabsf(b.w);
    }
    for (; i < nvec; i += stride) {
        const float4 a = W4[i];
        bad |= !(isfinite(a.x) && isfinite(a.y) && isfinite(a.z) && isfinite(a.w));
        acc += (double)fabsf(a.x) + (double)fabsf(a.y) + (double)fabsf(a.z) + (double)fabsf(a.w);
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        for (int64_t j = nvec << 2; j < count; ++j) {
            bad |= !isfinite(W[j]);
            acc += (double)fabsf(W[j]);
        }
    }
    if (bad) atomicOr(status, kStatusNonfiniteW);
    const double t = block_sum_fixed(acc, red);
    if (threadIdx.x == 0) partial[blockIdx.x] = t;
}

__global__ void __launch_bounds__(kReduceThreads)
absmean_finalize_kernel(const double* __restrict__ partial, int blocks, int64_t count, double eps,
                        double* gamma64, float* gamma32, float* thr)
{
    __shared__ double red[kReduceThreads / 32];
    double acc = 0.0;
    for (int i = threadIdx.x; i < blocks; i += blockDim.x) acc += partial[i];
    const double sum = block_sum_fixed(acc, red);
    if (threadIdx.x == 0) {
        const double g = sum / (double)count;
        *gamma64 = g;
        *gamma32 = __double2float_rn(g);
        const double d = g + eps;
        *thr = __double2float_rd(0.5 * d);
    }
}

// 2-bit value of one weight, code + 1: 10 for +1, 01 for 0, 00 for -1.
__device__ __forceinline__ uint32_t code_bits(float w, float thr)
{
    return (w > thr) ? 2u : ((w < -thr) ? 0u : 1u);
}

__global__ void __launch_bounds__(256)
pack_kernel(const float* __restrict__ W, int64_t N, int64_t K, int64_t total,
            const float* __restrict__ thr_p, uint8_t* __restrict__ packed)
{
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= total) return;
    const int64_t C = chunks_per_row(K);
    const int64_t tile = t / (C * 8);
    const int64_t rem = t - tile * C * 8;
    const int64_t c = rem >> 3;
    const int r = (int)(rem & 7);
    const int64_t n = tile * 8 + r;
    uint4 out;
    if (n >= N) {
        out = make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u);   // padding rows: 01
    } else {
        const float thr = *thr_p;
        const float* row = W + n * K;
        const int64_t k0 = c * 64;
        uint32_t word[4];
        if ((K & 3) == 0 && k0 + 64 <= K) {
            // full chunk, 16-byte aligned: float4 j covers k0 + 4j .. +3,
            // j = 4*word + field, component = byte.
            const float4* src = reinterpret_cast<const float4*>(row + k0);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t w = 0;
#pragma unroll
                for (int f = 0; f < 4; ++f) {
                    const float4 v = __ldcs(src + 4 * i + f);
                    w |= code_bits(v.x, thr) << (2 * f);
                    w |= code_bits(v.y, thr) << (8 + 2 * f);
                    w |= code_bits(v.z, thr) << (16 + 2 * f);
                    w |= code_bits(v.w, thr) << (24 + 2 * f);
                }
                word[i] = w;
            }
        } else {
#pragma unroll 1
            for (int i = 0; i < 4; ++i) {
                uint32_t w = 0;
                for (int f = 0; f < 4; ++f)
                    for (int b = 0; b < 4; ++b) {
                        const int64_t k = k0 + 16 * i + 4 * f + b;
                        const uint32_t bits = (k < K) ? code_bits(row[k], thr) : 1u;
                        w |= bits << (8 * b + 2 * f);
                    }
                word[i] = w;
            }
        }
        out = make_uint4(word[0], word[1], word[2], word[3]);
    }
    reinterpret_cast<uint4*>(packed)[t] = out;
}

}  // namespace

int absmean_blocks(int64_t count)
{
    // fixed for a given size: enough blocks to stream HBM, at most 2048
    int64_t b = (count / 4 + kReduceThreads * 8 - 1) / (kReduceThreads * 8);
    if (b < 1) b = 1;
    if (b > 2048) b = 2048;
    return (int)b;
}

cudaError_t launch_absmean_partial(const float* W, int64_t count, double* partial, int blocks,
                                   unsigned* status, cudaStream_t st)
{
    absmean_partial_kernel<<<blocks, kReduceThreads, 0, st>>>(W, count, partial, status);
    return cudaGetLastError();
}

cudaError_t launch_absmean_finalize(const double* partial, int blocks, int64_t count, double eps,
                                    double* gamma64, float* gamma32, float* thr, cudaStream_t st)
{
    absmean_finalize_kernel<<<1, kReduceThreads, 0, st>>>(partial, blocks, count, eps, gamma64,
                                                          gamma32, thr);
    return cudaGetLastError();
}

cudaError_t launch_pack(const float* W, int64_t N, int64_t K, const float* thr, uint8_t* packed,
                        cudaStream_t st)
{
    const int64_t total = padded_n(N) * chunks_per_row(K);   // 16-byte outputs
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    pack_kernel<<<(unsigned)blocks, threads, 0, st>>>(W, N, K, total, thr, packed);
    return cudaGetLastError();
}

}  // namespace bl
