// bl_gemv_lut.cu -- decode BitLinear (M = 1) by table lookup instead of
// multiply-accumulate: the approach of the CPU inference engine the pages
// describe (aratech.ae, "How BitNet.cpp achieves its speed": a lookup-table
// kernel in the manner of T-MAC; devtrends.ru, "How does it work?": lookup
// tables instead of matrix multiplications), here as a GPU A/B counterpart
// of the dp4a and tensor-core decode kernels.  Same result, bit for bit.
//
// The packed fields are u = code + 1 in {0, 1, 2} (include/bitlinear.h),
// two bits: u = lo + 2 * hi.  So
//     sum_k code_k * q_k = sum_k lo_k q_k + 2 * sum_k hi_k q_k - sum_k q_k .
// Byte b of packed word wd of chunk c holds the fields of the four
// activations k_t = 64c + 16wd + 4t + b (t = 0..3): one "group".  For every
// group the kernel tabulates the 16 subset sums of its four activations,
// S[idx] = sum over the set bits t of idx of q_{k_t}; the lo bits of a
// packed byte (bits 0, 2, 4, 6) and its hi bits (1, 3, 5, 7), each squeezed
// into a 4-bit index, then look up sum_t lo_t q_t and sum_t hi_t q_t
// directly.  The tables take 32 bytes per group, 8 * Kp bytes in all, built
// once per CTA in shared memory.
//
// Work: each CTA owns a contiguous range of whole 8-row tiles; warps take
// 512-byte spans (16 bytes per lane, the streaming kernels' lane mapping)
// straight from global memory.  Per-lane sums go to shared per-row
// accumulators when the tile changes; the epilogue adds the two planes and
// rescales, y = (float)((double)acc * (double)gamma32 / (double)s).
#include "bl_internal.cuh"

namespace bl {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kLutSmemMax = 200 * 1024;   // tables + per-row accumulators

__device__ __forceinline__ uint4 ldg_stream(const void* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// bits 0, 2, 4, 6 of every byte -> bits 0..3 of that byte
__device__ __forceinline__ uint32_t squeeze(uint32_t v)
{
    v &= 0x55555555u;
    v = (v | (v >> 1)) & 0x33333333u;
    v = (v | (v >> 2)) & 0x0F0F0F0Fu;
    return v;
}

template <typename YT>
__device__ __forceinline__ void store_y(YT* y, int64_t i, float v);
template <>
__device__ __forceinline__ void store_y<float>(float* y, int64_t i, float v) { y[i] = v; }
template <>
__device__ __forceinline__ void store_y<__nv_bfloat16>(__nv_bfloat16* y, int64_t i, float v)
{
    y[i] = __float2bfloat16_rn(v);
}

template <typename YT>
__global__ void __launch_bounds__(kThreads)
lut_kernel(const int8_t* __restrict__ q, const float* __restrict__ s_in, const uint8_t* __restrict__ packed,
           const float* __restrict__ gamma32, int64_t N, int64_t K, int tiles_base, int tiles_extra,
           YT* __restrict__ y, int32_t* __restrict__ acc_out)
{
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ int red[kWarps];
    const int C = (int)chunks_per_row(K);
    const int Kp = C * 64;
    const int groups = Kp / 4;
    int16_t* tab = reinterpret_cast<int16_t*>(smem);                 // [groups][16]
    int* lo_acc = reinterpret_cast<int*>(smem + (size_t)groups * 32);  // [tiles * 8]
    const int ci = blockIdx.x;
    const int64_t t0 = (int64_t)ci * tiles_base + (ci < tiles_extra ? ci : tiles_extra);
    const int ntl = tiles_base + (ci < tiles_extra ? 1 : 0);
    int* hi_acc = lo_acc + ntl * 8;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- tables (and sum q): group g = 16c + 4wd + b, activations
    //      k_t = 64c + 16wd + 4t + b
    int part = 0;
    for (int g = threadIdx.x; g < groups; g += kThreads) {
        const int c = g >> 4, wd = (g >> 2) & 3, b = g & 3;
        const int kb = 64 * c + 16 * wd + b;
        const int a0 = q[kb], a1 = q[kb + 4], a2 = q[kb + 8], a3 = q[kb + 12];
        part += a0 + a1 + a2 + a3;
        int16_t e[16];
#pragma unroll
        for (int idx = 0; idx < 16; ++idx)
            e[idx] = (int16_t)(((idx & 1) ? a0 : 0) + ((idx & 2) ? a1 : 0) + ((idx & 4) ? a2 : 0) +
                               ((idx & 8) ? a3 : 0));
        uint4 w0, w1;
        w0.x = (uint16_t)e[0] | ((uint32_t)(uint16_t)e[1] << 16);
        w0.y = (uint16_t)e[2] | ((uint32_t)(uint16_t)e[3] << 16);
        w0.z = (uint16_t)e[4] | ((uint32_t)(uint16_t)e[5] << 16);
        w0.w = (uint16_t)e[6] | ((uint32_t)(uint16_t)e[7] << 16);
        w1.x = (uint16_t)e[8] | ((uint32_t)(uint16_t)e[9] << 16);
        w1.y = (uint16_t)e[10] | ((uint32_t)(uint16_t)e[11] << 16);
        w1.z = (uint16_t)e[12] | ((uint32_t)(uint16_t)e[13] << 16);
        w1.w = (uint16_t)e[14] | ((uint32_t)(uint16_t)e[15] << 16);
        reinterpret_cast<uint4*>(tab + g * 16)[0] = w0;
        reinterpret_cast<uint4*>(tab + g * 16)[1] = w1;
    }
    for (int i = threadIdx.x; i < ntl * 16; i += kThreads) lo_acc[i] = 0;   // lo_acc and hi_acc
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) red[warp] = part;
    __syncthreads();
    int sumq = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) sumq += red[w];

    // ---- spans: lane = (chunk sub, row r); span g of tile t covers chunks
    //      4g .. 4g + 3 of the tile's 8 rows
    const int spt = (C + 3) / 4;                 // spans per tile (the last may be short)
    const int r = lane & 7, sub = lane >> 3;
    const uint8_t* base = packed + t0 * (int64_t)C * 128;
    int cur = -1, slo = 0, shi = 0;
    for (int sp = warp; sp < ntl * spt; sp += kWarps) {
        const int tile = sp / spt, gin = sp - tile * spt;
        const int c = 4 * gin + sub;
        if (tile != cur) {
            if (cur >= 0) {
                atomicAdd(&lo_acc[cur * 8 + r], slo);
                atomicAdd(&hi_acc[cur * 8 + r], shi);
            }
            cur = tile;
            slo = shi = 0;
        }
        if (c < C) {
            const uint4 wv = ldg_stream(base + ((int64_t)tile * C + c) * 128 + r * 16);
            const uint32_t w[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
                const uint32_t lo = squeeze(w[wd]), hi = squeeze(w[wd] >> 1);
                const int16_t* tg = tab + (16 * c + 4 * wd) * 16;   // group of byte 0
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    slo += tg[b * 16 + ((lo >> (8 * b)) & 15)];
                    shi += tg[b * 16 + ((hi >> (8 * b)) & 15)];
                }
            }
        }
    }
    if (cur >= 0) {
        atomicAdd(&lo_acc[cur * 8 + r], slo);
        atomicAdd(&hi_acc[cur * 8 + r], shi);
    }
    __syncthreads();

    // ---- epilogue
    const double g = (double)*gamma32;
    const double s = (double)*s_in;
    for (int i = threadIdx.x; i < ntl * 8; i += kThreads) {
        const int64_t n = t0 * 8 + i;
        if (n < N) {
            const int a = lo_acc[i] + 2 * hi_acc[i] - sumq;
            if (acc_out) acc_out[n] = a;
            store_y(y, n, (float)((double)a * g / s));
        }
    }
}

}  // namespace

bool lut_supported(int64_t M, int64_t K)
{
    if (M != 1) return false;
    return padded_k(K) * 8 + 4096 <= kLutSmemMax;
}

cudaError_t launch_lut(const int8_t* q, const float* s, const uint8_t* packed, const float* gamma32, int64_t N,
                       int64_t K, void* y, bl_dtype yt, int32_t* acc, cudaStream_t st)
{
    const int64_t tiles = padded_n(N) / 8;
    int grid = 2 * sm_count();
    if (grid > tiles) grid = (int)tiles;
    const int base = (int)(tiles / grid), extra = (int)(tiles % grid);
    const int per = base + (extra ? 1 : 0);
    const size_t smem = (size_t)padded_k(K) * 8 + (size_t)per * 16 * 4;
    if (smem > (size_t)kLutSmemMax) return cudaErrorNotSupported;
    if (yt == BL_F32) {
        cudaError_t e = cudaFuncSetAttribute(lut_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kLutSmemMax);
        if (e != cudaSuccess) return e;
        lut_kernel<float><<<grid, kThreads, smem, st>>>(q, s, packed, gamma32, N, K, base, extra,
                                                        static_cast<float*>(y), acc);
    } else {
        cudaError_t e = cudaFuncSetAttribute(lut_kernel<__nv_bfloat16>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kLutSmemMax);
        if (e != cudaSuccess) return e;
        lut_kernel<__nv_bfloat16><<<grid, kThreads, smem, st>>>(q, s, packed, gamma32, N, K, base, extra,
                                                                static_cast<__nv_bfloat16*>(y), acc);
    }
    return cudaGetLastError();
}

}  // namespace bl
