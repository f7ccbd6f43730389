// bl_gemv.cu -- memory-bound decode kernel: packed ternary weights x int8
// activations -> int32 -> y = acc * gamma / s  (bhfrc.com/news/56965 sec. 1.1:
// a ternary weight adds, subtracts or skips an activation; aratech.ae
// "BitLinear: the building block" for the int8 per-token activations).
//
// Work decomposition.  One CTA (8 warps) owns one 8-row tile of one problem.
// In the packed layout a tile stores chunk c (64 weights) of its 8 rows as
// 128 contiguous bytes, so chunk group g (4 chunks x 8 rows) is a contiguous
// 512-byte span: warp w reads groups w, w+8, ... with lane l loading bytes
// [16l, 16l+16) of the span -- one fully coalesced 128-bit load per lane.
// Lane l works on row r = l % 8 and chunk 4g + l / 8.
//
// Decode.  A 32-bit word holds 16 codes (byte b, field t -> k = 16i+4t+b),
// each stored as u = code + 1 in {0, 1, 2} (padding 01 -> u = 1, code 0).
// Field t of every byte is w & (0x03030303 << 2t), i.e. 4^t * u; dp4a
// (unsigned x signed) with the 4 activations k = 16i+4t .. +3 gives
// 4^t * sum(u * q), accumulated in its own register a_t.  Finally
//     sum(code*q) = sum_t a_t / 4^t  -  sum_k q_k
// (all exact integer arithmetic; the shifts divide exact multiples).
//
// Epilogue: per-lane totals are reduced over the 4 lanes of a row (shuffle)
// and the 8 warps (shared memory, fixed order), then
//     y = (float)((double)acc * (double)gamma32 / (double)s_m)
// which is the oracle's rescale bit for bit.
//
// Fused form (FUSED): the CTA quantises its x rows into shared memory first
// (same arithmetic as bl_quant.cu), while an L2 bulk prefetch of its weight
// tile is in flight, so q and s never go through HBM.
#include "bl_internal.cuh"

namespace bl {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c)
{
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ int dp4a_ss(uint32_t a, uint32_t b, int c)
{
    int d;
    asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint4 ldg_stream(const void* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ float x_at(const float* x, int64_t i) { return x[i]; }
__device__ __forceinline__ float x_at(const __nv_bfloat16* x, int64_t i) { return __bfloat162float(x[i]); }

__device__ __forceinline__ void store_y(float* y, int64_t i, float v) { y[i] = v; }
__device__ __forceinline__ void store_y(__nv_bfloat16* y, int64_t i, float v) { y[i] = __float2bfloat16_rn(v); }

template <int G>
struct Batch {
    GemvProblem p[G];
    int count;
    int64_t M;
};

template <int MT, bool FUSED, typename XT, typename YT, int G>
__global__ void __launch_bounds__(kThreads)
gemv_kernel(const __grid_constant__ Batch<G> b, unsigned* status)
{
    extern __shared__ __align__(16) int8_t smem_q[];   // FUSED: [MT][Kp] int8
    __shared__ int red[kWarps][MT][8];
    __shared__ int sumq[MT];
    __shared__ float sc[MT];
    __shared__ float amax_red[kWarps];

    // ---- locate problem and tile
    int pi = 0;
#pragma unroll 1
    for (int i = 1; i < b.count; ++i)
        if ((int64_t)blockIdx.x >= b.p[i].tile_begin) pi = i;
    const GemvProblem& P = b.p[pi];
    const int64_t tile = (int64_t)blockIdx.x - P.tile_begin;
    const int64_t K = P.K, N = P.N;
    const int64_t Kp = padded_k(K);
    const int C = (int)(Kp / 64);
    const int groups = (C + 3) / 4;
    const uint8_t* tile_ptr = P.packed + tile * (int64_t)C * 128;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r = lane & 7, sub = lane >> 3;

    if (threadIdx.x == 0) prefetch_l2_bulk(tile_ptr, (uint32_t)(C * 128));
    const float g32 = *P.gamma32;

#pragma unroll 1
    for (int64_t m0 = 0; m0 < b.M; m0 += MT) {
        const int mcount = (int)((b.M - m0) < MT ? (b.M - m0) : MT);

        // ---- prologue: activations for tokens m0 .. m0+mcount-1
        if constexpr (FUSED) {
            const XT* xb = static_cast<const XT*>(P.x);
#pragma unroll 1
            for (int m = 0; m < mcount; ++m) {
                const XT* row = xb + (m0 + m) * K;
                float amax = 0.0f;
                bool bad = false;
                for (int64_t k = threadIdx.x; k < K; k += kThreads) {
                    const float v = x_at(row, k);
                    bad |= !isfinite(v);
                    amax = fmaxf(amax, fabsf(v));
                }
                if (bad) atomicOr(status, kStatusNonfiniteX);
                for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                if (lane == 0) amax_red[warp] = amax;
                __syncthreads();
                amax = amax_red[0];
#pragma unroll
                for (int w = 1; w < kWarps; ++w) amax = fmaxf(amax, amax_red[w]);
                amax = fmaxf(amax, 1e-5f);
                const float s = 127.0f / amax;
                int part = 0;
                int8_t* qrow = smem_q + (int64_t)m * Kp;
                for (int64_t k4 = (int64_t)threadIdx.x * 4; k4 < Kp; k4 += kThreads * 4) {
                    uint32_t word = 0;
#pragma unroll
                    for (int bb = 0; bb < 4; ++bb) {
                        const int64_t k = k4 + bb;
                        int v = 0;
                        if (k < K) {
                            float rr = rintf(__fmul_rn(x_at(row, k), s));
                            rr = fminf(fmaxf(rr, -127.0f), 127.0f);
                            v = (int)rr;
                        }
                        word |= (uint32_t)(uint8_t)(int8_t)v << (8 * bb);
                    }
                    *reinterpret_cast<uint32_t*>(qrow + k4) = word;
                    part = dp4a_ss(word, 0x01010101u, part);
                }
                for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
                __syncthreads();   // amax_red reuse below / red reuse
                if (lane == 0) red[warp][0][0] = part;
                __syncthreads();
                if (threadIdx.x == 0) {
                    int t = 0;
#pragma unroll
                    for (int w = 0; w < kWarps; ++w) t += red[w][0][0];
                    sumq[m] = t;
                    sc[m] = s;
                }
                __syncthreads();
            }
        } else {
            // unfused: s from memory, sum of q over the padded row
#pragma unroll 1
            for (int m = 0; m < mcount; ++m) {
                const uint32_t* qw = reinterpret_cast<const uint32_t*>(P.q + (m0 + m) * Kp);
                int part = 0;
                for (int64_t i = threadIdx.x; i < Kp / 4; i += kThreads) part = dp4a_ss(__ldg(qw + i), 0x01010101u, part);
                for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
                if (lane == 0) red[warp][0][0] = part;
                __syncthreads();
                if (threadIdx.x == 0) {
                    int t = 0;
#pragma unroll
                    for (int w = 0; w < kWarps; ++w) t += red[w][0][0];
                    sumq[m] = t;
                    sc[m] = P.s[m0 + m];
                }
                __syncthreads();
            }
        }

        // ---- main loop
        int acc[MT][4];
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int t = 0; t < 4; ++t) acc[m][t] = 0;

#pragma unroll 2
        for (int g = warp; g < groups; g += kWarps) {
            const int c = 4 * g + sub;
            if (c < C) {
                const uint4 wv = ldg_stream(tile_ptr + (int64_t)g * 512 + lane * 16);
                const uint32_t U[4] = {wv.x, wv.y, wv.z, wv.w};   // stored fields are u = code + 1
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < mcount) {
                        const uint4* arow;
                        if constexpr (FUSED)
                            arow = reinterpret_cast<const uint4*>(smem_q + (int64_t)m * Kp + (int64_t)c * 64);
                        else
                            arow = reinterpret_cast<const uint4*>(P.q + (m0 + m) * Kp + (int64_t)c * 64);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            uint4 a;
                            if constexpr (FUSED) a = arow[i];
                            else a = __ldg(arow + i);
                            acc[m][0] = dp4a_us(U[i] & 0x03030303u, a.x, acc[m][0]);
                            acc[m][1] = dp4a_us(U[i] & 0x0C0C0C0Cu, a.y, acc[m][1]);
                            acc[m][2] = dp4a_us(U[i] & 0x30303030u, a.z, acc[m][2]);
                            acc[m][3] = dp4a_us(U[i] & 0xC0C0C0C0u, a.w, acc[m][3]);
                        }
                    }
                }
            }
        }

        // ---- reduce: fields, 4 lanes of a row, 8 warps
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            int tot = acc[m][0] + (acc[m][1] >> 2) + (acc[m][2] >> 4) + (acc[m][3] >> 6);
            tot += __shfl_xor_sync(0xffffffffu, tot, 8);
            tot += __shfl_xor_sync(0xffffffffu, tot, 16);
            if (sub == 0) red[warp][m][r] = tot;
        }
        __syncthreads();
        if (threadIdx.x < MT * 8) {
            const int m = threadIdx.x >> 3, rr = threadIdx.x & 7;
            const int64_t n = tile * 8 + rr;
            if (m < mcount && n < N) {
                int t = 0;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) t += red[w][m][rr];
                const int a = t - sumq[m];
                const int64_t o = (m0 + m) * N + n;
                if (P.acc) P.acc[o] = a;
                const float yv = (float)((double)a * (double)g32 / (double)sc[m]);
                store_y(static_cast<YT*>(P.y), o, yv);
            }
        }
        __syncthreads();
    }
}

template <int MT, bool FUSED, typename XT, typename YT, int G>
cudaError_t launch_t(const GemvBatch& gb, unsigned* status, cudaStream_t st)
{
    Batch<G> b;
    int64_t tiles = 0;
    for (int i = 0; i < gb.count; ++i) {
        b.p[i] = gb.p[i];
        b.p[i].tile_begin = tiles;
        tiles += padded_n(gb.p[i].N) / 8;
    }
    b.count = gb.count;
    b.M = gb.M;
    size_t smem = 0;
    if (FUSED) {
        int64_t kmax = 0;
        for (int i = 0; i < gb.count; ++i) kmax = kmax > padded_k(gb.p[i].K) ? kmax : padded_k(gb.p[i].K);
        smem = (size_t)(MT * kmax);
        auto kfn = gemv_kernel<MT, FUSED, XT, YT, G>;
        cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    gemv_kernel<MT, FUSED, XT, YT, G><<<(unsigned)tiles, kThreads, smem, st>>>(b, status);
    return cudaGetLastError();
}

template <bool FUSED, typename XT, typename YT, int G>
cudaError_t launch_mt(const GemvBatch& b, unsigned* status, cudaStream_t st)
{
    if (b.M <= 1) return launch_t<1, FUSED, XT, YT, G>(b, status, st);
    if (b.M <= 2) return launch_t<2, FUSED, XT, YT, G>(b, status, st);
    if (b.M <= 4) return launch_t<4, FUSED, XT, YT, G>(b, status, st);
    if (b.M <= 8) return launch_t<8, FUSED, XT, YT, G>(b, status, st);
    return launch_t<16, FUSED, XT, YT, G>(b, status, st);
}

template <bool FUSED, typename XT, int G>
cudaError_t launch_y(const GemvBatch& b, bl_dtype yt, unsigned* status, cudaStream_t st)
{
    if (yt == BL_F32) return launch_mt<FUSED, XT, float, G>(b, status, st);
    return launch_mt<FUSED, XT, __nv_bfloat16, G>(b, status, st);
}

}  // namespace

cudaError_t launch_gemv(const GemvBatch& b, bool fused, bl_dtype xt, bl_dtype yt, unsigned* status,
                        cudaStream_t st)
{
    if (!fused) return launch_y<false, float, 1>(b, yt, status, st);
    if (b.count == 1) {
        if (xt == BL_F32) return launch_y<true, float, 1>(b, yt, status, st);
        return launch_y<true, __nv_bfloat16, 1>(b, yt, status, st);
    }
    if (xt == BL_F32) return launch_y<true, float, kMaxGroup>(b, yt, status, st);
    return launch_y<true, __nv_bfloat16, kMaxGroup>(b, yt, status, st);
}

}  // namespace bl
