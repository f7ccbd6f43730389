// bl_quant_rows.cuh -- the activation quantiser for several token rows at
// once, for the prologues of the decode kernels (M > 1).
//
// Arithmetic per row as bl_quant.cu (aratech.ae "BitLinear: the building
// block": per-token absmax int8, optionally after the SubLN read as RMS
// normalisation with a gain):
//   [norm]  r = fp32(1 / sqrt(sum x^2 / K + eps)) (sum in fp64), x <- (x*r)*g
//   s = 127 / max(max |x|, 1e-5),  q = rint(x * s)   (|x * s| < 127.5)
//
// All rows advance together: each thread walks its 16-byte vectors with the
// rows as the inner (unrolled) loop, so the loads of every row are in flight
// at once, and per-row partials meet in shared memory once per phase --
// max |x| and sum q through integer atomics (exact, order-free), the fp64
// sums of squares through a per-warp array added in a fixed order.  A row
// loop with barriers inside would pay a full load latency per row.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "bl_internal.cuh"
#include "bl_ptx.cuh"

namespace bl {

struct QuantRowsShared {
    uint32_t amax[16];     // bit patterns of max |x| per row
    int sumq[16];
    float r[16];           // SubLN factors
};

// XT: float or bf16.  NT threads take part (tid in [0, NT)); sync() is a
// barrier over exactly those threads.  store(m, kw, word) receives the int8x4
// word of token m for k = 4kw .. 4kw + 3 (kw < ceil(K/4); words past K are
// zero-padded).  ss_part: NT/32 * 16 doubles of shared scratch (NORM only).
// On return threads tid < M have written s_out[tid] and sumq_out[tid] (the
// row's scale and sum of q); the caller's next barrier publishes them.
template <int MT, int NT, typename XT, bool NORM, typename Store, typename Sync>
__device__ __forceinline__ void quantise_rows(const XT* __restrict__ x, int M, int K, const float* __restrict__ gain,
                                              double eps, int tid, QuantRowsShared& sh, double* ss_part,
                                              float* s_out, int* sumq_out, Store&& store, Sync&& sync,
                                              unsigned* status)
{
    static_assert(MT <= 16, "at most 16 token rows");
    constexpr bool BF16 = sizeof(XT) == 2;
    constexpr int VE = 16 / sizeof(XT);   // elements per 16-byte vector
    const int lane = tid & 31, wid = tid >> 5;
    const bool vec = (K % VE) == 0;
    const int nv = K / VE;
    // element i of a vector as fp32 (bf16 widening is exact)
    auto elem = [&](const uint4& u, int i) -> float {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        if constexpr (BF16) return __uint_as_float((i & 1) ? (w[i >> 1] & 0xFFFF0000u) : (w[i >> 1] << 16));
        return __uint_as_float(w[i]);
    };
    auto xval = [&](int m, int k) -> float {
        if constexpr (BF16) return __bfloat162float(x[(int64_t)m * K + k]);
        return x[(int64_t)m * K + k];
    };
    const uint4* rv = reinterpret_cast<const uint4*>(x);   // row m, vector v: rv[m * nv + v] when vec
    // vector v of every row, all loads issued before any is used
    auto load_rows = [&](int v, uint4 (&u)[MT]) {
#pragma unroll
        for (int m = 0; m < MT; ++m)
            if (m < M) u[m] = __ldg(rv + (int64_t)m * nv + v);
    };
    // the gains of vector v (VE floats, 16-byte aligned), loaded together
    auto gains_of = [&](int v, float (&g)[VE]) {
        const float4* gp = reinterpret_cast<const float4*>(gain) + v * (VE / 4);
#pragma unroll
        for (int p = 0; p < VE / 4; ++p) {
            const float4 f = __ldg(gp + p);
            g[4 * p] = f.x;
            g[4 * p + 1] = f.y;
            g[4 * p + 2] = f.z;
            g[4 * p + 3] = f.w;
        }
    };

    if (tid < 16) {
        sh.amax[tid] = 0u;
        sh.sumq[tid] = 0;
    }
    sync();

    // ---- SubLN factors
    float r[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) r[m] = 1.0f;
    if constexpr (NORM) {
        double ss[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) ss[m] = 0.0;
        if (vec) {
            for (int v = tid; v < nv; v += NT) {
                uint4 u[MT];
                load_rows(v, u);
#pragma unroll
                for (int m = 0; m < MT; ++m)
                    if (m < M) {
#pragma unroll
                        for (int i = 0; i < VE; ++i) {
                            const double d = (double)elem(u[m], i);
                            ss[m] += d * d;
                        }
                    }
            }
        } else {
            for (int k = tid; k < K; k += NT) {
#pragma unroll
                for (int m = 0; m < MT; ++m)
                    if (m < M) {
                        const double d = (double)xval(m, k);
                        ss[m] += d * d;
                    }
            }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            double v = ss[m];
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) ss_part[wid * 16 + m] = v;
        }
        sync();
        if (tid < M) {
            double t = 0.0;   // fixed order over the warps
            for (int w = 0; w < NT / 32; ++w) t += ss_part[w * 16 + tid];
            sh.r[tid] = (float)(1.0 / sqrt(t / (double)K + eps));
        }
        sync();
#pragma unroll
        for (int m = 0; m < MT; ++m)
            if (m < M) r[m] = sh.r[m];
    }
    auto xn = [&](float v, int m, int k) -> float {
        if constexpr (NORM) return __fmul_rn(__fmul_rn(v, r[m]), __ldg(gain + k));
        return v;
    };

    // ---- max |x| per row: unsigned max of the bit patterns, sign cleared
    uint32_t mb[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) mb[m] = 0u;
    if (vec) {
        for (int v = tid; v < nv; v += NT) {
            uint4 u[MT];
            load_rows(v, u);
            float g[VE];
            if constexpr (NORM) gains_of(v, g);
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m < M) {
#pragma unroll
                    for (int i = 0; i < VE; ++i) {
                        float e = elem(u[m], i);
                        if constexpr (NORM) e = __fmul_rn(__fmul_rn(e, r[m]), g[i]);
                        mb[m] = max(mb[m], __float_as_uint(e) & 0x7FFFFFFFu);
                    }
                }
        }
    } else {
        for (int k = tid; k < K; k += NT) {
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m < M) mb[m] = max(mb[m], __float_as_uint(xn(xval(m, k), m, k)) & 0x7FFFFFFFu);
        }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        uint32_t v = mb[m];
        for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0 && m < M) atomicMax(&sh.amax[m], v);
    }
    sync();
    // lane m of every warp divides for row m; the others take it by shuffle
    // (one IEEE divide per thread rather than one per row)
    float s[MT];
    {
        const uint32_t bits = (lane < M) ? sh.amax[lane & 15] : 0u;
        if (bits >= 0x7F800000u && tid < M) atomicOr(status, kStatusNonfiniteX);
        const float mine = 127.0f / fmaxf(__uint_as_float(bits), 1e-5f);
#pragma unroll
        for (int m = 0; m < MT; ++m) s[m] = __shfl_sync(0xffffffffu, mine, m);
    }

    // ---- codes (rint_low_byte: |x * s| < 127.5)
    //      and sum q per row
    int part[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) part[m] = 0;
    if (vec) {
        for (int v = tid; v < nv; v += NT) {
            uint4 u[MT];
            load_rows(v, u);
            float g[VE];
            if constexpr (NORM) gains_of(v, g);
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m < M) {
#pragma unroll
                    for (int p = 0; p < VE / 4; ++p) {
                        int c[4];
#pragma unroll
                        for (int b = 0; b < 4; ++b) {
                            float e = elem(u[m], 4 * p + b);
                            if constexpr (NORM) e = __fmul_rn(__fmul_rn(e, r[m]), g[4 * p + b]);
                            c[b] = (int)rint_low_byte(__fmul_rn(e, s[m]));
                        }
                        const uint32_t word = __byte_perm(__byte_perm(c[0], c[1], 0x0040),
                                                          __byte_perm(c[2], c[3], 0x0040), 0x5410);
                        part[m] = dp4a_ss(word, 0x01010101u, part[m]);
                        store(m, v * (VE / 4) + p, word);
                    }
                }
        }
    } else {
        for (int kw = tid; kw < (K + 3) / 4; kw += NT) {
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m < M) {
                    int c[4];
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        const int k = 4 * kw + b;
                        c[b] = (k < K) ? (int)rint_low_byte(__fmul_rn(xn(xval(m, k), m, k), s[m])) : 0;
                    }
                    const uint32_t word = __byte_perm(__byte_perm(c[0], c[1], 0x0040),
                                                      __byte_perm(c[2], c[3], 0x0040), 0x5410);
                    part[m] = dp4a_ss(word, 0x01010101u, part[m]);
                    store(m, kw, word);
                }
        }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        int v = part[m];
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && m < M) atomicAdd(&sh.sumq[m], v);
    }
    sync();
    if (tid < M) {
        float mine = s[0];
#pragma unroll
        for (int m = 1; m < MT; ++m)
            if (tid == m) mine = s[m];
        s_out[tid] = mine;
        sumq_out[tid] = sh.sumq[tid];
    }
}

// The unfused form's counterpart: copy q rows (int8 [M][Kp], 16-byte rows)
// into the kernel's layout through store(m, kw, word) and sum each row;
// thread tid < M writes sumq_out[tid].
template <int MT, int NT, typename Store, typename Sync>
__device__ __forceinline__ void copy_q_rows(const int8_t* __restrict__ q, int M, int Kp, int tid, QuantRowsShared& sh,
                                            int* sumq_out, Store&& store, Sync&& sync)
{
    const int lane = tid & 31;
    if (tid < 16) sh.sumq[tid] = 0;
    sync();
    const uint4* gq = reinterpret_cast<const uint4*>(q);
    const int nv = Kp / 16;
    int part[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) part[m] = 0;
    for (int v = tid; v < nv; v += NT) {
        uint4 u[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m)
            if (m < M) u[m] = __ldg(gq + (int64_t)m * nv + v);
#pragma unroll
        for (int m = 0; m < MT; ++m)
            if (m < M) {
                const uint32_t w[4] = {u[m].x, u[m].y, u[m].z, u[m].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    part[m] = dp4a_ss(w[i], 0x01010101u, part[m]);
                    store(m, 4 * v + i, w[i]);
                }
            }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        int v = part[m];
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && m < M) atomicAdd(&sh.sumq[m], v);
    }
    sync();
    if (tid < M) sumq_out[tid] = sh.sumq[tid];
}

}  // namespace bl
