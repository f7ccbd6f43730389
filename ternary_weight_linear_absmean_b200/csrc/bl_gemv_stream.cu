// bl_gemv_stream.cu -- persistent, HBM-streaming decode kernel (M <= 16):
// packed ternary weights x int8 activations -> int32 -> y = acc * gamma / s
// (bhfrc.com/news/56965 sec. 1.1: a ternary weight adds, subtracts or skips
// an activation; aratech.ae "BitLinear: the building block" for the int8
// per-token activations).
//
// Launch: 4 CTAs per SM (up to 4 tokens; 2 above), with programmatic
// dependent launch.  CTAs are shared out among the problems of the launch so
// that the largest per-CTA share of whole tiles is as small as possible
// (assign_ctas), and each CTA owns a contiguous range of whole 8-row tiles of
// one problem -- in the packed layout that is one contiguous byte range.
//
// Inside a CTA (8 warps):
//   warp 0, lane 0  producer (long ranges): streams the range into a ring of
//                   16 KiB shared-memory stages with 1-D bulk copies
//                   (cp.async.bulk), one mbarrier pair (full/empty) per
//                   stage; it issues its first copies only after the
//                   consumers have issued their activation loads.
//   warps 1..7      consumers: first quantise x into shared memory (fused
//                   form, optionally with SubLN) or copy q there; then take
//                   512-byte spans (4 chunks x 8 rows of a tile) round-robin,
//                   lane l reading 16 bytes, row r = l % 8, and accumulate
//                   with dp4a (decode as in bl_gemv.cu).  Short ranges
//                   (<= 128 KiB) skip the ring: the consumers read their
//                   spans straight from global memory, four in flight per
//                   lane.  Per-lane partial sums are added into a per-(tile,
//                   row, token) int32 array in shared memory (integer adds:
//                   exact and order-independent) whenever the lane's tile
//                   changes.
//   epilogue        y = (float)((double)acc * (double)gamma32 / (double)s_m),
//                   bit-identical to the oracle's rescale.
#include "bl_internal.cuh"
#include "bl_ptx.cuh"
#include "bl_quant_rows.cuh"

namespace bl {
namespace {

constexpr int kThreads = 256;
constexpr int kConsumerWarps = 7;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kStageBytes = 16384;
constexpr uint32_t kDirectMaxBytes = 128 * 1024;   // per-CTA range up to which the consumers load directly
constexpr int kSpan = 512;

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ void store_y(float* y, int64_t i, float v) { y[i] = v; }
__device__ __forceinline__ void store_y(__nv_bfloat16* y, int64_t i, float v) { y[i] = __float2bfloat16_rn(v); }

// sum over the 224 consumer threads (named barrier 1); fixed order
__device__ __forceinline__ double consumers_sum_f64(double v, double* red)
{
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int cw = (threadIdx.x >> 5) - 1;
    if ((threadIdx.x & 31) == 0) red[cw] = v;
    named_bar(1, kConsumers);
    double t = red[0];
#pragma unroll
    for (int w = 1; w < kConsumerWarps; ++w) t += red[w];
    named_bar(1, kConsumers);   // red is reused right after
    return t;
}

__device__ __forceinline__ int consumers_sum(int v, int* red)
{
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int cw = (threadIdx.x >> 5) - 1;
    if ((threadIdx.x & 31) == 0) red[cw] = v;
    named_bar(1, kConsumers);
    int t = 0;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) t += red[w];
    return t;
}

__device__ __forceinline__ int consumers_max_int(int v, int* red)
{
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int cw = (threadIdx.x >> 5) - 1;
    if ((threadIdx.x & 31) == 0) red[cw] = v;
    named_bar(1, kConsumers);
    int m = red[0];
#pragma unroll
    for (int w = 1; w < kConsumerWarps; ++w) m = max(m, red[w]);
    named_bar(1, kConsumers);   // red is reused right after
    return m;
}

// four int32 codes in [-127, 127] -> one packed int8x4 word
__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d)
{
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Quantise x row (K elements) into q (Kp bytes) in shared memory; returns s.
// Same arithmetic as bl_quant.cu: with a gain vector (SubLN), first
// ms = sum x^2 / K in fp64, r = fp32(1 / sqrt(ms + eps)) and x <- (x * r) * g
// in fp32; then amax over the row, s = 127 / max(amax, 1e-5) (IEEE divide),
// q = clamp(rint(x * s), -127, 127) in fp32.  Two exact shortcuts: (1)
// max|x| is taken as an unsigned max over the bit patterns with the sign
// cleared -- for non-negative IEEE values integer order is numeric order,
// and NaN/Inf patterns sort above every finite value, so the same max also
// flags non-finite input; (2) rint + clamp + convert is one
// round-to-nearest-even addition (rint_low_byte), since |x * s| < 127.5 for finite x (the
// clamp can never bind).
template <typename XT, bool NORM>
__device__ float quantise_row(const XT* __restrict__ row, int K, int Kp, int8_t* q, int* redi, double* redd,
                              const float* __restrict__ gain, double eps, int* sumq_out, unsigned* status,
                              bool signal_loads)
{
    const int t = threadIdx.x - 32;
    constexpr bool BF16 = sizeof(XT) == 2;
    constexpr int VE = 16 / sizeof(XT);   // elements per 16-byte vector
    constexpr int VR = 4;                 // vectors a thread keeps in registers
    const int nv = K / VE;
    const bool vec = (K % VE) == 0;
    const bool held = vec && nv <= VR * kConsumers;   // later passes need no reload
    uint4 keep[VR];
    const uint4* rv = reinterpret_cast<const uint4*>(row);
    if (held) {
#pragma unroll
        for (int j = 0; j < VR; ++j) {
            const int v = t + j * kConsumers;
            keep[j] = v < nv ? __ldg(rv + v) : make_uint4(0, 0, 0, 0);
        }
    }
    // the loads above are issued: the producer may now queue the weight copies
    if (signal_loads) named_bar_arrive(4, kThreads);
    // f(vector, index) for each of this thread's vectors (static indices
    // into keep[]: no local memory)
    auto each = [&](auto&& f) {
        if (held) {
#pragma unroll
            for (int j = 0; j < VR; ++j) {
                const int v = t + j * kConsumers;
                if (v < nv) f(keep[j], v);
            }
        } else {
            for (int v = t; v < nv; v += kConsumers) f(__ldg(rv + v), v);
        }
    };
    // element i of a vector as fp32 (bf16 widening is exact)
    auto elem = [&](const uint4& u, int i) -> float {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        if constexpr (BF16) return __uint_as_float((i & 1) ? (w[i >> 1] & 0xFFFF0000u) : (w[i >> 1] << 16));
        return __uint_as_float(w[i]);
    };

    float r32 = 1.0f;
    if constexpr (NORM) {
        double ss = 0.0;
        if (vec) {
            each([&](const uint4& u, int) {
#pragma unroll
                for (int i = 0; i < VE; ++i) {
                    const double d = (double)elem(u, i);
                    ss += d * d;
                }
            });
        } else {
            for (int k = t; k < K; k += kConsumers) {
                const double d = (double)to_f(row[k]);
                ss += d * d;
            }
        }
        ss = consumers_sum_f64(ss, redd);
        r32 = (float)(1.0 / sqrt(ss / (double)K + eps));
    }
    auto xn = [&](float v, int k) -> float {
        if constexpr (NORM) return __fmul_rn(__fmul_rn(v, r32), __ldg(gain + k));
        return v;
    };
    // the gains of vector v (E floats, 16-byte aligned), loaded together
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

    uint32_t mbits = 0;
    if (vec) {
        each([&](const uint4& u, int v) {
            if constexpr (!NORM) {
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if constexpr (BF16) {
                        mbits = max(mbits, w[i] & 0x7FFF0000u);
                        mbits = max(mbits, (w[i] << 16) & 0x7FFF0000u);
                    } else {
                        mbits = max(mbits, w[i] & 0x7FFFFFFFu);
                    }
                }
            } else {
                float g[VE];
                gains_of(v, g);
#pragma unroll
                for (int i = 0; i < VE; ++i)
                    mbits = max(mbits, __float_as_uint(__fmul_rn(__fmul_rn(elem(u, i), r32), g[i])) & 0x7FFFFFFFu);
            }
        });
    } else {
        for (int k = t; k < K; k += kConsumers) mbits = max(mbits, __float_as_uint(xn(to_f(row[k]), k)) & 0x7FFFFFFFu);
    }
    mbits = (uint32_t)consumers_max_int((int)mbits, redi);
    if (mbits >= 0x7F800000u && t == 0) atomicOr(status, kStatusNonfiniteX);
    const float amax = fmaxf(__uint_as_float(mbits), 1e-5f);
    const float s = 127.0f / amax;
    int part = 0;
    if (vec) {
        each([&](const uint4& u, int v) {
            float g[VE];
            if constexpr (NORM) gains_of(v, g);
            uint32_t w[VE / 4];
#pragma unroll
            for (int p = 0; p < VE / 4; ++p) {
                int c[4];
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    float e = elem(u, 4 * p + b);
                    if constexpr (NORM) e = __fmul_rn(__fmul_rn(e, r32), g[4 * p + b]);
                    c[b] = (int)rint_low_byte(__fmul_rn(e, s));
                }
                w[p] = pack4(c[0], c[1], c[2], c[3]);
                part = dp4a_ss(w[p], 0x01010101u, part);
            }
            if constexpr (BF16)
                *reinterpret_cast<uint2*>(q + v * 8) = make_uint2(w[0], w[1]);
            else
                *reinterpret_cast<uint32_t*>(q + v * 4) = w[0];
        });
        for (int k4 = K + 4 * t; k4 < Kp; k4 += 4 * kConsumers) *reinterpret_cast<uint32_t*>(q + k4) = 0u;
    } else {
        for (int k4 = 4 * t; k4 < Kp; k4 += 4 * kConsumers) {
            int c[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int k = k4 + b;
                c[b] = (k < K) ? (int)rint_low_byte(__fmul_rn(xn(to_f(row[k]), k), s)) : 0;
            }
            const uint32_t word = pack4(c[0], c[1], c[2], c[3]);
            *reinterpret_cast<uint32_t*>(q + k4) = word;
            part = dp4a_ss(word, 0x01010101u, part);
        }
    }
    *sumq_out = consumers_sum(part, redi);
    return s;
}

// 16-byte streaming load that bypasses L1 (read once)
__device__ __forceinline__ uint4 ldg_stream(const void* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// One 16-byte chunk (64 weights of row r) against the activations of chunk
// c for every token slot; slots m >= M hold zero activations.
template <int MT>
__device__ __forceinline__ void dot_chunk(const uint4 wv, const int8_t* qs, int Kp, int c, int (&acc)[MT][4])
{
    const uint32_t U[4] = {wv.x, wv.y, wv.z, wv.w};   // stored fields are u = code + 1
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        {
            const uint4* a4 = reinterpret_cast<const uint4*>(qs + m * Kp + c * 64);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 a = a4[i];
                acc[m][0] = dp4a_us(U[i] & 0x03030303u, a.x, acc[m][0]);
                acc[m][1] = dp4a_us(U[i] & 0x0C0C0C0Cu, a.y, acc[m][1]);
                acc[m][2] = dp4a_us(U[i] & 0x30303030u, a.z, acc[m][2]);
                acc[m][3] = dp4a_us(U[i] & 0xC0C0C0C0u, a.w, acc[m][3]);
            }
        }
    }
}

template <int MT, bool FUSED, typename XT, typename YT, int MINB, bool NORM>
__global__ void __launch_bounds__(kThreads, MINB)
stream_kernel(const __grid_constant__ StreamBatch b, unsigned* status)
{
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t full_bar[kMaxStages], empty_bar[kMaxStages];
    __shared__ float s_scale[MT];
    __shared__ int s_sumq[MT];
    __shared__ double redd[kConsumerWarps];
    __shared__ int redi[kConsumerWarps];
    __shared__ int abort_flag;
    __shared__ QuantRowsShared qsh;
    __shared__ double ss_rows[NORM && MT > 1 ? kConsumerWarps * 16 : 1];

    // ---- which problem, which tiles (cheap: the CTA's first copy waits on it)
    int pi = 0;
#pragma unroll 1
    for (int i = 1; i < b.count; ++i)
        if ((int)blockIdx.x >= b.cta_begin[i]) pi = i;
    const StreamProblem& P = b.p[pi];
    const int K = (int)P.K, Kp = (int)padded_k(P.K);
    const int64_t N = P.N;
    const uint32_t TB = (uint32_t)(chunks_per_row(K) * 128);   // bytes per tile
    const int ci = (int)blockIdx.x - P.cta_begin;
    const int64_t t0 = (int64_t)ci * P.tiles_base + (ci < P.tiles_extra ? ci : P.tiles_extra);
    const int ntl = P.tiles_base + (ci < P.tiles_extra ? 1 : 0);
    const uint32_t range = (uint32_t)ntl * TB;                    // < 2^31 (host-checked)
    const uint8_t* src = P.packed + t0 * (int64_t)TB;
    const int stages = b.stages;
    const int npieces = (int)((range + kStageBytes - 1) / kStageBytes);

    uint8_t* ring = smem;
    int8_t* qs = reinterpret_cast<int8_t*>(smem + (size_t)stages * kStageBytes);
    int* sacc = reinterpret_cast<int*>(smem + (size_t)stages * kStageBytes + b.q_bytes);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // The producer initialises the barriers and puts the first `stages`
    // pieces in flight straight away; the consumers quantise x meanwhile and
    // the whole CTA meets at the __syncthreads below before anyone waits.
    const int first = npieces < stages ? npieces : stages;
    // Direct mode, for short ranges of whole-span tiles: the consumers read
    // the weights straight from global memory, several spans in flight per
    // lane, with no ring, copies or stage barriers.  Measured against the
    // ring on one B200: faster up to ~45 KB per CTA (2B block +1%, 7B +2-5%),
    // slower on the 100B layers (~360 KB per CTA, -7%), where 16 KiB bulk
    // copies with a deep ring stream better.
    const bool direct = (TB % kSpan) == 0 && range <= kDirectMaxBytes;
    // Let the next kernel in the stream start launching now; it waits for
    // this one to finish before it touches anything this one writes.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], kConsumerWarps);
        }
        abort_flag = 0;
        fence_barrier_init();
        // This grid may have started before the previous kernel finished
        // (programmatic dependent launch), so nothing it reads is safe to
        // read yet -- but an L2 prefetch is: it only warms the coherent L2,
        // and the copies below read after the wait.  Only the bytes of the
        // first copies: more would just evict each other on large layers.
        const uint32_t head = (uint32_t)first * kStageBytes < range ? (uint32_t)first * kStageBytes : range;
        for (uint32_t o = 0; o < head; o += kStageBytes)
            prefetch_l2_bulk(src + o, (head - o) < (uint32_t)kStageBytes ? (head - o) : (uint32_t)kStageBytes);
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (warp == 0) {
        // The consumers' first activation loads go out before the weight
        // copies: the row is small and on the critical path (quantisation
        // precedes every product), and behind ~50 KB of copies per CTA it
        // would wait its turn in the memory system.
        named_bar(4, kThreads);
        if (lane == 0 && !direct) {
            for (int j = 0; j < first; ++j) {
                const uint32_t left = range - (uint32_t)j * kStageBytes;
                const uint32_t len = left < (uint32_t)kStageBytes ? left : (uint32_t)kStageBytes;
                mbar_arrive_expect_tx(&full_bar[j], len);
                bulk_g2s(ring + (size_t)j * kStageBytes, src + (int64_t)j * kStageBytes, len, &full_bar[j]);
            }
        }
    }

    const int M = b.M;
    if (warp != 0) {
        // ------------------------------------------- consumers: prologue
        for (int i = threadIdx.x - 32; i < ntl * 8 * MT; i += kConsumers) sacc[i] = 0;
        const int tp = threadIdx.x - 32;
        auto store_q = [&](int m, int kw, uint32_t w) { *reinterpret_cast<uint32_t*>(qs + m * Kp + 4 * kw) = w; };
        auto sync_consumers = [&]() { named_bar(1, kConsumers); };
        if constexpr (FUSED && MT == 1) {
            int sq;
            const float s = quantise_row<XT, NORM>(static_cast<const XT*>(P.x), K, Kp, qs, redi, redd, P.gain,
                                                   b.eps_norm, &sq, status, true);
            if (tp == 0) {
                s_scale[0] = s;
                s_sumq[0] = sq;
            }
        } else if constexpr (FUSED) {
            // all rows at once; their loads go out ahead of the weight copies
            named_bar_arrive(4, kThreads);
            quantise_rows<MT, kConsumers, XT, NORM>(static_cast<const XT*>(P.x), M, K, P.gain, b.eps_norm, tp, qsh,
                                                    ss_rows, s_scale, s_sumq, store_q, sync_consumers, status);
            // words past K (the stores above stop at ceil(K/4))
            const int kw0 = (K + 3) / 4;
            for (int i = tp; i < M * (Kp / 4 - kw0); i += kConsumers)
                store_q(i / (Kp / 4 - kw0), kw0 + i % (Kp / 4 - kw0), 0u);
        } else {
            named_bar_arrive(4, kThreads);
            copy_q_rows<MT, kConsumers>(P.q, M, Kp, tp, qsh, s_sumq, store_q, sync_consumers);
            if (tp < M) s_scale[tp] = P.s[tp];
        }
        // token slots M .. MT-1 get zero activations, so the dot loop needs
        // no token guard (their sums are never written out)
        for (int i = threadIdx.x - 32; i < (MT - M) * Kp / 16; i += kConsumers)
            reinterpret_cast<uint4*>(qs + M * Kp)[i] = make_uint4(0, 0, 0, 0);
    }
    __syncthreads();

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (direct) return;
        if (lane == 0) {
            int issued = first;
            for (int j = first; j < npieces; ++j) {
                const int s = j % stages, round = j / stages;
                if (!wait_parity(&empty_bar[s], (round - 1) & 1, status, &abort_flag)) break;
                const uint32_t left = range - (uint32_t)j * kStageBytes;
                const uint32_t len = left < (uint32_t)kStageBytes ? left : (uint32_t)kStageBytes;
                mbar_arrive_expect_tx(&full_bar[s], len);
                bulk_g2s(ring + (size_t)s * kStageBytes, src + (int64_t)j * kStageBytes, len, &full_bar[s]);
                issued = j + 1;
            }
            // every copy this thread issued lands before it exits (the last
            // use of each stage is that stage's latest phase)
            for (int j = issued - stages < 0 ? 0 : issued - stages; j < issued; ++j)
                wait_parity(&full_bar[j % stages], (j / stages) & 1, status, nullptr, true);
        }
        return;
    }

    // ---------------------------------------------------- consumers: loop
    const int cw = warp - 1;

    const int r = lane & 7;
    const int sub = lane >> 3;
    int cur = -1;
    int acc[MT][4];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int t = 0; t < 4; ++t) acc[m][t] = 0;

    auto flush = [&]() {
        if (cur >= 0) {
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m < M) {
                    const int tot = acc[m][0] + (acc[m][1] >> 2) + (acc[m][2] >> 4) + (acc[m][3] >> 6);
                    atomicAdd(&sacc[(cur * 8 + r) * MT + m], tot);
                }
#pragma unroll
                for (int t = 0; t < 4; ++t) acc[m][t] = 0;
            }
        }
    };

    if (direct) {
        constexpr int U = 4;                               // spans in flight per lane
        const uint32_t nsp = range / kSpan;
        const uint32_t spt = TB / kSpan;
        const uint8_t* gp = src + (size_t)cw * kSpan + lane * 16;
        uint32_t tile = (uint32_t)cw / spt, gin = (uint32_t)cw - tile * spt;
#pragma unroll 1
        for (uint32_t sp = (uint32_t)cw; sp < nsp; sp += U * kConsumerWarps) {
            uint4 wv[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t spu = sp + u * kConsumerWarps;
                if (spu < nsp) wv[u] = ldg_stream(gp + (size_t)(spu - cw) * kSpan);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (sp + u * kConsumerWarps < nsp) {
                    if ((int)tile != cur) {
                        flush();
                        cur = (int)tile;
                    }
                    dot_chunk<MT>(wv[u], qs, Kp, (int)(4 * gin) + sub, acc);
                    gin += kConsumerWarps;
                    while (gin >= spt) {
                        gin -= spt;
                        ++tile;
                    }
                }
            }
        }
    } else {
    constexpr uint32_t kStep = kConsumerWarps * kSpan;   // bytes between a warp's spans
    const bool aligned = (TB % kSpan) == 0;
    const uint32_t spans_per_tile = TB / kSpan;
#pragma unroll 1
    for (int j = 0; j < npieces; ++j) {
        const int s = j % stages, round = j / stages;
        // Each consumer warp waits for the stage itself (try_wait suspends
        // the thread in hardware until the phase completes, and gives every
        // thread its own acquire of the data); no warp waits for the others.
        // The verdict is made warp-uniform; the only named barrier after
        // this loop is reached by every consumer warp exactly once.
        const bool ok = wait_parity(&full_bar[s], round & 1, status, &abort_flag);
        if (!__all_sync(0xffffffffu, ok) || abort_flag) break;
        const uint32_t poff = (uint32_t)j * kStageBytes;
        const uint32_t len = (range - poff) < (uint32_t)kStageBytes ? (range - poff) : (uint32_t)kStageBytes;
        const uint8_t* stage = ring + (size_t)s * kStageBytes;
        if (aligned) {
            // Tiles are whole 512-byte spans: a span lies in one tile, so the
            // tile index is the same for the whole warp and is tracked with
            // one division per stage.
            const uint32_t nsp = len / kSpan;
            uint32_t gsp = poff / kSpan + (uint32_t)cw;        // span index in the CTA range
            uint32_t tile = gsp / spans_per_tile;
            uint32_t gin = gsp - tile * spans_per_tile;       // chunk group within the tile
            const uint8_t* wp = stage + cw * kSpan + lane * 16;
            // two spans per trip: independent dot chains and half the loop
            // overhead (the tile check stays per span)
#pragma unroll 2
            for (uint32_t sp = (uint32_t)cw; sp < nsp; sp += kConsumerWarps, wp += kStep) {
                if ((int)tile != cur) {
                    flush();
                    cur = (int)tile;
                }
                dot_chunk<MT>(*reinterpret_cast<const uint4*>(wp), qs, Kp, (int)(4 * gin) + sub, acc);
                gin += kConsumerWarps;
                if (gin >= spans_per_tile) {
                    gin -= spans_per_tile;
                    ++tile;
                    if (gin >= spans_per_tile) {
                        tile += gin / spans_per_tile;
                        gin %= spans_per_tile;
                    }
                }
            }
        } else {
            // general case: a span may cross a tile boundary, so each lane
            // tracks its own tile (one division per stage, then incremental)
            uint32_t boff = (uint32_t)cw * kSpan + (uint32_t)lane * 16;
            uint32_t tile = (poff + boff) / TB;
            uint32_t within = (poff + boff) - tile * TB;
#pragma unroll 1
            for (uint32_t sb = (uint32_t)cw * kSpan; sb < len; sb += kStep, boff += kStep) {
                if (boff < len) {
                    if ((int)tile != cur) {
                        flush();
                        cur = (int)tile;
                    }
                    dot_chunk<MT>(*reinterpret_cast<const uint4*>(stage + boff), qs, Kp, (int)(within >> 7), acc);
                }
                within += kStep;
                if (within >= TB) {
                    if (TB >= kStep) {
                        within -= TB;
                        ++tile;
                    } else {
                        tile += within / TB;
                        within %= TB;
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[s]);
    }
    }
    flush();
    named_bar(1, kConsumers);
    if (abort_flag) return;

    // ---------------------------------------------------------- epilogue
    const float g32 = *P.gamma32;
    for (int i = threadIdx.x - 32; i < ntl * 8 * M; i += kConsumers) {
        const int m = i % M;
        const int row = i / M;                    // tile_local * 8 + r
        const int64_t n = t0 * 8 + row;
        if (n < N) {
            const int a = sacc[row * MT + m] - s_sumq[m];
            const int64_t o = (int64_t)m * N + n;
            if (P.acc) P.acc[o] = a;
            store_y(static_cast<YT*>(P.y), o, (float)((double)a * (double)g32 / (double)s_scale[m]));
        }
    }
}

template <int MT, bool FUSED, typename XT, typename YT, int MINB, bool NORM>
cudaError_t launch_t(const StreamBatch& b, int grid, size_t smem, unsigned* status, cudaStream_t st)
{
    auto fn = stream_kernel<MT, FUSED, XT, YT, MINB, NORM>;
    static bool configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, stream_budget(MINB));
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    // Programmatic dependent launch: this grid may start while the previous
    // kernel in the stream is still finishing.  Until griddepcontrol.wait it
    // only sets up and prefetches its weights into L2; every read of an
    // input and every write happens after the wait, so a dependency on the
    // previous kernel (e.g. the packer that wrote the weights) stays safe.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, fn, b, status);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <bool FUSED, typename XT, typename YT, int MINB, bool NORM>
cudaError_t launch_m(const StreamBatch& b, int grid, size_t smem, unsigned* status, cudaStream_t st)
{
    switch (stream_tokens(b.M)) {
        case 1: return launch_t<1, FUSED, XT, YT, MINB, NORM>(b, grid, smem, status, st);
        case 2: return launch_t<2, FUSED, XT, YT, MINB, NORM>(b, grid, smem, status, st);
        case 4: return launch_t<4, FUSED, XT, YT, MINB, NORM>(b, grid, smem, status, st);
        case 8: return launch_t<8, FUSED, XT, YT, MINB, NORM>(b, grid, smem, status, st);
        default: return launch_t<16, FUSED, XT, YT, MINB, NORM>(b, grid, smem, status, st);
    }
}

// 4 CTAs per SM (64 registers) only for up to 4 tokens; more tokens need
// the registers of the 2-CTA form.
template <bool FUSED, typename XT, typename YT, bool NORM>
cudaError_t launch_n(const StreamBatch& b, int minb, int grid, size_t smem, unsigned* status, cudaStream_t st)
{
    if (minb == 4) {
        switch (stream_tokens(b.M)) {
            case 1: return launch_t<1, FUSED, XT, YT, 4, NORM>(b, grid, smem, status, st);
            case 2: return launch_t<2, FUSED, XT, YT, 4, NORM>(b, grid, smem, status, st);
            case 4: return launch_t<4, FUSED, XT, YT, 4, NORM>(b, grid, smem, status, st);
            default: return cudaErrorNotSupported;
        }
    }
    return launch_m<FUSED, XT, YT, 2, NORM>(b, grid, smem, status, st);
}

// The normalising prologue (SubLN) is a separate instantiation, so the
// plain kernels keep their own register allocation.
template <bool FUSED, typename XT, typename YT>
cudaError_t launch_b(const StreamBatch& b, int minb, int grid, size_t smem, unsigned* status, cudaStream_t st)
{
    if constexpr (FUSED) {
        if (b.p[0].gain) return launch_n<true, XT, YT, true>(b, minb, grid, smem, status, st);
    }
    return launch_n<FUSED, XT, YT, false>(b, minb, grid, smem, status, st);
}

}  // namespace

int stream_tokens(int64_t M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16; }

int sm_count()
{
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        cached[dev] = v;
    }
    return cached[dev];
}

// CTAs per problem so that the largest per-CTA share of packed bytes,
// ceil(tiles / ctas) * tile bytes, is as small as possible (greedy: the next
// CTA always goes to the problem whose share is currently largest; one CTA
// per problem at least, one per tile at most).  Whole tiles per CTA make the
// granularity coarse for long rows (13.8 KB per tile at K = 6912), so a
// share proportional to bytes alone can leave one problem's CTAs with 45%
// more work than the rest.
bool assign_ctas(StreamBatch& b, int target)
{
    if (b.count > target) return false;
    int64_t tiles[kMaxGroup], tb[kMaxGroup];
    for (int i = 0; i < b.count; ++i) {
        tiles[i] = padded_n(b.p[i].N) / 8;
        tb[i] = tile_bytes(b.p[i].K);
        b.p[i].ctas = 1;
    }
    for (int used = b.count; used < target; ++used) {
        int best = -1;
        int64_t worst = -1;
        for (int i = 0; i < b.count; ++i) {
            if (b.p[i].ctas >= tiles[i]) continue;
            const int64_t load = (tiles[i] + b.p[i].ctas - 1) / b.p[i].ctas * tb[i];
            if (load > worst) {
                worst = load;
                best = i;
            }
        }
        if (best < 0) break;
        b.p[best].ctas++;
    }
    return true;
}

// Plans CTAs per problem (assign_ctas) and the shared
// memory split for `minb` resident CTAs per SM.  Returns false if the
// problems do not fit.
bool plan_stream(StreamBatch& b, int minb, int* grid, size_t* smem)
{
    const int target = minb * sm_count();
    const int MT = stream_tokens(b.M);
    int64_t total = 0, kp_max = 0;
    for (int i = 0; i < b.count; ++i) {
        const int64_t bytes = padded_n(b.p[i].N) * padded_k(b.p[i].K) / 4;
        if (bytes >= (int64_t(1) << 31)) return false;
        total += bytes;
        kp_max = kp_max > padded_k(b.p[i].K) ? kp_max : padded_k(b.p[i].K);
    }
    if (!assign_ctas(b, target)) return false;
    int64_t tiles_max = 1;
    int begin = 0;
    for (int i = 0; i < b.count; ++i) {
        const int64_t tiles = padded_n(b.p[i].N) / 8;
        b.p[i].cta_begin = begin;
        b.cta_begin[i] = begin;
        b.p[i].tiles_base = (int)(tiles / b.p[i].ctas);
        b.p[i].tiles_extra = (int)(tiles % b.p[i].ctas);
        begin += b.p[i].ctas;
        const int64_t per = (tiles + b.p[i].ctas - 1) / b.p[i].ctas;
        tiles_max = tiles_max > per ? tiles_max : per;
    }
    b.q_bytes = (int)(MT * kp_max);
    const int64_t acc_bytes = tiles_max * 8 * MT * 4;
    const int64_t left = (int64_t)stream_budget(minb) - b.q_bytes - acc_bytes;
    int stages = (int)(left / 16384);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 2) return false;
    b.stages = stages;
    *grid = begin;
    *smem = (size_t)stages * 16384 + b.q_bytes + acc_bytes;
    return true;
}

cudaError_t launch_stream(StreamBatch& b, bool fused, bl_dtype xt, bl_dtype yt, unsigned* status,
                          cudaStream_t st)
{
    int grid = 0, minb = stream_tokens(b.M) <= 4 ? 4 : 2;
    size_t smem = 0;
    if (!plan_stream(b, minb, &grid, &smem)) {
        minb = 2;
        if (!plan_stream(b, minb, &grid, &smem)) return cudaErrorNotSupported;
    }
    if (!fused) {
        if (yt == BL_F32) return launch_b<false, float, float>(b, minb, grid, smem, status, st);
        return launch_b<false, float, __nv_bfloat16>(b, minb, grid, smem, status, st);
    }
    if (xt == BL_F32) {
        if (yt == BL_F32) return launch_b<true, float, float>(b, minb, grid, smem, status, st);
        return launch_b<true, float, __nv_bfloat16>(b, minb, grid, smem, status, st);
    }
    if (yt == BL_F32) return launch_b<true, __nv_bfloat16, float>(b, minb, grid, smem, status, st);
    return launch_b<true, __nv_bfloat16, __nv_bfloat16>(b, minb, grid, smem, status, st);
}

}  // namespace bl
