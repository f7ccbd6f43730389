// bl_gemm_tc.cu -- prefill BitLinear on the 5th-generation tensor cores
// (tcgen05 kind::i8): D[n, m] = sum_k code[n, k] * q[m, k] with int32
// accumulation in tensor memory, then y[m, n] = D * (gamma32 / s_m).
// (bhfrc.com/news/56965 sec. 1.1: ternary weights make the product pure
// integer adds; aratech.ae "BitLinear: the building block" for the int8
// per-token activations.)
//
// Persistent kernel, one CTA per SM, looping over 128 (weight rows, MMA M)
// x 128 (tokens, MMA N) output tiles; K in stages of 256 (eight MMAs of
// K = 32 per barrier round trip), 4 stages deep.
// The weights never exist as int8 in memory: the packed 2-bit codes are
// TMA-loaded (4 KiB per stage), eight expansion warps decode them to signed
// int8 in registers and write them straight into tensor memory with
// tcgen05.st, where the MMA reads them as its A operand.  Shared memory only
// carries the activation tiles (B operand, TMA with 128-byte swizzle).
//
// Tensor memory (512 columns): two 128-column int32 accumulators (tile i is
// drained by the epilogue while tile i+1 accumulates into the other) and
// four 64-column A stages.
//
// Warp roles (512 threads):
//   warp 0       TMEM allocation; TMA producer (one lane)
//   warps 1, 2   MMA issuers (one lane each, tokens 0-63 and 64-127 of the
//                tile): 8 x tcgen05.mma (N = 64, K = 32) per stage,
//                tcgen05.commit -> stage-free barrier; per tile -> acc-full.
//                They wait only for the expansion barrier: the expansion
//                threads arrive there after observing the stage's TMA
//                barrier, so the activation tile is complete by then too
//   warps 4-11   expansion, two groups of four taking alternate stages:
//                warp w writes TMEM lanes 32*(w%4) .. +31 of its stages
//   warps 12-15  epilogue: per-token factors f_m = gamma32 / s_m (fp32,
//                correctly rounded), tcgen05.ld of the finished accumulator,
//                y = fp32(acc) * f_m (the conversion is exact below 2^24), store,
//                then release the accumulator
// All mbarrier waits are bounded (bl_ptx.cuh); every role reaches the final
// barrier, after which the allocating warp frees the tensor memory.
//
// Decode to signed int8: the packed fields hold u = code + 1 (include/
// bitlinear.h); field t of every byte, ((w >> 2t) & 0x03030303), plus
// 0x7F7F7F7F then xor 0x80808080 gives the bytes 0xFF, 0x00, 0x01.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "bl_internal.cuh"
#include "bl_ptx.cuh"
#include "bl_tc.cuh"

namespace bl {
namespace {

constexpr int BM = 128;        // weight rows per tile (MMA M)
constexpr int BN = 128;        // tokens per tile (MMA N)
constexpr int BK = 256;        // k per stage (bytes of int8): 8 MMAs per barrier round trip
constexpr int STAGES = 4;
constexpr int kThreads = 512;
constexpr int Q_ATOM = BN * 128;             // one 128-byte-wide K slab of the token tile
constexpr int Q_STAGE = BN * BK;             // 32 KiB: two 128B-swizzled slabs
constexpr int W_HALF = (BM / 8) * 256;       // 16 tiles x 2 chunks x 128 B = 4 KiB
constexpr int W_STAGE = 2 * W_HALF;          // 4 chunks of every row: 8 KiB
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = BN;                 // one accumulator buffer
constexpr int A_COL0 = 2 * ACC_COLS;         // A stages after the two accumulators
constexpr int A_STAGE_COLS = BK / 4;         // 64 columns per stage
constexpr int EXP_WARP0 = 4, EPI_WARP0 = 12;

struct Smem {
    uint8_t q[STAGES][Q_STAGE];              // 1024-aligned (first member)
    uint8_t w[STAGES][W_STAGE];
    uint64_t full[STAGES], expanded[STAGES], empty[STAGES];
    uint64_t acc_full[2], acc_empty[2], done;
    uint32_t tmem_base;
    int abort_flag;
    int epi_ok[2];
};

// Field t of every byte (u = code + 1 in {0, 1, 2}) -> signed int8 code:
// u + 0x7F is 0x7F, 0x80 or 0x81 (no carry out of the byte); flipping the
// top bit gives 0xFF, 0x00, 0x01 = -1, 0, +1.
__device__ __forceinline__ uint32_t signed_codes(int t, uint32_t w)
{
    return (((w >> (2 * t)) & 0x03030303u) + 0x7F7F7F7Fu) ^ 0x80808080u;
}

// kind::i8, D = S32, A = B = signed int8, both K-major, M = 128, N = BN/2:
// two issuing threads each take half of the tokens (one thread issues a
// tcgen05.mma only every ~57 cycles; two keep the tensor pipe busy).
constexpr int HALF_N = BN / 2;
constexpr uint32_t kIdesc = idesc_i8(BM, HALF_N);

__device__ __forceinline__ void store_y(float* y, int64_t i, float v) { y[i] = v; }
// bf16 round-to-nearest-even on the bit pattern (y is always finite here):
// add 0x7FFF plus the lowest kept bit, then truncate.
__device__ __forceinline__ void store_y(__nv_bfloat16* y, int64_t i, float v)
{
    uint32_t u = __float_as_uint(v);
    u += 0x7FFFu + ((u >> 16) & 1u);
    reinterpret_cast<uint16_t*>(y)[i] = (uint16_t)(u >> 16);
}

// int32 -> fp32, exact for |a| < 2^22 with two ALU-pipe instructions: the
// float with bit pattern 0x4B400000 + a is 1.5 * 2^23 + a (its unit in the
// last place is 1), and subtracting 1.5 * 2^23 leaves a.
__device__ __forceinline__ float small_int_to_float(int a)
{
    return __fsub_rn(__int_as_float(0x4B400000 + a), 12582912.0f);
}

template <typename YT>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_w,
               const float* __restrict__ s_in, const float* __restrict__ gamma32, int M, int N, int nk,
               YT* __restrict__ y, int32_t* __restrict__ acc_out, unsigned* status)
{
    extern __shared__ uint8_t smem_raw[];
    // per-token factors gamma32 / s_m of the two accumulator buffers; a
    // static array, so the compiler sees shared-memory loads it may batch
    __shared__ float s_fac[2][BN];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_n = (N + BM - 1) / BM, tiles_m = (M + BN - 1) / BN;
    const int total = tiles_n * tiles_m;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.expanded[s], 128);   // one expansion group
            mbar_init(&sm.empty[s], 2);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.acc_full[b], 2);
            mbar_init(&sm.acc_empty[b], 128);
        }
        mbar_init(&sm.done, 2);
        sm.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        __syncwarp();
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&sm.tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int* abort = &sm.abort_flag;

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmap_q);
            prefetch_tmap(&tmap_w);
            int g = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
                const int n0 = (t % tiles_n) * BM, m0 = (t / tiles_n) * BN;
                for (int kb = 0; kb < nk; ++kb, ++g) {
                    const int s = g % STAGES, round = g / STAGES;
                    if (round > 0 && !wait_parity(&sm.empty[s], (round - 1) & 1, status, abort)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sm.full[s], Q_STAGE + W_STAGE);
                    tma_load_2d(sm.q[s], &tmap_q, kb * BK, m0, &sm.full[s]);
                    tma_load_2d(sm.q[s] + Q_ATOM, &tmap_q, kb * BK + 128, m0, &sm.full[s]);
                    tma_load_2d(sm.w[s], &tmap_w, kb * 512, n0 / 8, &sm.full[s]);
                    tma_load_2d(sm.w[s] + W_HALF, &tmap_w, kb * 512 + 256, n0 / 8, &sm.full[s]);
                }
            }
            // every copy issued has landed before this thread leaves
            for (int j = g - STAGES < 0 ? 0 : g - STAGES; j < g; ++j)
                wait_parity(&sm.full[j % STAGES], (j / STAGES) & 1, status, nullptr, true);
        }
    } else if (warp == 1 || warp == 2) {
        // ----------------------------------------------------- MMA issuers
        // warp 1: tokens 0..63 of the tile, warp 2: tokens 64..127 (B rows
        // 64.. start 8 swizzle groups = 8 KiB into each slab; D columns 64..)
        if (lane == 0) {
            const int hn = warp - 1;
            int g = 0, i = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < total; t += gridDim.x, ++i) {
                const int b = i & 1, ar = i >> 1;
                if (ar > 0 && !wait_parity(&sm.acc_empty[b], (ar - 1) & 1, status, abort)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + b * ACC_COLS + hn * HALF_N;
                for (int kb = 0; kb < nk; ++kb, ++g) {
                    const int s = g % STAGES;
                    const uint32_t ph = (g / STAGES) & 1;
                    if (!wait_parity(&sm.expanded[s], ph, status, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t qaddr = smem_u32(sm.q[s]) + hn * (HALF_N / 8) * 1024;
#pragma unroll
                    for (int j = 0; j < BK / 32; ++j)
                        mma_i8_ts(d_tmem, tmem + A_COL0 + s * A_STAGE_COLS + j * 8,
                                  make_bdesc(qaddr + (j >> 2) * Q_ATOM + (j & 3) * 32), kIdesc, (kb | j) != 0);
                    mma_commit(&sm.empty[s]);
                }
                if (ok) mma_commit(&sm.acc_full[b]);
            }
            mma_commit(&sm.done);   // retires every MMA this thread issued
        }
    } else if (warp >= EXP_WARP0 && warp < EPI_WARP0) {
        // --------------------------------------------- expansion warps 4..11
        // Two groups of four warps take alternate stages, so each thread has
        // two MMA-stage periods to decode, store into TMEM and wait for the
        // store; the four warps of a group cover the 128 TMEM lanes.
        const int quarter = warp & 3;
        const int grp = (warp - EXP_WARP0) >> 2;               // stages g with g % 2 == grp
        const int rr = 32 * quarter + lane;                    // TMEM lane = weight row in tile
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        const int woff = (rr >> 3) * 256 + (rr & 7) * 16;
        int g = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
            for (int kb = 0; kb < nk; ++kb, ++g) {
                if ((g & 1) != grp) continue;
                const int s = g % STAGES;
                const bool got = wait_parity(&sm.full[s], (g / STAGES) & 1, status, abort);
                if (!__all_sync(0xffffffffu, got)) {   // warp-uniform: tcgen05.st is .aligned
                    ok = false;
                    break;
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {          // chunks 2h, 2h+1 of the stage
                    uint32_t out[32];
#pragma unroll
                    for (int cl = 0; cl < 2; ++cl) {
                        const uint4 wv = *reinterpret_cast<const uint4*>(sm.w[s] + h * W_HALF + woff + cl * 128);
                        const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
#pragma unroll
                            for (int tt = 0; tt < 4; ++tt) out[16 * cl + 4 * i + tt] = signed_codes(tt, words[i]);
                        }
                    }
                    tmem_st32(tmem + lane_base + A_COL0 + s * A_STAGE_COLS + 32 * h, out);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&sm.expanded[s]);
            }
        }
    } else if (warp >= EPI_WARP0) {
        // ------------------------------------------------ epilogue 12..15
        const int et = threadIdx.x - 32 * EPI_WARP0;          // 0..127
        const int quarter = warp & 3;
        const int rr = 32 * quarter + lane;
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        const float gam = *gamma32;
        // |acc| <= 127 * Kp: below 2^22 the conversion needs no converter unit
        const bool small_acc = (int64_t)127 * nk * BK < (int64_t(1) << 22);
        int i = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++i) {
            const int b = i & 1, ar = i >> 1;
            const int n0 = (t % tiles_n) * BM, m0 = (t / tiles_n) * BN;
            {
                const int m = m0 + et;
                s_fac[b][et] = (m < M) ? __fdiv_rn(gam, s_in[m]) : 0.0f;
            }
            // one thread waits for the accumulator; the verdict goes through
            // shared memory so all four warps take the same branch
            if (et == 0) sm.epi_ok[b] = wait_parity(&sm.acc_full[b], ar & 1, status, abort, true) ? 1 : 0;
            named_bar(3, 128);
            if (!sm.epi_ok[b]) break;
            tc_fence_after();
            const int n = n0 + rr;
            const uint32_t acc_tmem = tmem + lane_base + b * ACC_COLS;
#pragma unroll 1
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint32_t v[32];
                tmem_ld32(acc_tmem + cc * 32, v);
                tmem_wait_ld();
                if (n < N) {
                    // 8 tokens at a time: factors first (independent
                    // loads), then 8 independent rescale chains, then the
                    // stores, so no load waits behind a store
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        float f[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) f[j] = s_fac[b][cc * 32 + h * 8 + j];
                        float o[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int a = (int)v[h * 8 + j];
                            o[j] = __fmul_rn(small_acc ? small_int_to_float(a) : __int2float_rn(a), f[j]);
                        }
                        const int mb = m0 + cc * 32 + h * 8;
                        if (acc_out) {
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                if (mb + j < M) acc_out[(int64_t)(mb + j) * N + n] = (int)v[h * 8 + j];
                        }
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            if (mb + j < M) store_y(y, (int64_t)(mb + j) * N + n, o[j]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&sm.acc_empty[b]);
        }
    }
    __syncthreads();
    if (warp == 0) {
        wait_parity(&sm.done, 0, status, nullptr, true);
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS)
                     : "memory");
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

bool make_2d_u8(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t stride,
                uint32_t box_in, uint32_t box_out, CUtensorMapSwizzle sw)
{
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {stride};
    const cuuint32_t box[2] = {box_in, box_out};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename YT>
cudaError_t launch_typed(const CUtensorMap& tq, const CUtensorMap& tw, const float* s, const float* g, int M,
                         int N, int nk, void* y, int32_t* acc, unsigned* status, cudaStream_t st)
{
    const size_t smem = sizeof(Smem) + 1024;
    static bool configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<YT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    const int tiles = ((N + BM - 1) / BM) * ((M + BN - 1) / BN);
    const int grid = tiles < sm_count() ? tiles : sm_count();
    gemm_tc_kernel<YT><<<grid, kThreads, smem, st>>>(tq, tw, s, g, M, N, nk, static_cast<YT*>(y), acc, status);
    return cudaGetLastError();
}

}  // namespace

bool gemm_tc_supported(int64_t M, int64_t N, int64_t K)
{
    return M > 16 && M < (int64_t(1) << 31) && N < (int64_t(1) << 31) &&
           ((N + BM - 1) / BM) * ((M + BN - 1) / BN) < (int64_t(1) << 31) && padded_k(K) < (int64_t(1) << 31) &&
           encode_fn() != nullptr;
}

cudaError_t launch_gemm_tc(const int8_t* q, const float* s, const uint8_t* packed, const float* gamma32,
                           int64_t M, int64_t N, int64_t K, void* y, bl_dtype yt, int32_t* acc,
                           unsigned* status, cudaStream_t st)
{
    const int64_t Kp = padded_k(K);
    const int64_t TB = chunks_per_row(K) * 128;
    CUtensorMap tq, tw;
    if (!make_2d_u8(&tq, q, (uint64_t)Kp, (uint64_t)M, (uint64_t)Kp, 128, BN, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_2d_u8(&tw, packed, (uint64_t)TB, (uint64_t)(padded_n(N) / 8), (uint64_t)TB, 256, BM / 8,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const int nk = (int)((Kp + BK - 1) / BK);
    if (yt == BL_F32)
        return launch_typed<float>(tq, tw, s, gamma32, (int)M, (int)N, nk, y, acc, status, st);
    return launch_typed<__nv_bfloat16>(tq, tw, s, gamma32, (int)M, (int)N, nk, y, acc, status, st);
}

}  // namespace bl
