// bl_decode_tc.cu -- decode BitLinear (M <= 16 tokens) on the tensor cores.
//
// y[m, n] = (sum_k code[n, k] * q[m, k]) * gamma / s_m, the ternary x int8
// product of aratech.ae "BitLinear: the building block" with the add /
// subtract / skip weights of bhfrc.com/news/56965 sec. 1.1.
//
// Decode streams every packed weight byte once, so the time is HBM time as
// long as the instructions spent per byte stay small.  Here the weights are
// not multiplied by the CUDA cores at all: each 32-bit word of 16 packed
// fields (u = code + 1, include/bitlinear.h) becomes four operand words by
// masking alone,
//     plane 0: w & 0x03030303          bytes u      (k = 16j + b)
//     plane 1: w & 0x0C0C0C0C          bytes 4u     (k = 16j + 4 + b)
//     plane 2: w & 0x30303030          bytes 16u    (k = 16j + 8 + b)
//     plane 3: (w >> 2) & 0x30303030   bytes 16u    (k = 16j + 12 + b)
// (five instructions per 16 weights; every byte is a valid signed int8),
// which go straight into tensor memory with tcgen05.st.  tcgen05.mma
// kind::i8 multiplies each plane by the activations of its k, into one
// accumulator per plane, and
//     sum_k u*q = D0 + D1/4 + D2/16 + D3/16,   sum_k code*q = that - sum_k q
// with exact integer shifts.
//
// MMA shape M = 128 (tensor-memory lanes), N = 16, K = 32.  The operand
// layout has MT token slots (1, 2, 4, 8 or 16; at least M, chosen per launch
// as large as shared memory allows): the 128 lanes are R = 8*MT weight rows
// times S = 16/MT k-slices, and the 16 B-operand rows are S slices times MT
// tokens.  Lane (row, slice) only uses the accumulator columns of its own
// slice, and the slices of a row are summed in the epilogue (with S = 1
// each lane is one whole row).  One "job" is up to MT tiles of 8 rows over
// the whole K -- a CTA owns a range of whole tiles, exactly as in the
// streaming dp4a kernel, and no partial sums cross CTAs.  Larger MT means
// longer jobs, so the per-job epilogue is amortised over more bytes.
//
// Per stage (8 KiB of packed weights) each lane takes 4 chunks (256 k) of
// its row: slice s of stage j holds chunks 4(jS + s) .. 4(jS + s) + 3.  The
// activations of all k are quantised once per CTA into shared memory, laid
// out as the B operand (K-major, 128-byte swizzle) in that same plane and
// slice order, so the MMA descriptors just step through it.
//
// Weight bytes reach shared memory by 16-byte cp.async issued by the
// expansion threads themselves, each for its own four chunks of a stage,
// several stages ahead (one commit group per stage): a stage is scattered
// over up to 16 tiles, and one bulk copy per tile piece (512 B at 16 tiles
// per job) would cost far more per byte than a 16 KiB copy.
//
// Warp roles (512 threads, one CTA per SM):
//   warps 0-3    MMA issuers (one lane each), warp t for plane t: one thread
//                issues a tcgen05.mma only every ~60-80 cycles (plus ~50 per
//                commit), and a stage needs 8 of them, so the four planes --
//                separate accumulators -- go to four threads; warp 0 also
//                allocates and frees the tensor memory
//   warps 4-11   expansion, two groups of four taking alternate stages, each
//                with its own ring of prefetched stages
//   warps 12-15  epilogue: tcgen05.ld, plane and slice sums, rescale, store
//   warps 4-15 also quantise x (fused form) or copy q (unfused) first, all
//                token rows together (bl_quant_rows.cuh).
// Tensor memory (512 columns): five 64-column A stages, three 64-column
// accumulator sets (4 planes x N = 16), so three jobs can be in flight --
// decode jobs are short (one or a few stages).
// All waits are bounded (bl_ptx.cuh); every role reaches the final barrier
// and the allocating warp frees the tensor memory.
#include "bl_internal.cuh"
#include "bl_ptx.cuh"
#include "bl_tc.cuh"
#include "bl_quant_rows.cuh"

namespace bl {
namespace {

constexpr int kThreads = 512;
constexpr int kStage = 8192;                 // packed bytes per stage
constexpr int kAStages = 5;
constexpr int kAColsPerStage = 64;           // 4 planes x 16 words
constexpr int kAccCol0 = kAStages * kAColsPerStage;   // 320
constexpr int kAccCols = 64;                 // 4 planes x N = 16
constexpr int kAccBufs = 3;                  // jobs in flight: 320 + 3 * 64 = 512 columns
constexpr int kTmemCols = 512;
constexpr int kExpWarp0 = 4, kEpiWarp0 = 12;
constexpr int kPrologueThreads = 384;        // warps 4..15
constexpr int kAtom = 2048;                  // 16 rows x 128 B (swizzled)
constexpr uint32_t kIdescDec = idesc_i8(128, 16);
constexpr int kPrefetch = 6;                 // stages in flight per expansion group (at most;
                                             // 4 or 2 when the resident operand is large)
constexpr int kSmemBudget = 227 * 1024;     // static + dynamic, per CTA
constexpr int kStaticReserve = 10 * 1024;   // barriers, ep[] (4 KiB at MT = 8), scratch

// Offset of the int8x4 activation word (k = 4*kw .. 4*kw+3, token m) in the
// resident B operand.  The word's k fixes its chunk c = kw/16, the word
// within the chunk wd, and its plane t; chunk group c/4 = j*S + s gives the
// stage j and the slice s; B row n = s*MT + m.  Atom 2j + t/2 holds planes
// 2*(t/2) and 2*(t/2)+1 of stage j for all 16 rows, 64 bytes each; within
// an atom the bytes follow the 128-byte swizzle (16-byte unit index xor
// row mod 8), as the MMA descriptor expects.
template <int MT>
__device__ __forceinline__ uint32_t bres_offset(int kw, int m)
{
    constexpr int S = 16 / MT;
    const int c = kw >> 4;
    const int wd = (kw >> 2) & 3;
    const int t = kw & 3;
    const int i = c & 3;
    const int gs = c >> 2;
    const int j = gs / S, s = gs % S;
    const int p = 4 * i + wd;
    const int n = s * MT + m;
    const int a = 2 * j + (t >> 1);
    const int x = (t & 1) * 64 + 4 * p;
    return (uint32_t)(a * kAtom + (n >> 3) * 1024 + (n & 7) * 128 + ((((x >> 4) ^ (n & 7)) << 4) | (x & 15)));
}

// stages of one job: ceil(C / (4 S))
template <int MT>
__host__ __device__ __forceinline__ int job_stages(int64_t K)
{
    constexpr int S = 16 / MT;
    return (int)((chunks_per_row(K) + 4 * S - 1) / (4 * S));
}

__device__ __forceinline__ void store_y(float* y, int64_t i, float v) { y[i] = v; }
__device__ __forceinline__ void store_y(__nv_bfloat16* y, int64_t i, float v) { y[i] = __float2bfloat16_rn(v); }

template <int MT, bool FUSED, typename XT, typename YT, bool NORM>
__global__ void __launch_bounds__(kThreads, 1) dec_tc_kernel(const __grid_constant__ StreamBatch b, unsigned* status)
{
    constexpr int S = 16 / MT;      // k-slices per row
    constexpr int R = 8 * MT;       // weight rows per job (tensor-memory lanes / S)
    constexpr int TJ = MT;          // tiles per job

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t expanded[kAStages], afree[kAStages];
    __shared__ uint64_t acc_full[kAccBufs], acc_empty[kAccBufs], done_bar;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    __shared__ int epi_ok;
    __shared__ float s_scale[16];
    __shared__ int s_sumq[16];
    __shared__ int ep[S > 1 ? 128 * MT : 1];
    __shared__ QuantRowsShared qsh;
    __shared__ double ss_rows[NORM ? kPrologueThreads / 32 * 16 : 1];

    // 1024-aligned dynamic region: resident B operand, then the two
    // expansion groups' rings of D prefetched stages each
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* bres = base;

    // ---- problem and tile range of this CTA
    int pi = 0;
#pragma unroll 1
    for (int i = 1; i < b.count; ++i)
        if ((int)blockIdx.x >= b.cta_begin[i]) pi = i;
    const StreamProblem& P = b.p[pi];
    const int K = (int)P.K, Kp = (int)padded_k(P.K);
    const int C = (int)chunks_per_row(P.K);
    const int64_t N = P.N;
    const int64_t TB = tile_bytes(P.K);
    const int ci = (int)blockIdx.x - P.cta_begin;
    const int64_t t0 = (int64_t)ci * P.tiles_base + (ci < P.tiles_extra ? ci : P.tiles_extra);
    const int ntl = P.tiles_base + (ci < P.tiles_extra ? 1 : 0);
    const int njobs = (ntl + TJ - 1) / TJ;
    const int tpj = (ntl + njobs - 1) / njobs;   // tiles per job, balanced
    const int J = job_stages<MT>(P.K);
    const int total = njobs * J;
    const uint32_t bres_bytes = (uint32_t)J * 2 * kAtom;
    // The region was planned for the group's largest operand with rings of
    // b.stages; a CTA of a problem with a smaller operand (shorter K) gives
    // the difference to deeper rings: D = 2, 4 or 6 stages per group.
    uint8_t* ring = base + bres_bytes;
    const int D = [&] {
        const uint32_t fit = ((uint32_t)b.q_bytes + 2u * (uint32_t)b.stages * kStage - bres_bytes) / (2u * kStage);
        return fit >= (uint32_t)kPrefetch ? kPrefetch : fit >= 4 ? 4 : 2;
    }();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        for (int i = 0; i < kAStages; ++i) {
            mbar_init(&expanded[i], 128);
            mbar_init(&afree[i], 4);
        }
        for (int i = 0; i < kAccBufs; ++i) {
            mbar_init(&acc_full[i], 4);
            mbar_init(&acc_empty[i], 128);
        }
        mbar_init(&done_bar, 4);
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        __syncwarp();
        tmem_alloc(&tmem_base, kTmemCols);
    }
    // the previous kernel in the stream may still be running (programmatic
    // dependent launch): nothing is read before this point
    asm volatile("griddepcontrol.wait;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    volatile int* abort = &abort_flag;

    // stage g = (job q, stage j of the job); jt tiles in the job; len
    // chunks per tile in this stage (the last stage of a job may be short)
    auto stage_geom = [&](int g, int& q, int& j, int& jt, int& len) {
        q = g / J;
        j = g - q * J;
        jt = ntl - q * tpj < tpj ? ntl - q * tpj : tpj;
        const int rem = C - 4 * j * S;
        len = rem < 4 * S ? rem : 4 * S;
    };

    // expansion thread identity: tensor-memory lane l = (row rho, slice s)
    const int grp = (warp - kExpWarp0) >> 2;              // stages g with g % 2 == grp
    const int l = 32 * (warp & 3) + lane;
    const int e_rho = l % R, e_s = l / R;
    const int e_tau = e_rho >> 3, e_r = e_rho & 7;
    uint8_t* gring = ring + (size_t)grp * D * kStage;      // this group's ring
    // Prefetch of this thread's 4 chunks of its k-th stage (g = grp + 2k)
    // into slot k % D: 16-byte cp.async per chunk, zero-filled (source size
    // 0, nothing read) past the job's tiles or the row's chunks; one commit
    // group per stage, empty past the last stage so the group count stays
    // uniform.  Slot layout: chunk i of lane l at i * 2048 + l * 16.
    auto prefetch = [&](int k) {
        const int g = grp + 2 * k;
        if (g < total) {
            int q, j, jt, len;
            stage_geom(g, q, j, jt, len);
            const bool row_ok = e_tau < jt;
            const uint8_t* src = P.packed + (t0 + (int64_t)q * tpj + (row_ok ? e_tau : 0)) * TB +
                                 (int64_t)(4 * (j * S + e_s)) * 128 + e_r * 16;
            const uint32_t dst = smem_u32(gring + (size_t)(k % D) * kStage + l * 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const bool ok = row_ok && (4 * e_s + i < len);
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst + i * 2048),
                             "l"(ok ? src + i * 128 : P.packed), "r"(ok ? 16 : 0)
                             : "memory");
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    const int my_stages = total > grp ? (total - grp + 1) / 2 : 0;
    if (warp >= kExpWarp0 && warp < kEpiWarp0)
        for (int k = 0; k < D; ++k) prefetch(k);

    // ---- prologue (warps 4..15): activations into the resident operand
    if (warp >= kExpWarp0) {
        const int tp = threadIdx.x - 32 * kExpWarp0;
        for (uint32_t o = (uint32_t)tp * 16; o < bres_bytes; o += kPrologueThreads * 16)
            *reinterpret_cast<uint4*>(bres + o) = make_uint4(0, 0, 0, 0);
        named_bar(1, kPrologueThreads);
        const int M = b.M;
        auto store_b = [&](int m, int kw, uint32_t w) {
            *reinterpret_cast<uint32_t*>(bres + bres_offset<MT>(kw, m)) = w;
        };
        auto sync_pro = [&]() { named_bar(1, kPrologueThreads); };
        if constexpr (FUSED) {
            quantise_rows<MT, kPrologueThreads, XT, NORM>(static_cast<const XT*>(P.x), M, K, P.gain, b.eps_norm, tp,
                                                          qsh, ss_rows, s_scale, s_sumq, store_b, sync_pro, status);
        } else {
            copy_q_rows<MT, kPrologueThreads>(P.q, M, Kp, tp, qsh, s_sumq, store_b, sync_pro);
            if (tp < M) s_scale[tp] = P.s[tp];
        }
        // generic-proxy writes of the operand, read next by the tensor cores
        fence_proxy_async_smem();
    }
    __syncthreads();

    if (warp < 4) {
        // ---------------------------------------------------- MMA issuers
        if (lane == 0) {
            const int t = warp;                        // plane
            const uint32_t bplane = smem_u32(bres) + (t >> 1) * kAtom + (t & 1) * 64;
            bool ok = true;
            int g = 0, as = 0, aph = 0;                // stage, A slot, its phase
            for (int q = 0; ok && q < njobs; ++q) {
                const int bf = q % kAccBufs;
                if (q >= kAccBufs && !wait_parity(&acc_empty[bf], ((q / kAccBufs) - 1) & 1, status, abort)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + kAccCol0 + bf * kAccCols + t * 16;
                for (int j = 0; j < J; ++j, ++g) {
                    if (!wait_parity(&expanded[as], aph, status, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_tmem = tmem + as * kAColsPerStage + t * 16;
                    const uint32_t baddr = bplane + j * (2 * kAtom);
                    mma_i8_ts(d_tmem, a_tmem, make_bdesc(baddr), kIdescDec, j != 0);
                    mma_i8_ts(d_tmem, a_tmem + 8, make_bdesc(baddr + 32), kIdescDec, 1u);
                    mma_commit(&afree[as]);
                    if (++as == kAStages) {
                        as = 0;
                        aph ^= 1;
                    }
                }
                if (ok) mma_commit(&acc_full[bf]);
            }
            mma_commit(&done_bar);
        }
    } else if (warp >= kExpWarp0 && warp < kEpiWarp0) {
        // ------------------------------------------------------ expansion
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        for (int k = 0; k < my_stages; ++k) {
            const int g = grp + 2 * k;
            const int as = g % kAStages;
            bool got = true;
            if (g >= kAStages) got = wait_parity(&afree[as], ((g / kAStages) - 1) & 1, status, abort);
            if (!__all_sync(0xffffffffu, got)) break;   // warp-uniform: tcgen05.st is .aligned
            // this thread's copies of stage k have landed (D - 1 younger
            // groups may still be in flight)
            if (D == 6)
                asm volatile("cp.async.wait_group 5;" ::: "memory");
            else if (D == 4)
                asm volatile("cp.async.wait_group 3;" ::: "memory");
            else
                asm volatile("cp.async.wait_group 1;" ::: "memory");
            const uint8_t* sp = gring + (size_t)(k % D) * kStage + l * 16;
            uint32_t lo[32], hi[32];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 wv = *reinterpret_cast<const uint4*>(sp + i * 2048);
                const uint32_t w[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                for (int wd = 0; wd < 4; ++wd) {
                    const int p = 4 * i + wd;
                    lo[p] = w[wd] & 0x03030303u;
                    lo[16 + p] = w[wd] & 0x0C0C0C0Cu;
                    hi[p] = w[wd] & 0x30303030u;
                    hi[16 + p] = (w[wd] >> 2) & 0x30303030u;
                }
            }
            // the slot is read (the values are in registers): refill it
            prefetch(k + D);
            tmem_st32(tmem + lane_base + as * kAColsPerStage, lo);
            tmem_st32(tmem + lane_base + as * kAColsPerStage + 32, hi);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&expanded[as]);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp >= kEpiWarp0) {
        // ------------------------------------------------------- epilogue
        const int et = threadIdx.x - 32 * kEpiWarp0;   // 0..127
        const int l = 32 * (warp & 3) + lane;
        const int s = l / R;
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        const int M = b.M;
        const double g32 = (double)*P.gamma32;
        for (int q = 0; q < njobs; ++q) {
            const int bf = q % kAccBufs;
            if (et == 0) epi_ok = wait_parity(&acc_full[bf], (q / kAccBufs) & 1, status, abort) ? 1 : 0;
            named_bar(3, 128);
            if (!epi_ok) break;
            tc_fence_after();
            uint32_t d01[32], d23[32];
            tmem_ld32(tmem + lane_base + kAccCol0 + bf * kAccCols, d01);
            tmem_ld32(tmem + lane_base + kAccCol0 + bf * kAccCols + 32, d23);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&acc_empty[bf]);
            // plane sums per accumulator column (exact: D1 is a multiple of
            // 4, D2 and D3 of 16)
            int tot[16];
#pragma unroll
            for (int c = 0; c < 16; ++c)
                tot[c] = (int)d01[c] + ((int)d01[16 + c] >> 2) + ((int)d23[c] >> 4) + ((int)d23[16 + c] >> 4);
            const int jt = ntl - q * tpj < tpj ? ntl - q * tpj : tpj;
            const int64_t n0 = (t0 + (int64_t)q * tpj) * 8;
            if constexpr (S == 1) {
                // one lane = one whole row: column m is token m
                const int64_t n = n0 + l;
                if (l < jt * 8 && n < N) {
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        if (m < M) {
                            const int a = tot[m] - s_sumq[m];
                            const int64_t o = (int64_t)m * N + n;
                            if (P.acc) P.acc[o] = a;
                            store_y(static_cast<YT*>(P.y), o, (float)((double)a * g32 / (double)s_scale[m]));
                        }
                    }
                }
            } else {
                // this lane's slice s: columns s*MT .. s*MT + MT - 1; the S
                // slices of a row meet in shared memory
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    int v = tot[m];
#pragma unroll
                    for (int ss = 1; ss < S; ++ss)
                        if (s == ss) v = tot[ss * MT + m];
                    ep[l * MT + m] = v;
                }
                named_bar(3, 128);
                const int rows = jt * 8;
                for (int i = et; i < rows * M; i += 128) {
                    const int m = i / rows, rr = i - m * rows;
                    const int64_t n = n0 + rr;
                    if (n < N) {
                        int a = -s_sumq[m];
#pragma unroll
                        for (int ss = 0; ss < S; ++ss) a += ep[(ss * R + rr) * MT + m];
                        const int64_t o = (int64_t)m * N + n;
                        if (P.acc) P.acc[o] = a;
                        store_y(static_cast<YT*>(P.y), o, (float)((double)a * g32 / (double)s_scale[m]));
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        wait_parity(&done_bar, 0, status, nullptr, true);
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int MT, bool FUSED, typename XT, typename YT, bool NORM>
cudaError_t launch_t(const StreamBatch& b, int grid, size_t smem, unsigned* status, cudaStream_t st)
{
    auto fn = dec_tc_kernel<MT, FUSED, XT, YT, NORM>;
    static bool configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        cudaError_t e =
            cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget - kStaticReserve);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
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

template <bool FUSED, typename XT, typename YT, bool NORM>
cudaError_t launch_mn(const StreamBatch& b, int MT, int grid, size_t smem, unsigned* status, cudaStream_t st)
{
    switch (MT) {
        case 1: return launch_t<1, FUSED, XT, YT, NORM>(b, grid, smem, status, st);
        case 2: return launch_t<2, FUSED, XT, YT, NORM>(b, grid, smem, status, st);
        case 4: return launch_t<4, FUSED, XT, YT, NORM>(b, grid, smem, status, st);
        case 8: return launch_t<8, FUSED, XT, YT, NORM>(b, grid, smem, status, st);
        default: return launch_t<16, FUSED, XT, YT, NORM>(b, grid, smem, status, st);
    }
}

// The normalising prologue (SubLN) is a separate instantiation.
template <bool FUSED, typename XT, typename YT>
cudaError_t launch_m(const StreamBatch& b, int MT, int grid, size_t smem, unsigned* status, cudaStream_t st)
{
    if constexpr (FUSED) {
        if (b.p[0].gain) return launch_mn<true, XT, YT, true>(b, MT, grid, smem, status, st);
    }
    return launch_mn<FUSED, XT, YT, false>(b, MT, grid, smem, status, st);
}

int job_stages_rt(int MT, int64_t K)
{
    switch (MT) {
        case 1: return job_stages<1>(K);
        case 2: return job_stages<2>(K);
        case 4: return job_stages<4>(K);
        case 8: return job_stages<8>(K);
        default: return job_stages<16>(K);
    }
}

}  // namespace

// One CTA per SM.  CTAs go to the problems by assign_ctas (smallest largest
// per-CTA share; at least one each, at most one per tile); each CTA gets a
// contiguous range of whole tiles.  Shared memory: the resident activation
// operand (MT * Kp bytes, rounded up to whole stages) and two rings of 6
// (else 4 or 2) 8 KiB stages.  MT (the operand's token slots, >= M) is the
// largest for which that fits.
// Whether one problem of M tokens and K columns fits the kernel's shared
// memory at all: the resident operand of M's own slot count beside rings of
// two stages.
bool dec_tc_fits(int64_t M, int64_t K)
{
    const int64_t budget = kSmemBudget - kStaticReserve - 1024;
    return M >= 1 && M <= 16 && (int64_t)job_stages_rt(stream_tokens(M), K) * 2 * kAtom + 2 * 2 * kStage <= budget;
}

bool plan_dec_tc(StreamBatch& b, int* grid, size_t* smem)
{
    const int target = sm_count();
    if (b.count > target) return false;
    int64_t total = 0;
    for (int i = 0; i < b.count; ++i) {
        const int64_t bytes = padded_n(b.p[i].N) * padded_k(b.p[i].K) / 4;
        if (bytes >= (int64_t(1) << 31)) return false;
        total += bytes;
    }
    // operand layout: the most token slots (longest jobs) whose resident
    // operand still leaves room for both expansion groups' rings of 6
    // stages; failing that, M's own slot count with rings of 4 or 2
    const int64_t budget = kSmemBudget - kStaticReserve - 1024;   // static shared memory, alignment slack
    int MT = 0, depth = 0;
    int64_t bres_max = 0;
    auto bres_of = [&](int cand) {
        int64_t br = 0;
        for (int i = 0; i < b.count; ++i) {
            const int64_t x = (int64_t)job_stages_rt(cand, b.p[i].K) * 2 * kAtom;
            br = br > x ? br : x;
        }
        return br;
    };
    for (int cand = 16; cand >= stream_tokens(b.M) && MT == 0; cand >>= 1) {
        const int64_t br = bres_of(cand);
        if (br + 2 * kPrefetch * kStage <= budget) {
            MT = cand;
            depth = kPrefetch;
            bres_max = br;
        }
    }
    if (MT == 0) {
        const int64_t br = bres_of(stream_tokens(b.M));
        for (int d = 4; d >= 2 && MT == 0; d -= 2)
            if (br + 2 * d * kStage <= budget) {
                MT = stream_tokens(b.M);
                depth = d;
                bres_max = br;
            }
    }
    if (MT == 0) return false;
    const int64_t rings = 2 * (int64_t)depth * kStage;
    if (!assign_ctas(b, target)) return false;
    int begin = 0;
    for (int i = 0; i < b.count; ++i) {
        const int64_t tiles = padded_n(b.p[i].N) / 8;
        b.p[i].cta_begin = begin;
        b.cta_begin[i] = begin;
        b.p[i].tiles_base = (int)(tiles / b.p[i].ctas);
        b.p[i].tiles_extra = (int)(tiles % b.p[i].ctas);
        begin += b.p[i].ctas;
    }
    b.stages = depth;
    b.q_bytes = (int)bres_max;
    b.layout_tokens = MT;
    *grid = begin;
    // at least ~116 KiB so that a second CTA never shares the SM (and its
    // tensor memory)
    size_t need = (size_t)(bres_max + rings) + 1024;
    if (need < 116 * 1024) need = 116 * 1024;
    *smem = need;
    return true;
}

cudaError_t launch_dec_tc(StreamBatch& b, bool fused, bl_dtype xt, bl_dtype yt, unsigned* status, cudaStream_t st)
{
    int grid = 0;
    size_t smem = 0;
    if (!plan_dec_tc(b, &grid, &smem)) return cudaErrorNotSupported;
    const int MT = b.layout_tokens;
    if (!fused) {
        if (yt == BL_F32) return launch_m<false, float, float>(b, MT, grid, smem, status, st);
        return launch_m<false, float, __nv_bfloat16>(b, MT, grid, smem, status, st);
    }
    if (xt == BL_F32) {
        if (yt == BL_F32) return launch_m<true, float, float>(b, MT, grid, smem, status, st);
        return launch_m<true, float, __nv_bfloat16>(b, MT, grid, smem, status, st);
    }
    if (yt == BL_F32) return launch_m<true, __nv_bfloat16, float>(b, MT, grid, smem, status, st);
    return launch_m<true, __nv_bfloat16, __nv_bfloat16>(b, MT, grid, smem, status, st);
}

}  // namespace bl
