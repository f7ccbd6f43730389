// bl_internal.cuh -- private declarations shared by the library's .cu files.
//
// Nothing here is part of the C ABI (include/bitlinear.h is).  The packed
// weight layout constants below restate that header's layout spec.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/bitlinear.h"

namespace bl {

// ---- packed layout (include/bitlinear.h) -------------------------------
constexpr int kTileRows = 8;        // rows per tile
constexpr int kChunkK = 64;         // weights per 16-byte chunk
constexpr int kChunkBytes = 16;

__host__ __device__ inline int64_t padded_k(int64_t K) { return (K + 63) / 64 * 64; }
__host__ __device__ inline int64_t padded_n(int64_t N) { return (N + 7) / 8 * 8; }
__host__ __device__ inline int64_t chunks_per_row(int64_t K) { return padded_k(K) / 64; }
// bytes of one 8-row tile
__host__ __device__ inline int64_t tile_bytes(int64_t K) { return chunks_per_row(K) * 8 * 16; }

// ---- activation code rounding --------------------------------------------
// rint(v), ties to even, for |v| <= 127.5, delivered in the low byte of a
// float's bit pattern: adding 1.5 * 2^23 puts the sum in [2^23, 2^24), where
// the fp32 spacing is 1, so the IEEE round-to-nearest-even addition rounds
// v to an integer r (the constant is even, so ties go the way rint's do)
// and the sum's bits are 0x4B400000 + r, whose low byte is r as an int8.
// One addition on the FMA pipe in place of a float-to-int conversion, which
// issues at a fraction of that rate; the caller packs the low bytes.
__device__ __forceinline__ uint32_t rint_low_byte(float v) { return __float_as_uint(__fadd_rn(v, 12582912.0f)); }

// ---- device status word bits --------------------------------------------
constexpr unsigned kStatusNonfiniteW = 1u;
constexpr unsigned kStatusNonfiniteX = 2u;

// Device address of the current device's status word (NULL on failure).
unsigned* status_word_ptr();

// ---- launch helpers (host side, one per .cu file) ------------------------
// Each returns cudaSuccess or the launch error; validation is done by the
// caller in bl_api.cu.
cudaError_t launch_absmean_partial(const float* W, int64_t count, double* partial, int blocks,
                                   unsigned* status, cudaStream_t st);
cudaError_t launch_absmean_finalize(const double* partial, int blocks, int64_t count, double eps,
                                    double* gamma64, float* gamma32, float* thr, cudaStream_t st);
cudaError_t launch_pack(const float* W, int64_t N, int64_t K, const float* thr, uint8_t* packed,
                        cudaStream_t st);
int absmean_blocks(int64_t count);

cudaError_t launch_quant(const void* x, bl_dtype xt, int64_t M, int64_t K, int8_t* q, float* s,
                         unsigned* status, cudaStream_t st);
// SubLN (RMS normalisation with gain [K], epsilon eps) then the quantiser.
cudaError_t launch_rmsnorm_quant(const void* x, bl_dtype xt, const float* gain, double eps, int64_t M, int64_t K,
                                 int8_t* q, float* s, unsigned* status, cudaStream_t st);
// The quantiser over the rows of several problems in one launch (one block
// per row): problem i has rows [row_begin, row_begin + M) of the grid.
struct QuantProblem {
    const void* x;          // activations [M][K]
    const float* gain;      // SubLN gain [K], or NULL
    int8_t* q;              // [M][Kp]
    float* s;               // [M]
    int64_t K;
    int row_begin;
};
constexpr int kMaxQuantGroup = 16;
struct QuantBatch {
    int row_begin[kMaxQuantGroup];   // copy of p[i].row_begin for the block -> problem search
    QuantProblem p[kMaxQuantGroup];
    int count;
    int rows;               // total rows (the grid)
    double eps;             // SubLN epsilon
};
cudaError_t launch_quant_grouped(const QuantBatch& b, bl_dtype xt, unsigned* status, cudaStream_t st);

// One problem of the decode kernel (packed ternary x int8 -> y).
struct GemvProblem {
    const void* x;          // fused form: activations [M][K] (fp32/bf16)
    const int8_t* q;        // unfused form: int8 [M][Kp]
    const float* s;         // unfused form: fp32 [M]
    const uint8_t* packed;  // packed ternary weights
    const float* gamma32;   // per-tensor scale
    void* y;                // [M][N]
    int32_t* acc;           // optional int32 [M][N]
    int64_t N, K;
    int64_t tile_begin;     // first 8-row tile index of this problem in the grid
};
constexpr int kMaxGroup = 16;
struct GemvBatch {
    GemvProblem p[kMaxGroup];
    int count;
    int64_t M;
};

cudaError_t launch_gemv(const GemvBatch& b, bool fused, bl_dtype xt, bl_dtype yt, unsigned* status,
                        cudaStream_t st);
// Largest M the fused decode kernel accepts.
constexpr int kFusedMaxM = 16;

// Persistent streaming decode kernel (bl_gemv_stream.cu), M <= 16.
struct StreamProblem {
    const void* x;          // fused form: activations [M][K] (fp32/bf16)
    const int8_t* q;        // unfused form: int8 [M][Kp]
    const float* s;         // unfused form: fp32 [M]
    const uint8_t* packed;
    const float* gamma32;
    void* y;
    int32_t* acc;           // optional
    const float* gain;      // fused form: SubLN gain [K] (RMS normalisation before the quantiser), or NULL
    int64_t N, K;
    int cta_begin;          // set by plan_stream
    int ctas;               // set by plan_stream
    int tiles_base;         // set by plan_stream: every CTA gets tiles_base tiles,
    int tiles_extra;        //   the first tiles_extra CTAs one more
};
struct StreamBatch {
    int cta_begin[kMaxGroup];   // copy of p[i].cta_begin, packed for the CTA -> problem search
    StreamProblem p[kMaxGroup];
    int count;
    int M;
    int stages;             // set by plan_stream
    int q_bytes;            // set by plan_stream
    int layout_tokens;      // tensor-core kernel: token slots of its operand layout
    double eps_norm;        // SubLN epsilon (problems with a gain)
};
constexpr int kMaxStages = 12;
// dynamic shared memory per CTA for `minb` resident CTAs per SM
constexpr int stream_budget(int minb) { return minb >= 4 ? 54 * 1024 : 110 * 1024; }
int stream_tokens(int64_t M);
int sm_count();
bool plan_stream(StreamBatch& b, int minb, int* grid, size_t* smem);
// CTAs per problem (fills p[i].ctas) minimising the largest per-CTA byte share.
bool assign_ctas(StreamBatch& b, int target);
// Returns cudaErrorNotSupported if the shapes do not fit (shared memory).
cudaError_t launch_stream(StreamBatch& b, bool fused, bl_dtype xt, bl_dtype yt, unsigned* status,
                          cudaStream_t st);

// Tensor-core decode kernel (bl_decode_tc.cu), M <= 16: same batch as the
// streaming kernel (plan fields are filled by its own planner).  Returns
// cudaErrorNotSupported if the shapes do not fit (shared memory).
bool plan_dec_tc(StreamBatch& b, int* grid, size_t* smem);
bool dec_tc_fits(int64_t M, int64_t K);
cudaError_t launch_dec_tc(StreamBatch& b, bool fused, bl_dtype xt, bl_dtype yt, unsigned* status,
                          cudaStream_t st);

// Table-lookup decode kernel (bl_gemv_lut.cu): M = 1, q and s given.
bool lut_supported(int64_t M, int64_t K);
cudaError_t launch_lut(const int8_t* q, const float* s, const uint8_t* packed, const float* gamma32, int64_t N,
                       int64_t K, void* y, bl_dtype yt, int32_t* acc, cudaStream_t st);

// Prefill tensor-core GEMM (tcgen05 kind::i8).  Returns cudaErrorNotSupported
// when the shape is outside what the kernel handles; the caller then uses
// the decode kernel.
cudaError_t launch_gemm_tc(const int8_t* q, const float* s, const uint8_t* packed,
                           const float* gamma32, int64_t M, int64_t N, int64_t K, void* y,
                           bl_dtype yt, int32_t* acc, unsigned* status, cudaStream_t st);
bool gemm_tc_supported(int64_t M, int64_t N, int64_t K);

}  // namespace bl
