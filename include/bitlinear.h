/*
 * bitlinear.h -- C ABI of the B200 (sm_100a) BitNet b1.58 BitLinear library.
 *
 * The layer (BitNet b1.58 pages: aratech.ae, "BitNet b1.58: Microsoft's 1-bit
 * LLM that runs a 100B model on a single CPU", sections "Ternary weights
 * {-1, 0, +1}" and "BitLinear: the building block"; bhfrc.com/news/56965,
 * sec. 1.1 and sec. 4.1):
 *
 *   gamma   = mean_{n,k} |W_nk|                       (per tensor, fp64 sum)
 *   code_nk = clip(round(W_nk / (gamma + eps)), -1, 1)            in {-1,0,1}
 *   s_m     = 127 / max_k |x_mk|                      (per token, fp32)
 *   q_mk    = clip(rint(x_mk * s_m), -127, 127)                   int8
 *   acc_mn  = sum_k q_mk * code_nk                                int32
 *   y_mn    = acc_mn * gamma / s_m                    (fp32, or bf16 output)
 *
 * Conventions for every entry point:
 *   - Every pointer argument is a DEVICE pointer owned by the caller, except
 *     where a comment says "host".  The library never allocates, frees or
 *     retains memory; its only global state is one status word per device.
 *   - Device array pointers must be 16-byte aligned; the single-value
 *     pointers gamma64 / gamma32 need only their natural alignment
 *     (BL_ERR_ALIGN otherwise).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call only enqueues work on it and returns; results are
 *     ready when the stream reaches that point.
 *   - Arguments are validated on the host before anything is launched; a
 *     failed check returns its status and enqueues nothing.  A launch failure
 *     returns BL_ERR_CUDA.
 *   - Non-finite values met on the device (NaN/Inf in W or x) do not trap:
 *     they set the device status word, which bitlinear_get_status() returns.
 *   - Integer accumulation is int32, so K must satisfy 127 * K < 2^31
 *     (BL_ERR_OVERFLOW otherwise).
 *   - There is no bias term (the pages show none).
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BL_OK = 0,
    BL_ERR_NULL = 1,        /* a required pointer is NULL                         */
    BL_ERR_SHAPE = 2,       /* M, N or K out of range                              */
    BL_ERR_ALIGN = 3,       /* a device pointer is not 16-byte aligned             */
    BL_ERR_DTYPE = 4,       /* unknown bl_dtype value                              */
    BL_ERR_WORKSPACE = 5,   /* workspace smaller than the *_workspace_bytes() size */
    BL_ERR_OVERFLOW = 6,    /* 127 * K >= 2^31: int32 accumulator could overflow   */
    BL_ERR_NONFINITE = 7,   /* device saw NaN/Inf in W or x (from get_status)      */
    BL_ERR_CUDA = 8,        /* a CUDA runtime call or kernel launch failed          */
    BL_ERR_ARG = 9,         /* another argument is invalid (eps < 0, count <= 0)   */
    BL_ERR_TIMEOUT = 10     /* a kernel gave up a bounded wait (from get_status)    */
} bl_status;

typedef enum { BL_F32 = 0, BL_BF16 = 1 } bl_dtype;

/* ------------------------------------------------------------------------
 * Packed ternary weight layout (2 bits per weight, row-tiled, chunk-major;
 * 2 bits per weight as in bhfrc.com/news/56965 sec. 4.1).  Each weight is
 * stored as u = code + 1: 00 -> -1, 01 -> 0, 10 -> +1 (11 never occurs), so
 * a decoder only masks fields out.  Padding holds 01 (code 0).
 *   Kp = ceil(K/64)*64, Np = ceil(N/8)*8, C = Kp/64 sixteen-byte chunks/row.
 *   Weight (n, k) sits in byte  (n/8)*(8*C*16) + ((k/64)*8 + n%8)*16
 *                                + ((k%64)/16)*4 + k%4
 *   at bits 2*((k%16)/4) .. +1.  Padded positions (n >= N or k >= K) hold 01.
 * So each 8-row tile stores chunk c of its 8 rows as 128 contiguous bytes,
 * and a warp reads 4 chunks x 8 rows as one 512-byte coalesced span.
 * ---------------------------------------------------------------------- */

/* Padded reduction length Kp = ceil(K/64)*64 (the row stride of q). */
int64_t bitlinear_padded_k(int64_t K);

/* Bytes of the packed weight buffer: Np * Kp / 4.  Returns 0 if N or K <= 0. */
int64_t bitlinear_packed_bytes(int64_t N, int64_t K);

/* Bytes of scratch bitlinear_pack_weights needs (fp64 partial sums). */
int64_t bitlinear_pack_workspace_bytes(int64_t N, int64_t K);

/* ------------------------------------------------------------------------
 * bitlinear_pack_weights -- absmean quantisation of one weight tensor to
 * ternary codes and the 2-bit packed layout above (aratech.ae, "Ternary
 * weights {-1, 0, +1}": scale 1/mean|W|, then clip(-1, 1)(round(.)) ).
 *
 *   W         fp32 [N][K] row-major (nn.Linear weight: out x in), device.
 *   eps       >= 0, added to gamma (fp64) in the code decision only.
 *   packed    uint8 [bitlinear_packed_bytes(N, K)], device, written.
 *   gamma64   one double, device, written: mean|W| (fp64 accumulation in a
 *             fixed, run-to-run deterministic order).
 *   gamma32   one float, device, written: (float)gamma64, used by forward.
 *   workspace >= bitlinear_pack_workspace_bytes(N, K) bytes, device scratch.
 * The code decision |W|/(gamma+eps) > 1/2 is taken exactly (as in fp64).
 * Errors: NULL, SHAPE (N, K <= 0 or N*K >= 2^40), ALIGN, WORKSPACE, ARG
 * (eps < 0 or not finite), CUDA.  NaN/Inf in W sets BL_ERR_NONFINITE.
 * ---------------------------------------------------------------------- */
bl_status bitlinear_pack_weights(const float* W, int64_t N, int64_t K, double eps,
                                 uint8_t* packed, double* gamma64, float* gamma32,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * bitlinear_pack_weights_noalloc -- bitlinear_pack_weights without the
 * workspace argument.  The BitNet pages have no counterpart to this call;
 * it is an interface addition of this library.
 *
 * For callers that cannot allocate device memory where they call the
 * packer: for example a host framework's custom-operator hook that hands
 * over its tensors but no allocator, or a deployment that reserves all
 * device memory when it starts and forbids cudaMalloc afterwards (a
 * cudaMalloc can synchronise the device and breaks a fixed memory plan).
 *
 * Arguments, results and errors are those of bitlinear_pack_weights minus
 * the workspace.  The reduction's fp64 partial sums live instead in a
 * fixed 16,640-byte array of the library's own device memory, which every
 * GPU that loads the library holds until the process exits.
 *   - Nothing is allocated: no cudaMalloc/cudaFree, no allocating library.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.
 *   - Every call on a device uses the same array, so calls whose kernels
 *     overlap on the GPU (different streams with no ordering between them)
 *     race and give wrong results: order them on one stream or with events.
 *   - A size whose scratch would not fit the array returns
 *     BL_ERR_WORKSPACE; the reduction's block count is capped at 2048, so
 *     every N, K accepted by bitlinear_pack_weights fits.
 * ---------------------------------------------------------------------- */
bl_status bitlinear_pack_weights_noalloc(const float* W, int64_t N, int64_t K, double eps,
                                         uint8_t* packed, double* gamma64, float* gamma32,
                                         void* stream);

/* ------------------------------------------------------------------------
 * bitlinear_quant_act -- per-token absmax int8 quantisation (aratech.ae,
 * "BitLinear: the building block": each token's largest |activation| is
 * mapped to 127).
 *
 *   x   [M][K] row-major, fp32 (xt = BL_F32) or bf16 (xt = BL_BF16), device.
 *   q   int8 [M][Kp] row-major, Kp = bitlinear_padded_k(K), device, written;
 *       columns K..Kp-1 are written as 0.
 *   s   fp32 [M], device, written: s_m = 127 / max(max_k |x_mk|, 1e-5).
 * q_mk = clamp(rint(x_mk * s_m), -127, 127) in fp32 (IEEE divide, no FMA).
 * Errors: NULL, SHAPE (M, K <= 0), ALIGN, DTYPE, OVERFLOW, CUDA.
 * ---------------------------------------------------------------------- */
bl_status bitlinear_quant_act(const void* x, bl_dtype xt, int64_t M, int64_t K, int8_t* q,
                              float* s, void* stream);

/* ------------------------------------------------------------------------
 * bitlinear_forward -- ternary x int8 product with int32 accumulation
 * (bhfrc.com/news/56965 sec. 1.1: each weight adds, subtracts or skips an
 * activation) and the rescale y = acc * gamma / s.
 *
 *   q        int8 [M][Kp] from bitlinear_quant_act, device.
 *   s        fp32 [M] from bitlinear_quant_act, device.
 *   packed   from bitlinear_pack_weights (same N, K), device.
 *   gamma32  one float from bitlinear_pack_weights, device.
 *   y        [M][N] row-major, fp32 (yt = BL_F32) or bf16 (BL_BF16), device.
 *   acc_debug  NULL, or int32 [M][N] device buffer that receives acc.
 * fp32 y equals (float)((double)acc * gamma32 / s_m) for M <= 16 (decode
 * kernel).  The tensor-core kernel (M > 16) computes fp32(acc) * f_m with
 * f_m = gamma32 / s_m correctly rounded to fp32: two fp32 roundings, so y
 * is within 2^-23 relative of that value (bf16 y: equal after rounding
 * unless the fp32 value sits that close to a bf16 rounding midpoint).
 * Errors: NULL, SHAPE (M, N, K <= 0), ALIGN, DTYPE, OVERFLOW, CUDA.
 * ---------------------------------------------------------------------- */
bl_status bitlinear_forward(const int8_t* q, const float* s, const uint8_t* packed,
                            const float* gamma32, int64_t M, int64_t N, int64_t K, void* y,
                            bl_dtype yt, int32_t* acc_debug, void* stream);

/* ------------------------------------------------------------------------
 * bitlinear_forward_x -- the same layer with the activation quantisation
 * fused into the product kernel's prologue: x goes in, y comes out, q and s
 * never reach memory.  Results are identical to bitlinear_quant_act followed
 * by bitlinear_forward.  Arguments as in those two calls.
 * Limits of this fused decode form: M <= 16, and the quantised activations
 * of every problem must fit one CTA's shared memory: M' * Kp <= 160 KiB
 * (M' = M rounded up to a power of two; every decode kernel), or else
 * M' * Kp' <= 184 KiB with Kp' = Kp rounded up to a multiple of 4096 / M'
 * (the tensor-core decode kernel only; e.g. M = 16 at K = 11008).
 * Errors: NULL, SHAPE (M, N, K <= 0; the limits above; no kernel that the
 * decode-kernel setting allows fits the shapes), ALIGN, DTYPE, OVERFLOW,
 * CUDA.
 * ---------------------------------------------------------------------- */
bl_status bitlinear_forward_x(const void* x, bl_dtype xt, const uint8_t* packed,
                              const float* gamma32, int64_t M, int64_t N, int64_t K, void* y,
                              bl_dtype yt, void* stream);

/* Host-side query, no device work: 1 if the fused decode forms
 * (bitlinear_forward_x, _grouped, _rmsnorm_grouped) accept M tokens of K
 * columns under the limits above with BL_DECODE_AUTO, else 0 (also for M,
 * K out of range).  Lets a caller choose between the fused form and
 * bitlinear_quant_act + bitlinear_forward without trying. */
int bitlinear_forward_x_supported(int64_t M, int64_t K);

/* ------------------------------------------------------------------------
 * SubLN before the activation quantiser.  aratech.ae, "BitLinear: the
 * building block": a sub-layer normalisation, a simplified LayerNorm, sits
 * before the activation quantisation.  The page does not define it further;
 * it is read here as RMS normalisation with a per-channel gain g [K]:
 *   r = fp32(1 / sqrt(sum_k x_k^2 / K + eps))   (the sum in fp64)
 *   x_k <- (x_k * r) * g_k                       (fp32, rounded in that order)
 * followed by the per-token absmax quantiser of bitlinear_quant_act.  The
 * sum's order differs from a sequential sum by ~1e-16 relative, so r (and
 * then q, s) can differ from another implementation's only when r lies that
 * close to an fp32 rounding midpoint.
 *
 * bitlinear_rmsnorm_quant_act -- the normalisation and the quantiser in one
 *   kernel: arguments as bitlinear_quant_act plus gain (fp32 [K], device,
 *   16-byte aligned) and eps (>= 0, finite, else BL_ERR_ARG).
 * bitlinear_forward_x_rmsnorm_grouped -- the fused decode form of
 *   bitlinear_forward_x_grouped with the normalisation in the prologue; each
 *   problem i has its own x[i] and gain[i] (pass the same pointers for
 *   linears that share one normalised input).  Same limits as that call
 *   (bitlinear_forward_x); BL_ERR_SHAPE also when neither streaming decode
 *   kernel fits, or when the per-tile kernel is forced (it has no
 *   normalising prologue).
 * ---------------------------------------------------------------------- */
bl_status bitlinear_rmsnorm_quant_act(const void* x, bl_dtype xt, const float* gain, double eps, int64_t M,
                                      int64_t K, int8_t* q, float* s, void* stream);
bl_status bitlinear_forward_x_rmsnorm_grouped(int count, const void* const* x, bl_dtype xt,
                                              const float* const* gain, double eps, const uint8_t* const* packed,
                                              const float* const* gamma32, int64_t M, const int64_t* N,
                                              const int64_t* K, void* const* y, bl_dtype yt, void* stream);

/* ------------------------------------------------------------------------
 * Decode-kernel choice for M <= 16 (bitlinear_forward, bitlinear_forward_x,
 * bitlinear_forward_x_grouped).  Process-wide, host-side; set it before
 * launching (and before capturing a CUDA graph).  All kernels give the same
 * results; the setting exists to compare and test them.
 *   BL_DECODE_AUTO    M <= 4: dp4a streaming kernel, else tensor-core
 *                     kernel; M > 4: tensor-core kernel, else dp4a; else the
 *                     per-tile kernel -- whichever first fits the shapes
 *   BL_DECODE_TENSOR  tcgen05 kind::i8 kernel with the weights expanded
 *                     into tensor memory (one CTA per SM)
 *   BL_DECODE_DP4A    persistent streaming kernel, dp4a on the CUDA cores
 *   BL_DECODE_TILE    per-tile kernel (the fallback for the largest shapes)
 *   BL_DECODE_LUT     table-lookup kernel: per group of four activations,
 *                     the 16 subset sums; the packed fields' two bit planes
 *                     index them (aratech.ae, "How BitNet.cpp achieves its
 *                     speed"; devtrends.ru, "How does it work?": lookup
 *                     tables instead of matrix multiplications).  Only
 *                     bitlinear_forward with M = 1 and 8 * Kp <= ~196 KiB;
 *                     the fused calls return BL_ERR_SHAPE under it.  An A/B
 *                     counterpart: AUTO never selects it.
 * A forced TENSOR or DP4A choice that does not fit the shapes makes the
 * forward calls return BL_ERR_SHAPE.  bitlinear_set_decode_kernel returns
 * BL_OK, or BL_ERR_ARG for an unknown value.  The pages define no such
 * setting: it selects between implementations of the same product.
 * ---------------------------------------------------------------------- */
enum { BL_DECODE_AUTO = 0, BL_DECODE_TENSOR = 1, BL_DECODE_DP4A = 2, BL_DECODE_TILE = 3, BL_DECODE_LUT = 4 };
int bitlinear_set_decode_kernel(int kind);
int bitlinear_get_decode_kernel(void);

/* ------------------------------------------------------------------------
 * bitlinear_forward_x_grouped -- `count` independent fused BitLinear layers
 * (the linears of one transformer block) in ONE kernel launch.  Host arrays
 * of length `count` give each problem's device pointers and sizes, with the
 * meaning of bitlinear_forward_x.  All problems share M, xt and yt.
 * Errors: as bitlinear_forward_x, plus ARG (count < 1 or > 16).
 * ---------------------------------------------------------------------- */
bl_status bitlinear_forward_x_grouped(int count, const void* const* x, bl_dtype xt,
                                      const uint8_t* const* packed, const float* const* gamma32,
                                      int64_t M, const int64_t* N, const int64_t* K,
                                      void* const* y, bl_dtype yt, void* stream);

/* ------------------------------------------------------------------------
 * Workspace forms of the grouped fused decode calls: the same layer
 * (aratech.ae, "BitLinear: the building block": per-token absmax int8
 * activations, ternary weights, rescale), the same arguments, results (bit
 * for bit) and errors as bitlinear_forward_x_grouped and
 * bitlinear_forward_x_rmsnorm_grouped -- except that under BL_DECODE_TILE
 * the SubLN form runs for M >= 2 (on the codes) -- plus a device workspace (16-byte
 * aligned, caller-owned, at least bitlinear_decode_workspace_bytes(count,
 * M, K) bytes, else BL_ERR_WORKSPACE; NULL: BL_ERR_NULL) that the call may
 * overwrite, in stream order.  For M >= 2 the call quantises every token
 * row once, in a launch of its own (bitlinear_quant_act's kernel, over all
 * problems), into the workspace and then runs the product kernel on the
 * codes: in the single-launch form each CTA of the product kernel
 * quantises all M rows of its problem itself, reading x from L2 twice, which
 * costs more than a second launch once M > 1.  For M = 1 the workspace is
 * not touched and the call is the single-launch form.  Two calls in flight
 * at once (different streams) need different workspaces.
 *
 * bitlinear_decode_workspace_bytes -- the bytes those calls need: per
 * problem M * Kp bytes of codes and M fp32 scales, each rounded up to 256.
 * Host-only; 0 for count outside 1..16, K NULL, M outside 1..16 or a K
 * outside 1..16,909,320.
 * ---------------------------------------------------------------------- */
int64_t bitlinear_decode_workspace_bytes(int count, int64_t M, const int64_t* K);
bl_status bitlinear_forward_x_grouped_ws(int count, const void* const* x, bl_dtype xt,
                                         const uint8_t* const* packed, const float* const* gamma32, int64_t M,
                                         const int64_t* N, const int64_t* K, void* const* y, bl_dtype yt,
                                         void* workspace, int64_t workspace_bytes, void* stream);
bl_status bitlinear_forward_x_rmsnorm_grouped_ws(int count, const void* const* x, bl_dtype xt,
                                                 const float* const* gain, double eps,
                                                 const uint8_t* const* packed, const float* const* gamma32,
                                                 int64_t M, const int64_t* N, const int64_t* K, void* const* y,
                                                 bl_dtype yt, void* workspace, int64_t workspace_bytes,
                                                 void* stream);

/* Synchronises `stream`, then returns and clears the device status word of
 * the current device: BL_OK; BL_ERR_TIMEOUT if a kernel abandoned one of its
 * bounded waits (its outputs are then invalid); else BL_ERR_NONFINITE if a
 * kernel met NaN/Inf.  Returns BL_ERR_CUDA if the synchronisation failed. */
bl_status bitlinear_get_status(void* stream);

/* Static, human-readable name of a status value (never NULL). */
const char* bitlinear_status_string(bl_status status);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H */
