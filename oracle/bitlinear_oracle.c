/*
 * bitlinear_oracle.c -- plain, slow, obviously-correct CPU statement of the
 * BitNet b1.58 BitLinear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file.  Only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or constant
 * generator with the CUDA library.
 *
 * Sources (web pages; cited by title and section):
 *   [ARATECH] "BitNet b1.58: Microsoft's 1-bit LLM that runs a 100B model on
 *             a single CPU" (aratech.ae, Arabic), sections
 *             "Ternary weights {-1, 0, +1}" and "BitLinear: the building block".
 *   [BHFRC]   "BitNet b1.58 on Windows: sm_86 kernels + AVX2" build notes
 *             (bhfrc.com/news/56965, Chinese), sec. 1.1 (ternary weights turn
 *             each multiply into add / subtract / skip) and sec. 4.1 (2 bits
 *             per weight, packed for wide loads).
 *
 * Readings taken where the pages are silent:
 *   R1  eps = 1e-5 (caller-chosen), added to gamma in fp64, used only for the
 *       codes; the rescale uses gamma itself.
 *   R2  "round" is IEEE round-half-to-even (rint).
 *   R3  one gamma per weight tensor.
 *   R4  activation amax is clamped to >= 1e-5 so an all-zero row gives q = 0.
 *   R5  activation codes are clamped to [-127, 127]; the clamp never binds
 *       (|x*s| <= 127*(1+2^-23)), and the oracle counts any element where it
 *       would have.
 *   R6  s = 127 / amax is a multiplier, so the rescale divides by s.
 *   R10 y is fp32: (float)((double)acc * (double)gamma32 / (double)s).
 *   R16 SubLN = RMS normalisation with a per-channel gain; the mean square
 *       is summed in fp64 and the factor rounded once to fp32 (see
 *       orc_rms_factor).
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared
 * (no FMA contraction: every float operation below rounds exactly once, in
 * the order written.)
 */
#include <math.h>
#include <pthread.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* A1: absmean weight scale.                                                */
/* [ARATECH] "Ternary weights": the scale is the inverse of the mean of the */
/* absolute value over the whole weight tensor, scale_w = 1 / mean(|W_ij|). */
/* gamma = mean |W_ij|, summed left to right in fp64 (one tensor, R3).      */
/* ------------------------------------------------------------------------ */
double orc_absmean_gamma(const float* W, int64_t N, int64_t K)
{
    if (N <= 0 || K <= 0) return 0.0;
    double sum = 0.0;
    for (int64_t i = 0; i < N * K; ++i) sum += fabs((double)W[i]);
    return sum / (double)(N * K);
}

/* ------------------------------------------------------------------------ */
/* A1: ternary codes.                                                       */
/* [ARATECH] "Ternary weights": W_q = clip(-1, 1)(round(W * scale_w)).      */
/* With gamma + eps in place of mean|W| (R1) and round = rint (R2):         */
/*   r = W / (gamma + eps)  (fp64),  code = clamp(rint(r), -1, 1).          */
/* boundary[i] = 1 where |r| lies within 1e-6 of the 0.5 rounding boundary; */
/* such codes are the only ones two correct implementations may disagree    */
/* on (different fp64 summation orders for gamma).  Returns their count.    */
/* ------------------------------------------------------------------------ */
int64_t orc_ternary_codes(const float* W, int64_t N, int64_t K, double gamma64,
                          double eps, int8_t* code, uint8_t* boundary)
{
    const double d = gamma64 + eps;
    int64_t n_boundary = 0;
    for (int64_t i = 0; i < N * K; ++i) {
        double r = (double)W[i] / d;
        double c = rint(r);
        if (c > 1.0) c = 1.0;
        if (c < -1.0) c = -1.0;
        code[i] = (int8_t)c;
        int near = fabs(fabs(r) - 0.5) <= 1e-6;
        if (boundary) boundary[i] = (uint8_t)near;
        n_boundary += near;
    }
    return n_boundary;
}

/* ------------------------------------------------------------------------ */
/* A2: 2-bit packed weight layout ("row-tiled, chunk-major"), as specified */
/* in include/bitlinear.h.  Each weight is stored as u = code + 1:           */
/* 00 -> -1, 01 -> 0, 10 -> +1; padding is 01 (code 0); 11 never occurs.    */
/* (The BitNet pages' CPU kernel ([BHFRC] sec. 4.1) uses a different 2-bit  */
/* table, 00 -> 0, 01 -> +1, 10 -> -1, 11 -> padding; storing code + 1 is   */
/* this layout's choice, so decoding needs masking only.)                   */
/*                                                                          */
/* Geometry (the library implements the same spec independently):          */
/*   Kp = ceil(K / 64) * 64            padded reduction length              */
/*   Np = ceil(N / 8) * 8              padded output rows                   */
/*   C  = Kp / 64                      16-byte chunks per row               */
/*   row tile  tau = n / 8, r = n % 8                                       */
/*   chunk c = k / 64; within it word i = (k % 64) / 16,                    */
/*   field t = (k % 16) / 4, byte b = k % 4                                 */
/*   byte offset = tau * (8 * C * 16) + (c * 8 + r) * 16 + i * 4 + b        */
/*   bit offset within that byte = 2 * t                                    */
/* Padded positions (k >= K or n >= N) hold 01.                             */
/* ------------------------------------------------------------------------ */
int64_t orc_padded_k(int64_t K) { return (K + 63) / 64 * 64; }
int64_t orc_padded_n(int64_t N) { return (N + 7) / 8 * 8; }
int64_t orc_packed_bytes(int64_t N, int64_t K) { return orc_padded_n(N) * orc_padded_k(K) / 4; }

static int64_t orc_code_byte_offset(int64_t n, int64_t k, int64_t K)
{
    const int64_t C = orc_padded_k(K) / 64;
    const int64_t tau = n / 8, r = n % 8;
    const int64_t c = k / 64, i = (k % 64) / 16, b = k % 4;
    return tau * (8 * C * 16) + (c * 8 + r) * 16 + i * 4 + b;
}
static int orc_code_bit_offset(int64_t k) { return (int)(2 * ((k % 16) / 4)); }

static uint8_t orc_code_to_bits(int8_t c) { return (uint8_t)(c + 1); }   /* -1,0,+1 -> 0,1,2 */

void orc_pack(const int8_t* code, int64_t N, int64_t K, uint8_t* packed)
{
    const int64_t Np = orc_padded_n(N), Kp = orc_padded_k(K);
    memset(packed, 0x55, (size_t)orc_packed_bytes(N, K));   /* all 01 = padding */
    for (int64_t n = 0; n < Np; ++n) {
        for (int64_t k = 0; k < Kp; ++k) {
            uint8_t bits = (n < N && k < K) ? orc_code_to_bits(code[n * K + k]) : 1u;
            int64_t off = orc_code_byte_offset(n, k, K);
            int sh = orc_code_bit_offset(k);
            packed[off] = (uint8_t)((packed[off] & ~(3u << sh)) | (bits << sh));
        }
    }
}

/* Inverse of orc_pack.  Returns the number of malformed fields found:      */
/* any 11, or a padded position not holding 01.                             */
int64_t orc_unpack(const uint8_t* packed, int64_t N, int64_t K, int8_t* code)
{
    const int64_t Np = orc_padded_n(N), Kp = orc_padded_k(K);
    int64_t bad = 0;
    for (int64_t n = 0; n < Np; ++n) {
        for (int64_t k = 0; k < Kp; ++k) {
            int64_t off = orc_code_byte_offset(n, k, K);
            unsigned bits = (packed[off] >> orc_code_bit_offset(k)) & 3u;
            if (n < N && k < K) {
                if (bits == 3u) ++bad;
                code[n * K + k] = (int8_t)((int)bits - 1);
            } else if (bits != 1u) {
                ++bad;
            }
        }
    }
    return bad;
}

/* ------------------------------------------------------------------------ */
/* A3: per-token absmax int8 activation quantisation.                       */
/* [ARATECH] "BitLinear": activations are quantised to INT8 with absmax,    */
/* per token, so that each row's largest |activation| lands on 127.         */
/*   amax_m = max_k |x_mk|, clamped to >= 1e-5 (R4)                         */
/*   s_m    = 127 / amax_m              (fp32, IEEE division)               */
/*   q_mk   = clamp(rintf(x_mk * s_m), -127, 127)   (fp32 multiply, R5)     */
/* Returns the number of elements where the clamp changed the value.        */
/* ------------------------------------------------------------------------ */
static int64_t orc_quant_row(const float* x, int64_t K, int8_t* q, float* s_out)
{
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(x[k]);
        if (a > amax) amax = a;
    }
    if (amax < 1e-5f) amax = 1e-5f;
    const float s = 127.0f / amax;
    int64_t clipped = 0;
    for (int64_t k = 0; k < K; ++k) {
        float v = rintf(x[k] * s);
        if (v > 127.0f) { v = 127.0f; ++clipped; }
        if (v < -127.0f) { v = -127.0f; ++clipped; }
        q[k] = (int8_t)v;
    }
    *s_out = s;
    return clipped;
}

int64_t orc_quant_act_f32(const float* x, int64_t M, int64_t K, int8_t* q, float* s)
{
    int64_t clipped = 0;
    for (int64_t m = 0; m < M; ++m) clipped += orc_quant_row(x + m * K, K, q + m * K, s + m);
    return clipped;
}

/* bf16 -> fp32 widening is exact: the bf16 bits are the high half. */
static float orc_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

int64_t orc_quant_act_bf16(const uint16_t* x, int64_t M, int64_t K, int8_t* q, float* s)
{
    float* row = (float*)malloc((size_t)K * sizeof(float));
    if (!row) return -1;
    int64_t clipped = 0;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) row[k] = orc_bf16_to_f32(x[m * K + k]);
        clipped += orc_quant_row(row, K, q + m * K, s + m);
    }
    free(row);
    return clipped;
}

/* ------------------------------------------------------------------------ */
/* SubLN before the activation quantiser.                                   */
/* [ARATECH] "BitLinear: the building block": a sub-layer normalisation, a  */
/* simplified variant of LayerNorm, sits before the activation quantisation */
/* for training stability; the page does not define it further.  Reading   */
/* R16: the simplified LayerNorm is RMS normalisation (no mean subtraction, */
/* no bias) with a per-channel gain g:                                      */
/*   ms   = (sum_k x_k^2) / K           fp64 (each square is exact in fp64, */
/*                                      summed left to right)               */
/*   r    = 1 / sqrt(ms + eps)          fp64, then rounded to fp32 (r32)    */
/*   xn_k = (x_k * r32) * g_k           fp32, two roundings, in that order  */
/* and xn is then quantised exactly like x (orc_quant_row).                 */
/* ------------------------------------------------------------------------ */
float orc_rms_factor(const float* x, int64_t K, double eps)
{
    double ss = 0.0;
    for (int64_t k = 0; k < K; ++k) ss += (double)x[k] * (double)x[k];
    const double r = 1.0 / sqrt(ss / (double)K + eps);
    return (float)r;
}

void orc_rmsnorm_row(const float* x, int64_t K, const float* g, double eps, float* xn)
{
    const float r32 = orc_rms_factor(x, K, eps);
    for (int64_t k = 0; k < K; ++k) {
        const float t = x[k] * r32;   /* rounds once (no contraction) */
        xn[k] = t * g[k];             /* rounds once */
    }
}

/* x given as fp32 (xt = 0) or bf16 bit patterns (xt = 1); writes the fp32   */
/* normalised rows, then q and s as orc_quant_act_*.  Returns the clipped    */
/* count, or -1 on allocation failure.                                       */
int64_t orc_rmsnorm_quant_act(const void* x, int xt, const float* g, double eps, int64_t M, int64_t K,
                              float* xn, int8_t* q, float* s)
{
    float* row = (float*)malloc((size_t)K * sizeof(float));
    if (!row) return -1;
    int64_t clipped = 0;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k)
            row[k] = xt ? orc_bf16_to_f32(((const uint16_t*)x)[m * K + k]) : ((const float*)x)[m * K + k];
        orc_rmsnorm_row(row, K, g, eps, xn + m * K);
        clipped += orc_quant_row(xn + m * K, K, q + m * K, s + m);
    }
    free(row);
    return clipped;
}

/* ------------------------------------------------------------------------ */
/* A4: ternary x int8 product with integer accumulation.                    */
/* [BHFRC] sec. 1.1: with ternary weights every product is "+x, -x or       */
/* nothing", so the matrix product needs only integer adds.                 */
/*   acc_mn = sum_k q_mk * code_nk   (int64, then checked to fit int32)     */
/* Returns 0, or -1 if some |acc| exceeds INT32_MAX.                        */
/* ------------------------------------------------------------------------ */
int orc_int_matmul(const int8_t* q, const int8_t* code, int64_t M, int64_t N, int64_t K,
                   int32_t* acc)
{
    int overflow = 0;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t a = 0;
            for (int64_t k = 0; k < K; ++k) a += (int64_t)q[m * K + k] * (int64_t)code[n * K + k];
            if (a > INT32_MAX || a < -(int64_t)INT32_MAX) overflow = 1;
            acc[m * N + n] = (int32_t)a;
        }
    }
    return overflow ? -1 : 0;
}

/* Same product for a list of sampled (m, n) output positions only. */
int orc_int_matmul_sampled(const int8_t* q, const int8_t* code, int64_t K,
                           const int64_t* ms, const int64_t* ns, int64_t count, int32_t* acc)
{
    int overflow = 0;
    for (int64_t i = 0; i < count; ++i) {
        int64_t a = 0;
        for (int64_t k = 0; k < K; ++k)
            a += (int64_t)q[ms[i] * K + k] * (int64_t)code[ns[i] * K + k];
        if (a > INT32_MAX || a < -(int64_t)INT32_MAX) overflow = 1;
        acc[i] = (int32_t)a;
    }
    return overflow ? -1 : 0;
}

/* ------------------------------------------------------------------------ */
/* A5: rescale.  W ~ gamma * code and x ~ q / s, so                         */
/*   y_mn = acc_mn * gamma32 / s_m   evaluated in fp64, rounded to fp32.    */
/* gamma32 = (float)gamma64 (round to nearest even).                        */
/* ------------------------------------------------------------------------ */
float orc_rescale_one(int32_t acc, float gamma32, float s)
{
    return (float)((double)acc * (double)gamma32 / (double)s);
}

void orc_rescale(const int32_t* acc, const float* s, float gamma32, int64_t M, int64_t N, float* y)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) y[m * N + n] = orc_rescale_one(acc[m * N + n], gamma32, s[m]);
}

/* fp32 -> bf16, round to nearest, ties to even (NaN kept quiet). */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

void orc_to_bf16(const float* y, int64_t count, uint16_t* out)
{
    for (int64_t i = 0; i < count; ++i) out[i] = orc_f32_to_bf16(y[i]);
}

/* ------------------------------------------------------------------------ */
/* Whole layer, for the CPU baseline timing: quantise x, multiply, rescale. */
/* Rows of the output are split over `threads` POSIX threads (plain loops   */
/* per thread, no blocking).  codes are the A1 result, unpacked int8.       */
/* ------------------------------------------------------------------------ */
typedef struct {
    const int8_t* q; const int8_t* code; const float* s; float gamma32;
    int64_t M, N, K, n0, n1; float* y; int overflow;
} orc_fwd_job;

static void* orc_fwd_worker(void* arg)
{
    orc_fwd_job* j = (orc_fwd_job*)arg;
    for (int64_t m = 0; m < j->M; ++m) {
        for (int64_t n = j->n0; n < j->n1; ++n) {
            int64_t a = 0;
            for (int64_t k = 0; k < j->K; ++k)
                a += (int64_t)j->q[m * j->K + k] * (int64_t)j->code[n * j->K + k];
            if (a > INT32_MAX || a < -(int64_t)INT32_MAX) j->overflow = 1;
            j->y[m * j->N + n] = orc_rescale_one((int32_t)a, j->gamma32, j->s[m]);
        }
    }
    return NULL;
}

int orc_forward_bf16_mt(const uint16_t* x, const int8_t* code, float gamma32, int64_t M,
                        int64_t N, int64_t K, float* y, int threads, int8_t* q_scratch,
                        float* s_scratch)
{
    if (threads < 1) threads = 1;
    if (orc_quant_act_bf16(x, M, K, q_scratch, s_scratch) < 0) return -2;
    if (threads > 256) threads = 256;
    pthread_t tid[256];
    int created[256];
    orc_fwd_job job[256];
    int64_t per = (N + threads - 1) / threads;
    int jobs = 0;
    for (int t = 0; t < threads; ++t) {
        int64_t n0 = t * per, n1 = n0 + per < N ? n0 + per : N;
        if (n0 >= n1) break;
        job[t] = (orc_fwd_job){q_scratch, code, s_scratch, gamma32, M, N, K, n0, n1, y, 0};
        created[t] = pthread_create(&tid[t], NULL, orc_fwd_worker, &job[t]) == 0;
        if (!created[t]) orc_fwd_worker(&job[t]);
        jobs = t + 1;
    }
    int overflow = 0;
    for (int t = 0; t < jobs; ++t) {
        if (created[t]) pthread_join(tid[t], NULL);
        overflow |= job[t].overflow;
    }
    return overflow ? -1 : 0;
}
