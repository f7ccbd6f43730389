/*
 * philox_oracle.c -- the oracle side's own Philox4x32-10 and the synthetic
 * weight recipe of the 100B-class decode sweep.
 *
 * TEST INFRASTRUCTURE ONLY (see bitlinear_oracle.c).  The weights of that
 * sweep (68 billion values) cannot be generated on the host and copied to
 * the device, so each side generates them from the same published
 * counter-based generator; this file is the oracle's implementation, written
 * from the definition in
 *   J. Salmon, M. Moraes, R. Dror, D. Shaw, "Parallel Random Numbers: As
 *   Easy as 1, 2, 3", SC'11 (Philox-4x32, 10 rounds),
 * and checked against that paper's published known-answer vectors.
 *
 * Weight recipe (element e = n*K + k of matrix `g`, generator `seed`):
 *   p = e / 2, h = e % 2
 *   out = Philox4x32-10(counter = (p mod 2^32, p / 2^32, g, 0), key = (seed, 0))
 *   a = out[2h], b = out[2h+1];  halves h0 = a & 0xFFFF, h1 = a >> 16,
 *                                        h2 = b & 0xFFFF, h3 = b >> 16
 *   u_i = (h_i + 0.5) * 2^-16                 (exact in fp32)
 *   z   = ((u0 + u1) + (u2 + u3)) - 2         (exact in fp32)
 *   w   = z * 0.02*sqrt(3) (fp32 constant 0x3d0de3bd; one rounding)
 * z is an Irwin-Hall(4) variable centred at 0 with variance 1/3, so w has
 * mean 0 and standard deviation 0.02, the N(0, 0.02) weights of the workload.
 */
#include <stdint.h>
#include <string.h>

static const uint32_t PHILOX_M0 = 0xD2511F53u, PHILOX_M1 = 0xCD9E8D57u;
static const uint32_t PHILOX_W0 = 0x9E3779B9u, PHILOX_W1 = 0xBB67AE85u;

void orc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { k0 += PHILOX_W0; k1 += PHILOX_W1; }   /* key schedule */
        uint64_t p0 = (uint64_t)PHILOX_M0 * c0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * c2;
        uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
        uint32_t n1 = (uint32_t)p1;
        uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        uint32_t n3 = (uint32_t)p0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

static float orc_synth_scale(void)
{
    uint32_t bits = 0x3d0de3bdu;   /* fp32 nearest to 0.02 * sqrt(3) */
    float f;
    memcpy(&f, &bits, 4);
    return f;
}

/* Weights of rows [row0, row0 + rows) of matrix g (row length K). */
void orc_synth_weights(uint32_t seed, uint32_t g, int64_t row0, int64_t rows, int64_t K, float* W)
{
    const float scale = orc_synth_scale();
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            uint64_t e = (uint64_t)(row0 + r) * (uint64_t)K + (uint64_t)k;
            uint64_t p = e >> 1;
            unsigned h = (unsigned)(e & 1u);
            uint32_t ctr[4] = {(uint32_t)p, (uint32_t)(p >> 32), g, 0u};
            uint32_t key[2] = {seed, 0u};
            uint32_t out[4];
            orc_philox4x32_10(ctr, key, out);
            uint32_t a = out[2 * h], b = out[2 * h + 1];
            float u0 = ((float)(a & 0xFFFFu) + 0.5f) * 0x1p-16f;
            float u1 = ((float)(a >> 16) + 0.5f) * 0x1p-16f;
            float u2 = ((float)(b & 0xFFFFu) + 0.5f) * 0x1p-16f;
            float u3 = ((float)(b >> 16) + 0.5f) * 0x1p-16f;
            float z = ((u0 + u1) + (u2 + u3)) - 2.0f;
            W[r * K + k] = z * scale;
        }
    }
}

/* Same recipe, rows split over POSIX threads (generation only). */
#include <pthread.h>
typedef struct { uint32_t seed, g; int64_t row0, rows, K; float* W; } orc_synth_job;
static void* orc_synth_worker(void* arg)
{
    orc_synth_job* j = (orc_synth_job*)arg;
    orc_synth_weights(j->seed, j->g, j->row0, j->rows, j->K, j->W);
    return NULL;
}
void orc_synth_weights_mt(uint32_t seed, uint32_t g, int64_t row0, int64_t rows, int64_t K,
                          float* W, int threads)
{
    if (threads < 1) threads = 1;
    if (threads > 256) threads = 256;
    pthread_t tid[256];
    int created[256];
    orc_synth_job job[256];
    int64_t per = (rows + threads - 1) / threads;
    int jobs = 0;
    for (int t = 0; t < threads; ++t) {
        int64_t r0 = t * per, r1 = r0 + per < rows ? r0 + per : rows;
        if (r0 >= r1) break;
        job[t] = (orc_synth_job){seed, g, row0 + r0, r1 - r0, K, W + r0 * K};
        created[t] = pthread_create(&tid[t], NULL, orc_synth_worker, &job[t]) == 0;
        if (!created[t]) orc_synth_worker(&job[t]);
        jobs = t + 1;
    }
    for (int t = 0; t < jobs; ++t)
        if (created[t]) pthread_join(tid[t], NULL);
}
