// synth_philox.cu -- GPU side of the synthetic-input generator for the
// 100B-class decode sweep: Philox4x32-10 (J. Salmon, M. Moraes, R. Dror,
// D. Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11) and the
// weight recipe below, written from that definition.  The CPU oracle has its
// own implementation; the two share no code and are each checked against
// the paper's published known-answer vectors.
//
// This library only draws inputs.  It is not part of the BitLinear library
// and holds none of the layer's arithmetic.
//
// Weight recipe (element e = n*K + k of matrix g, generator key `seed`):
//   p = e / 2, h = e % 2
//   out = Philox4x32-10(counter = (p mod 2^32, p / 2^32, g, 0), key = (seed, 0))
//   a = out[2h], b = out[2h+1];  16-bit halves h0 = a & 0xFFFF, h1 = a >> 16,
//                                               h2 = b & 0xFFFF, h3 = b >> 16
//   u_i = (h_i + 0.5) * 2^-16, z = ((u0 + u1) + (u2 + u3)) - 2   (exact)
//   w = z * 0x1.1bc77ap-5  (fp32 nearest 0.02*sqrt(3); the only rounding)
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ void philox10(uint32_t c[4], uint32_t k0, uint32_t k1)
{
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint32_t lo0 = 0xD2511F53u * c[0], hi0 = __umulhi(0xD2511F53u, c[0]);
        const uint32_t lo1 = 0xCD9E8D57u * c[2], hi1 = __umulhi(0xCD9E8D57u, c[2]);
        const uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
        c[0] = n0;
        c[1] = lo1;
        c[2] = n2;
        c[3] = lo0;
    }
}

__device__ __forceinline__ float uni16(uint32_t h) { return __fmul_rn(__fadd_rn((float)h, 0.5f), 0x1p-16f); }

__device__ __forceinline__ float weight_from(uint32_t a, uint32_t b)
{
    const float u0 = uni16(a & 0xFFFFu), u1 = uni16(a >> 16), u2 = uni16(b & 0xFFFFu), u3 = uni16(b >> 16);
    const float z = __fsub_rn(__fadd_rn(__fadd_rn(u0, u1), __fadd_rn(u2, u3)), 2.0f);
    return __fmul_rn(z, 0x1.1bc77ap-5f);
}

// one thread per pair of consecutive elements (one Philox call)
__global__ void synth_weights_kernel(float* __restrict__ W, uint32_t seed, uint32_t g, uint64_t e0,
                                     uint64_t count)
{
    const uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;   // local pair index
    const uint64_t first = e0 + 2 * i - (e0 & 1);                        // first element of the pair
    if (2 * i >= count + (e0 & 1)) return;
    const uint64_t p = first >> 1;
    uint32_t c[4] = {(uint32_t)p, (uint32_t)(p >> 32), g, 0u};
    philox10(c, seed, 0u);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint64_t e = first + h;
        if (e < e0 || e >= e0 + count) continue;
        W[e - e0] = weight_from(c[2 * h], c[2 * h + 1]);
    }
}

__global__ void philox_kat_kernel(const uint32_t* __restrict__ in, uint32_t* __restrict__ out, int n)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    uint32_t c[4] = {in[6 * i], in[6 * i + 1], in[6 * i + 2], in[6 * i + 3]};
    philox10(c, in[6 * i + 4], in[6 * i + 5]);
    for (int j = 0; j < 4; ++j) out[4 * i + j] = c[j];
}

}  // namespace

// Elements [row0*K, (row0+rows)*K) of matrix g into W (device, fp32).
extern "C" int synth_weights_device(float* W, uint32_t seed, uint32_t g, int64_t row0, int64_t rows, int64_t K,
                                    void* stream)
{
    if (!W || rows <= 0 || K <= 0 || row0 < 0) return 1;
    const uint64_t e0 = (uint64_t)row0 * (uint64_t)K, count = (uint64_t)rows * (uint64_t)K;
    const uint64_t pairs = (count + (e0 & 1) + 1) / 2;
    const unsigned threads = 256;
    const uint64_t blocks = (pairs + threads - 1) / threads;
    if (blocks > 0x7FFFFFFFull) return 2;
    synth_weights_kernel<<<(unsigned)blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(W, seed, g, e0,
                                                                                               count);
    return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

// n vectors of (ctr0..3, key0, key1) -> Philox4x32-10 outputs (device arrays).
extern "C" int synth_philox_device(const uint32_t* in, uint32_t* out, int n, void* stream)
{
    if (!in || !out || n <= 0) return 1;
    philox_kat_kernel<<<(n + 127) / 128, 128, 0, static_cast<cudaStream_t>(stream)>>>(in, out, n);
    return cudaGetLastError() == cudaSuccess ? 0 : 3;
}
