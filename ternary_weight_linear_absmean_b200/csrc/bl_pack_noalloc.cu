// bl_pack_noalloc.cu -- bitlinear_pack_weights for callers that cannot hand
// the library any device scratch memory.
//
// The absmean reduction behind bitlinear_pack_weights needs a small scratch
// buffer (one fp64 partial sum per reduction block plus the code threshold);
// the regular entry point takes it from the caller.  This variant keeps that
// scratch in a fixed array in the library's own device memory instead, so
// the call allocates nothing and needs nothing beyond its inputs and outputs.
//
// The array is file-scope `static __device__` storage: every GPU that loads
// the library holds it (kNoAllocScratchBytes) until the process exits.  On
// the host, the name g_pack_scratch is only a stand-in for the symbol, not a
// device address; the real address is looked up per device with
// cudaGetSymbolAddress the first time the entry point runs on that device
// (with that device current) and cached.
#include <mutex>

#include "bl_internal.cuh"

namespace {

// Largest scratch the reduction can use: at most 2048 fp64 partial sums
// (the block count is capped for every size) plus the threshold, padded.
constexpr size_t kNoAllocScratchBytes = 2048 * 8 + 256;

static __device__ __align__(256) unsigned char g_pack_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_pack_scratch on the current device, or NULL.
void* scratch_for_current_device()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_pack_scratch) != cudaSuccess || !p) return nullptr;
        g_scratch_addr[dev] = p;
    }
    return g_scratch_addr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" bl_status bitlinear_pack_weights_noalloc(const float* W, int64_t N, int64_t K, double eps,
                                                    uint8_t* packed, double* gamma64, float* gamma32,
                                                    void* stream)
{
    if (!W || !packed || !gamma64 || !gamma32) return BL_ERR_NULL;
    if (N <= 0 || K <= 0 || N > (int64_t(1) << 40) / K) return BL_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(packed) || (reinterpret_cast<uintptr_t>(gamma64) & 7u) ||
        (reinterpret_cast<uintptr_t>(gamma32) & 3u))
        return BL_ERR_ALIGN;
    if (!(eps >= 0.0) || !(eps < 1e308)) return BL_ERR_ARG;
    const int64_t count = N * K;
    const int blocks = bl::absmean_blocks(count);
    // partials (blocks * 8 bytes) followed by the fp32 threshold
    if ((size_t)blocks * 8 + 16 > kNoAllocScratchBytes) return BL_ERR_WORKSPACE;
    unsigned* status = bl::status_word_ptr();
    void* scratch = scratch_for_current_device();
    if (!status || !scratch) return BL_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    double* partial = static_cast<double*>(scratch);
    float* thr = reinterpret_cast<float*>(static_cast<char*>(scratch) + (size_t)blocks * 8);
    // every partial and the threshold are written before they are read, so
    // nothing left over from an earlier call needs clearing
    if (bl::launch_absmean_partial(W, count, partial, blocks, status, st) != cudaSuccess) return BL_ERR_CUDA;
    if (bl::launch_absmean_finalize(partial, blocks, count, eps, gamma64, gamma32, thr, st) != cudaSuccess)
        return BL_ERR_CUDA;
    if (bl::launch_pack(W, N, K, thr, packed, st) != cudaSuccess) return BL_ERR_CUDA;
    return BL_OK;
}
