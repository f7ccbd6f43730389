// bl_api.cu -- the C ABI of include/bitlinear.h: host-side argument checks,
// the per-device status word, and dispatch to the kernels.
#include <atomic>
#include <cmath>
#include <cstring>

#include "bl_internal.cuh"
#include "bl_ptx.cuh"

// One status word per device (device-side state of the library).
__device__ unsigned int g_bl_status_word;

namespace {

// Decode-kernel choice of bitlinear_set_decode_kernel (host-side, process-wide).
std::atomic<int> g_decode_kernel{BL_DECODE_AUTO};

constexpr int64_t kMaxK = (int64_t(1) << 31) / 127;   // 127*K must stay < 2^31
constexpr size_t kFusedSmemLimit = 160 * 1024;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned_to(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Decode (M <= 16) kernel choice.  AUTO: the dp4a streaming kernel up to 4
// tokens (measured faster there: its per-byte cost grows with M but starts
// below the tensor-core kernel's, which is bound by tcgen05 issue), the
// tensor-core kernel above; each falls back to the next when the shapes do
// not fit its shared memory.  Returns kTryNext when the per-tile kernel
// should run.
constexpr bl_status kTryNext = static_cast<bl_status>(-1);

bl_status dispatch_decode(bl::StreamBatch& sb, bool fused, bl_dtype xt, bl_dtype yt, unsigned* status,
                          cudaStream_t cs)
{
    const int kind = g_decode_kernel.load();
    if (kind == BL_DECODE_TILE) return kTryNext;
    if (kind == BL_DECODE_LUT) return BL_ERR_SHAPE;   // unfused form only
    const bool tensor_first = kind == BL_DECODE_TENSOR || (kind == BL_DECODE_AUTO && sb.M > 4);
    for (int pass = 0; pass < 2; ++pass) {
        const bool tensor = (pass == 0) == tensor_first;
        if (kind == BL_DECODE_TENSOR && !tensor) break;
        if (kind == BL_DECODE_DP4A && tensor) continue;
        bl::StreamBatch b = sb;   // each planner fills its own plan fields
        const cudaError_t e = tensor ? bl::launch_dec_tc(b, fused, xt, yt, status, cs)
                                     : bl::launch_stream(b, fused, xt, yt, status, cs);
        if (e != cudaErrorNotSupported) return e == cudaSuccess ? BL_OK : BL_ERR_CUDA;
    }
    return kind == BL_DECODE_AUTO ? kTryNext : BL_ERR_SHAPE;
}

unsigned* status_word()
{
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bl_status_word) != cudaSuccess) return nullptr;
    return static_cast<unsigned*>(p);
}

int pow2_tokens(int64_t M)
{
    return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16;
}

bl_status check_dtype(bl_dtype t) { return (t == BL_F32 || t == BL_BF16) ? BL_OK : BL_ERR_DTYPE; }

bl_status check_forward_shape(int64_t M, int64_t N, int64_t K)
{
    if (M <= 0 || N <= 0 || K <= 0) return BL_ERR_SHAPE;
    if (M > (int64_t(1) << 31) || N > (int64_t(1) << 31)) return BL_ERR_SHAPE;
    if (K > kMaxK) return BL_ERR_OVERFLOW;
    if ((bl::padded_n(N) / 8) > (int64_t(1) << 30)) return BL_ERR_SHAPE;
    return BL_OK;
}

// Workspace of the calls that quantise in a launch of their own: per
// problem its int8 codes [M][Kp], then its fp32 scales [M], each at a
// 256-byte aligned offset.  Returns the total; fills the pointers if given.
int64_t ws_layout(int count, int64_t M, const int64_t* K, void* ws, int8_t** q, float** s)
{
    auto up = [](int64_t v) { return (v + 255) / 256 * 256; };
    int64_t off = 0;
    for (int i = 0; i < count; ++i) {
        if (q) q[i] = reinterpret_cast<int8_t*>(static_cast<char*>(ws) + off);
        off += up(M * bl::padded_k(K[i]));
        if (s) s[i] = reinterpret_cast<float*>(static_cast<char*>(ws) + off);
        off += up(4 * M);
    }
    return off;
}

// Token count from which the calls given a workspace quantise every row
// once, in a launch of their own, and run the product kernel on the codes:
// each CTA of a fused product kernel quantises all M rows itself, so the
// CTAs together read x (M x K) twice each from L2, which costs more than a
// second launch once M > 1.
constexpr int64_t kSplitMinM = 2;

// The grouped fused decode calls (bitlinear_forward_x_grouped and its
// SubLN and workspace forms).  gain: NULL, or one gain vector per problem.
bl_status grouped_decode(int count, const void* const* x, bl_dtype xt, const float* const* gain, double eps,
                         const uint8_t* const* packed, const float* const* gamma32, int64_t M, const int64_t* N,
                         const int64_t* K, void* const* y, bl_dtype yt, void* ws, int64_t ws_bytes, bool has_ws,
                         void* stream)
{
    if (count < 1 || count > bl::kMaxGroup) return BL_ERR_ARG;
    if (!x || !packed || !gamma32 || !N || !K || !y) return BL_ERR_NULL;
    if (check_dtype(xt) != BL_OK || check_dtype(yt) != BL_OK) return BL_ERR_DTYPE;
    if (M <= 0 || M > bl::kFusedMaxM) return BL_ERR_SHAPE;
    if (gain && (!(eps >= 0.0) || !std::isfinite(eps))) return BL_ERR_ARG;
    bl::GemvBatch b;
    std::memset(&b, 0, sizeof(b));
    b.count = count;
    b.M = M;
    int64_t tiles = 0;
    bool tile_fits = true;   // the per-tile kernel holds M' * Kp of activations in shared memory
    for (int i = 0; i < count; ++i) {
        if (!x[i] || !packed[i] || !gamma32[i] || !y[i] || (gain && !gain[i])) return BL_ERR_NULL;
        bl_status st = check_forward_shape(M, N[i], K[i]);
        if (st != BL_OK) return st;
        if ((size_t)pow2_tokens(M) * (size_t)bl::padded_k(K[i]) > kFusedSmemLimit) {
            if (!bl::dec_tc_fits(M, K[i])) return BL_ERR_SHAPE;   // no decode kernel holds its activations
            tile_fits = false;
        }
        if (!aligned16(x[i]) || !aligned16(packed[i]) || !aligned_to(gamma32[i], 4) || !aligned16(y[i]) ||
            (gain && !aligned16(gain[i])))
            return BL_ERR_ALIGN;
        tiles += bl::padded_n(N[i]) / 8;
        b.p[i].x = x[i];
        b.p[i].packed = packed[i];
        b.p[i].gamma32 = gamma32[i];
        b.p[i].y = y[i];
        b.p[i].N = N[i];
        b.p[i].K = K[i];
    }
    if (tiles > (int64_t(1) << 31) - 1) return BL_ERR_SHAPE;
    if (has_ws) {
        if (!ws) return BL_ERR_NULL;
        if (!aligned16(ws)) return BL_ERR_ALIGN;
        if (ws_bytes < ws_layout(count, M, K, nullptr, nullptr, nullptr)) return BL_ERR_WORKSPACE;
    }
    unsigned* status = status_word();
    if (!status) return BL_ERR_CUDA;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    bl::StreamBatch sb;
    std::memset(&sb, 0, sizeof(sb));
    sb.count = count;
    sb.M = (int)M;
    sb.eps_norm = eps;
    for (int i = 0; i < count; ++i) {
        sb.p[i].x = x[i];
        sb.p[i].gain = gain ? gain[i] : nullptr;
        sb.p[i].packed = packed[i];
        sb.p[i].gamma32 = gamma32[i];
        sb.p[i].y = y[i];
        sb.p[i].N = N[i];
        sb.p[i].K = K[i];
    }
    const int kind = g_decode_kernel.load();
    if (has_ws && M >= kSplitMinM && kind != BL_DECODE_LUT) {
        // every row quantised once (one launch), then the product on the codes
        int8_t* q[bl::kMaxGroup];
        float* s[bl::kMaxGroup];
        ws_layout(count, M, K, ws, q, s);
        bl::QuantBatch qb;
        std::memset(&qb, 0, sizeof(qb));
        qb.count = count;
        qb.rows = (int)(M * count);
        qb.eps = eps;
        for (int i = 0; i < count; ++i) {
            qb.p[i].x = x[i];
            qb.p[i].gain = gain ? gain[i] : nullptr;
            qb.p[i].q = q[i];
            qb.p[i].s = s[i];
            qb.p[i].K = K[i];
            qb.p[i].row_begin = (int)(M * i);
            qb.row_begin[i] = qb.p[i].row_begin;
            sb.p[i].x = nullptr;
            sb.p[i].gain = nullptr;
            sb.p[i].q = q[i];
            sb.p[i].s = s[i];
            b.p[i].x = nullptr;
            b.p[i].q = q[i];
            b.p[i].s = s[i];
        }
        if (bl::launch_quant_grouped(qb, xt, status, cs) != cudaSuccess) return BL_ERR_CUDA;
        const bl_status r = dispatch_decode(sb, false, BL_F32, yt, status, cs);
        if (r != kTryNext) return r;
        // the per-tile kernel's unfused form takes one problem per launch
        for (int i = 0; i < count; ++i) {
            bl::GemvBatch one;
            std::memset(&one, 0, sizeof(one));
            one.count = 1;
            one.M = M;
            one.p[0] = b.p[i];
            if (bl::launch_gemv(one, false, BL_F32, yt, status, cs) != cudaSuccess) return BL_ERR_CUDA;
        }
        return BL_OK;
    }
    const bl_status r = dispatch_decode(sb, true, xt, yt, status, cs);
    if (r != kTryNext) return r;
    // the per-tile kernel has no normalising prologue
    if (gain || !tile_fits) return BL_ERR_SHAPE;
    return bl::launch_gemv(b, true, xt, yt, status, cs) == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}

}  // namespace

namespace bl {
unsigned* status_word_ptr() { return status_word(); }
}  // namespace bl

extern "C" {

int64_t bitlinear_padded_k(int64_t K) { return K <= 0 ? 0 : bl::padded_k(K); }

int64_t bitlinear_packed_bytes(int64_t N, int64_t K)
{
    if (N <= 0 || K <= 0) return 0;
    return bl::padded_n(N) * bl::padded_k(K) / 4;
}

int64_t bitlinear_pack_workspace_bytes(int64_t N, int64_t K)
{
    if (N <= 0 || K <= 0) return 0;
    return (int64_t)bl::absmean_blocks(N * K) * 8 + 16;
}

bl_status bitlinear_pack_weights(const float* W, int64_t N, int64_t K, double eps, uint8_t* packed,
                                 double* gamma64, float* gamma32, void* workspace,
                                 size_t workspace_bytes, void* stream)
{
    if (!W || !packed || !gamma64 || !gamma32 || !workspace) return BL_ERR_NULL;
    if (N <= 0 || K <= 0 || N > (int64_t(1) << 40) / K) return BL_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(packed) || !aligned16(workspace) || !aligned_to(gamma64, 8) ||
        !aligned_to(gamma32, 4))
        return BL_ERR_ALIGN;
    if (!(eps >= 0.0) || !std::isfinite(eps)) return BL_ERR_ARG;
    if ((int64_t)workspace_bytes < bitlinear_pack_workspace_bytes(N, K)) return BL_ERR_WORKSPACE;
    unsigned* status = status_word();
    if (!status) return BL_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t count = N * K;
    const int blocks = bl::absmean_blocks(count);
    double* partial = static_cast<double*>(workspace);
    float* thr = reinterpret_cast<float*>(static_cast<char*>(workspace) + (size_t)blocks * 8);
    if (bl::launch_absmean_partial(W, count, partial, blocks, status, st) != cudaSuccess) return BL_ERR_CUDA;
    if (bl::launch_absmean_finalize(partial, blocks, count, eps, gamma64, gamma32, thr, st) != cudaSuccess)
        return BL_ERR_CUDA;
    if (bl::launch_pack(W, N, K, thr, packed, st) != cudaSuccess) return BL_ERR_CUDA;
    return BL_OK;
}

bl_status bitlinear_quant_act(const void* x, bl_dtype xt, int64_t M, int64_t K, int8_t* q, float* s,
                              void* stream)
{
    if (!x || !q || !s) return BL_ERR_NULL;
    if (check_dtype(xt) != BL_OK) return BL_ERR_DTYPE;
    if (M <= 0 || K <= 0 || M > (int64_t(1) << 31) - 1) return BL_ERR_SHAPE;
    if (K > kMaxK) return BL_ERR_OVERFLOW;
    if (!aligned16(x) || !aligned16(q) || !aligned16(s)) return BL_ERR_ALIGN;
    unsigned* status = status_word();
    if (!status) return BL_ERR_CUDA;
    return bl::launch_quant(x, xt, M, K, q, s, status, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? BL_OK
               : BL_ERR_CUDA;
}

bl_status bitlinear_rmsnorm_quant_act(const void* x, bl_dtype xt, const float* gain, double eps, int64_t M,
                                      int64_t K, int8_t* q, float* s, void* stream)
{
    if (!x || !gain || !q || !s) return BL_ERR_NULL;
    if (check_dtype(xt) != BL_OK) return BL_ERR_DTYPE;
    if (M <= 0 || K <= 0 || M > (int64_t(1) << 31) - 1) return BL_ERR_SHAPE;
    if (K > kMaxK) return BL_ERR_OVERFLOW;
    if (!aligned16(x) || !aligned16(q) || !aligned16(s) || !aligned16(gain)) return BL_ERR_ALIGN;
    if (!(eps >= 0.0) || !std::isfinite(eps)) return BL_ERR_ARG;
    unsigned* status = status_word();
    if (!status) return BL_ERR_CUDA;
    return bl::launch_rmsnorm_quant(x, xt, gain, eps, M, K, q, s, status, static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? BL_OK
               : BL_ERR_CUDA;
}

bl_status bitlinear_forward(const int8_t* q, const float* s, const uint8_t* packed,
                            const float* gamma32, int64_t M, int64_t N, int64_t K, void* y,
                            bl_dtype yt, int32_t* acc_debug, void* stream)
{
    if (!q || !s || !packed || !gamma32 || !y) return BL_ERR_NULL;
    if (check_dtype(yt) != BL_OK) return BL_ERR_DTYPE;
    bl_status st = check_forward_shape(M, N, K);
    if (st != BL_OK) return st;
    if (!aligned16(q) || !aligned16(s) || !aligned16(packed) || !aligned_to(gamma32, 4) || !aligned16(y) ||
        (acc_debug && !aligned16(acc_debug)))
        return BL_ERR_ALIGN;
    unsigned* status = status_word();
    if (!status) return BL_ERR_CUDA;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (M > bl::kFusedMaxM && bl::gemm_tc_supported(M, N, K))
        return bl::launch_gemm_tc(q, s, packed, gamma32, M, N, K, y, yt, acc_debug, status, cs) == cudaSuccess
                   ? BL_OK
                   : BL_ERR_CUDA;
    if (g_decode_kernel.load() == BL_DECODE_LUT) {
        if (!bl::lut_supported(M, K)) return BL_ERR_SHAPE;
        const cudaError_t e = bl::launch_lut(q, s, packed, gamma32, N, K, y, yt, acc_debug, cs);
        return e == cudaSuccess ? BL_OK : e == cudaErrorNotSupported ? BL_ERR_SHAPE : BL_ERR_CUDA;
    }
    if (M <= bl::kFusedMaxM) {
        bl::StreamBatch sb;
        std::memset(&sb, 0, sizeof(sb));
        sb.count = 1;
        sb.M = (int)M;
        sb.p[0].q = q;
        sb.p[0].s = s;
        sb.p[0].packed = packed;
        sb.p[0].gamma32 = gamma32;
        sb.p[0].y = y;
        sb.p[0].acc = acc_debug;
        sb.p[0].N = N;
        sb.p[0].K = K;
        const bl_status r = dispatch_decode(sb, false, BL_F32, yt, status, cs);
        if (r != kTryNext) return r;
    }
    bl::GemvBatch b;
    std::memset(&b, 0, sizeof(b));
    b.count = 1;
    b.M = M;
    b.p[0].q = q;
    b.p[0].s = s;
    b.p[0].packed = packed;
    b.p[0].gamma32 = gamma32;
    b.p[0].y = y;
    b.p[0].acc = acc_debug;
    b.p[0].N = N;
    b.p[0].K = K;
    return bl::launch_gemv(b, false, BL_F32, yt, status, cs) == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}

bl_status bitlinear_forward_x_grouped(int count, const void* const* x, bl_dtype xt,
                                      const uint8_t* const* packed, const float* const* gamma32,
                                      int64_t M, const int64_t* N, const int64_t* K, void* const* y,
                                      bl_dtype yt, void* stream)
{
    return grouped_decode(count, x, xt, nullptr, 0.0, packed, gamma32, M, N, K, y, yt, nullptr, 0, false, stream);
}

bl_status bitlinear_forward_x_grouped_ws(int count, const void* const* x, bl_dtype xt,
                                         const uint8_t* const* packed, const float* const* gamma32, int64_t M,
                                         const int64_t* N, const int64_t* K, void* const* y, bl_dtype yt,
                                         void* workspace, int64_t workspace_bytes, void* stream)
{
    return grouped_decode(count, x, xt, nullptr, 0.0, packed, gamma32, M, N, K, y, yt, workspace,
                          workspace_bytes, true, stream);
}

int64_t bitlinear_decode_workspace_bytes(int count, int64_t M, const int64_t* K)
{
    if (count < 1 || count > bl::kMaxGroup || !K || M <= 0 || M > bl::kFusedMaxM) return 0;
    for (int i = 0; i < count; ++i)
        if (K[i] <= 0 || K[i] > kMaxK) return 0;
    return ws_layout(count, M, K, nullptr, nullptr, nullptr);
}

int bitlinear_set_decode_kernel(int kind)
{
    if (kind < BL_DECODE_AUTO || kind > BL_DECODE_LUT) return BL_ERR_ARG;
    g_decode_kernel.store(kind);
    return BL_OK;
}

int bitlinear_get_decode_kernel(void) { return g_decode_kernel.load(); }

bl_status bitlinear_forward_x_rmsnorm_grouped(int count, const void* const* x, bl_dtype xt,
                                              const float* const* gain, double eps, const uint8_t* const* packed,
                                              const float* const* gamma32, int64_t M, const int64_t* N,
                                              const int64_t* K, void* const* y, bl_dtype yt, void* stream)
{
    if (!gain) return BL_ERR_NULL;
    return grouped_decode(count, x, xt, gain, eps, packed, gamma32, M, N, K, y, yt, nullptr, 0, false, stream);
}

bl_status bitlinear_forward_x_rmsnorm_grouped_ws(int count, const void* const* x, bl_dtype xt,
                                                 const float* const* gain, double eps,
                                                 const uint8_t* const* packed, const float* const* gamma32,
                                                 int64_t M, const int64_t* N, const int64_t* K, void* const* y,
                                                 bl_dtype yt, void* workspace, int64_t workspace_bytes,
                                                 void* stream)
{
    if (!gain) return BL_ERR_NULL;
    return grouped_decode(count, x, xt, gain, eps, packed, gamma32, M, N, K, y, yt, workspace, workspace_bytes,
                          true, stream);
}

bl_status bitlinear_forward_x(const void* x, bl_dtype xt, const uint8_t* packed, const float* gamma32,
                              int64_t M, int64_t N, int64_t K, void* y, bl_dtype yt, void* stream)
{
    return bitlinear_forward_x_grouped(1, &x, xt, &packed, &gamma32, M, &N, &K, &y, yt, stream);
}

int bitlinear_forward_x_supported(int64_t M, int64_t K)
{
    if (check_forward_shape(M, 1, K) != BL_OK || M > bl::kFusedMaxM) return 0;
    return ((size_t)pow2_tokens(M) * (size_t)bl::padded_k(K) <= kFusedSmemLimit || bl::dec_tc_fits(M, K)) ? 1 : 0;
}

bl_status bitlinear_get_status(void* stream)
{
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return BL_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_bl_status_word, sizeof(v)) != cudaSuccess) return BL_ERR_CUDA;
    if (v != 0) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(g_bl_status_word, &zero, sizeof(zero)) != cudaSuccess) return BL_ERR_CUDA;
        return (v & bl::kStatusTimeout) ? BL_ERR_TIMEOUT : BL_ERR_NONFINITE;
    }
    return BL_OK;
}

const char* bitlinear_status_string(bl_status status)
{
    switch (status) {
        case BL_OK: return "BL_OK";
        case BL_ERR_NULL: return "BL_ERR_NULL: a required pointer is NULL";
        case BL_ERR_SHAPE: return "BL_ERR_SHAPE: M, N or K out of range";
        case BL_ERR_ALIGN: return "BL_ERR_ALIGN: a device pointer is not 16-byte aligned";
        case BL_ERR_DTYPE: return "BL_ERR_DTYPE: unknown dtype";
        case BL_ERR_WORKSPACE: return "BL_ERR_WORKSPACE: workspace too small";
        case BL_ERR_OVERFLOW: return "BL_ERR_OVERFLOW: 127*K >= 2^31, int32 accumulator could overflow";
        case BL_ERR_NONFINITE: return "BL_ERR_NONFINITE: NaN or Inf met in W or x";
        case BL_ERR_CUDA: return "BL_ERR_CUDA: a CUDA call or kernel launch failed";
        case BL_ERR_ARG: return "BL_ERR_ARG: invalid argument";
        case BL_ERR_TIMEOUT: return "BL_ERR_TIMEOUT: a kernel abandoned a bounded wait; outputs are invalid";
    }
    return "unknown bl_status";
}

}  // extern "C"
