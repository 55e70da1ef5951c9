// tidar_verify_noalloc: the verify with its scratch in a fixed device array
// instead of a caller-provided workspace.
//
// Some callers cannot hand the library a workspace: a plug-in running inside
// a host runtime that owns all device memory and forbids cudaMalloc on its
// decode path, or a latency-critical serving loop that must not allocate after
// start-up.  For them the verify's per-chunk statistics and residual sums live
// in `g_verify_scratch`, a file-scope device array that every GPU loading this
// library holds until the process exits.
//
// Host code cannot use the array's name as a device address (it is only a
// host-side stand-in), so the first call on each device, with that device
// current, resolves the real address with cudaGetSymbolAddress and caches it;
// that first call should therefore come before any stream capture.  Every
// call on a device shares the same array: calls whose kernels overlap on the
// GPU (other streams, or no ordering between them) race on it.  The one entry
// that must start at zero, the verify kernel's grid-barrier counter, is
// cleared in stream order at the start of every call (cudaMemsetAsync, which
// allocates nothing); every other entry is written before it is read.
#include <mutex>

#include "common.cuh"

namespace tidar {
size_t verify_workspace_bytes(int B, int k, int V);
cudaError_t verify_launch(const void *, const void *, int, const int32_t *, const uint8_t *, const float *,
                          const float *, int, int, int, float, int32_t *, int32_t *, int32_t *, int32_t *, float *,
                          float *, void *, int32_t *, cudaStream_t);
}  // namespace tidar

namespace {

constexpr size_t kScratchBytes = size_t(2) << 20;  // 2 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_verify_scratch[kScratchBytes];

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_verify_scratch on the current device (resolved once per device).
cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_verify_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

tidar_status tidar_verify_noalloc(const void *p_logits, const void *q_logits, int logits_dtype,
                                  const int32_t *drafts, const uint8_t *preaccepted, const float *u_acc,
                                  const float *u_res, int B, int k, int V, int32_t *accept_len, int32_t *resampled,
                                  int32_t *tokens, int32_t *n_emitted, float *logp_d, float *logq_d,
                                  int32_t *dev_status, void *stream) {
    if (B < 1 || k < 1 || V < 1) return TIDAR_ERR_INVALID_ARG;
    if (k > tidar::kMaxDraft || V > tidar::kMaxVocab) return TIDAR_ERR_UNSUPPORTED;
    if (logits_dtype != TIDAR_DT_BF16 && logits_dtype != TIDAR_DT_F32) return TIDAR_ERR_INVALID_ARG;
    if (!p_logits || !q_logits || !drafts || !preaccepted || !u_acc || !u_res || !accept_len || !resampled ||
        !tokens || !n_emitted || !dev_status)
        return TIDAR_ERR_INVALID_ARG;
    // sizes whose scratch would not fit the fixed array are refused, never truncated
    if (tidar::verify_workspace_bytes(B, k, V) > kScratchBytes) return TIDAR_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return TIDAR_ERR_CUDA;
    const cudaError_t e = tidar::verify_launch(p_logits, q_logits, logits_dtype, drafts, preaccepted, u_acc, u_res, B,
                                               k, V, 1.f, accept_len, resampled, tokens, n_emitted, logp_d, logq_d,
                                               scratch, dev_status, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TIDAR_OK : TIDAR_ERR_CUDA;
}

}  // extern "C"
