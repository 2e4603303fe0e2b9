// noalloc.cu -- stem_score_noalloc: stem_score for callers that cannot allocate device
// memory.  The pooled block representations that stem_score keeps in a caller-provided
// workspace live here in a fixed, file-scope device array instead.
#include <cstdio>
#include <mutex>

#include "../../include/bsa.h"
#include "internal.h"

namespace bsa {
namespace {

// Fixed scratch for the pooled Q/K representations and value norms.  Every GPU that loads
// the library holds these bytes until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device.  In host code the array's name
// is only a host-side stand-in, so the address is looked up once per device, with that
// device current, and cached.
bsa_status_t scratch_address(void** out) {
    static std::mutex mu;
    static void* addr[64] = {};
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        char msg[160];
        snprintf(msg, sizeof msg, "stem_score_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
        set_last_error(msg);
        return BSA_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(mu);
    if (addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) {
            char msg[160];
            snprintf(msg, sizeof msg, "stem_score_noalloc: cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
            set_last_error(msg);
            return BSA_ERR_CUDA;
        }
        addr[dev] = p;
    }
    *out = addr[dev];
    return BSA_OK;
}

}  // namespace
}  // namespace bsa

extern "C" {

bsa_status_t stem_score_noalloc(bsa_tensor_t q, bsa_tensor_t k, bsa_tensor_t v, int32_t B, int32_t N, int32_t Hq,
                                int32_t Hkv, int32_t d, int32_t block, int32_t metric, float softmax_scale,
                                float* scores, int32_t nb_stride, cudaStream_t stream) {
    using namespace bsa;
    // Sizes stem_score refuses for another reason (non-positive sizes, a head_dim, block or head
    // ratio it does not take) go straight to it, so the caller gets the same error it gives.
    if (B <= 0 || N <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || (d != 64 && d != 128) ||
        (block != 64 && block != 128))
        return stem_score(q, k, v, B, N, Hq, Hkv, d, block, metric, softmax_scale, scores, nb_stride, nullptr, 0,
                          stream);
    const int nb = (N + block - 1) / block;
    const size_t need = bsa_score_workspace_bytes(B, Hq, Hkv, nb, d);
    if (need > kNoAllocScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "stem_score_noalloc: this problem needs %zu bytes of scratch but the fixed scratch holds %zu; "
                 "call stem_score with a workspace instead",
                 need, kNoAllocScratchBytes);
        set_last_error(msg);
        return BSA_ERR_UNSUPPORTED;
    }
    void* ws = nullptr;
    const bsa_status_t st = scratch_address(&ws);
    if (st != BSA_OK) return st;
    return stem_score(q, k, v, B, N, Hq, Hkv, d, block, metric, softmax_scale, scores, nb_stride, ws,
                      kNoAllocScratchBytes, stream);
}

}  // extern "C"
