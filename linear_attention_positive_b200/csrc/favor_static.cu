// favor_fwd_static_scratch: the bidirectional bf16 forward for callers that cannot allocate.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: code that runs inside
// another allocator's callback (where a nested allocation would recurse), or in a process whose
// device memory is entirely reserved by a framework's caching allocator. For them this entry
// point takes its scratch from a fixed array that lives in the library's own device memory.
// It launches exactly the kernels favor_fwd launches for the bidirectional bf16 case, with the
// scratch pointer taken from that array instead of the caller.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds it until
// the process exits. In host code its name is only a host-side stand-in, so the device address
// is obtained once per device (with that device current) through cudaGetSymbolAddress.

#include <mutex>

namespace favor {

constexpr size_t kStaticScratchBytes = (size_t)FAVOR_STATIC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_static_mutex;
void *g_static_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device; fetched on the first call per device.
favor_status static_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FAVOR_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_static_mutex);
    if (g_static_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return FAVOR_ERR_CUDA;
        g_static_ptr[dev] = p;
    }
    *out = g_static_ptr[dev];
    return FAVOR_OK;
}

}  // namespace
}  // namespace favor

extern "C" favor_status favor_fwd_static_scratch(const favor_shape *s, const void *Q, const void *K, const void *V,
                                                 const void *W, float *out, void *stream) {
    using namespace favor;
    if (!shape_ok(s) || Q == nullptr || K == nullptr || V == nullptr || W == nullptr || out == nullptr)
        return FAVOR_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(W) || !aligned16(out))
        return FAVOR_ERR_INVALID_ARG;
    if (s->dtype != FAVOR_BF16) return FAVOR_ERR_UNSUPPORTED;
    const favor_status sup = shape_supported(s, 0, 0);
    if (sup != FAVOR_OK) return sup;
    const size_t need = favor_workspace_size(s, 0, 0, nullptr);
    if (need == 0) return FAVOR_ERR_UNSUPPORTED;
    if (need > kStaticScratchBytes) return FAVOR_ERR_WORKSPACE;
    void *ws = nullptr;
    const favor_status st = static_scratch(&ws);
    if (st != FAVOR_OK) return st;
    return fwd_bf16(s, Q, K, V, W, out, nullptr, (uint8_t *)ws, kStaticScratchBytes, nullptr, (cudaStream_t)stream, 0);
}
