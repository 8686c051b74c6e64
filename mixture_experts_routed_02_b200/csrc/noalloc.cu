// noalloc.cu -- moe_ffn_forward_static: the MoE layer for callers that cannot
// allocate device memory.
//
// Some callers have no way to obtain a workspace: code that runs while a CUDA
// stream is being captured into a graph (cudaMalloc is not allowed then), hosts
// whose device memory is owned by another allocator they cannot call into, and
// runtimes with a fixed, up-front memory budget.  For them this entry point
// uses a workspace that is part of the library itself: a file-scope device
// array of kStaticWorkspaceBytes.  The driver reserves it on a GPU when the
// library's device code is loaded there, and it stays reserved until the
// process exits.  Everything else is the ordinary layer call: this file only
// supplies the buffer to moe_ffn_forward.
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.cuh"

namespace moe {
namespace {

// 64 MiB: enough for decode-sized batches of Mixtral-8x7B experts (T = 16,
// d_model 4096, d_ff 14336, 8 experts, top-2 needs about 22 MB in FP8 and
// 43 MB in BF16).
constexpr size_t kStaticWorkspaceBytes = size_t(64) << 20;

static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

// Device address of the array in each CUDA context that has called this
// entry point.  In host code the array's name is only a stand-in, so the
// address is looked up (cudaGetSymbolAddress) with the context current.  It is
// keyed by the driver's context id, not by the device ordinal: a device reset
// or another context on the same device gets its own copy of the array at a
// different address, and a new context gets a new id.
constexpr int kMaxStaticContexts = 64;
struct StaticEntry {
    unsigned long long ctx_id;
    void* ptr;
};
StaticEntry g_static[kMaxStaticContexts];
int g_static_count = 0, g_static_next = 0;
std::mutex g_static_mutex;

int static_workspace(void** ptr) {
    std::lock_guard<std::mutex> lock(g_static_mutex);
    unsigned long long id = 0;
    if (context_key(&id)) {
        for (int i = 0; i < g_static_count; ++i)
            if (g_static[i].ctx_id == id) {
                *ptr = g_static[i].ptr;
                return MOE_OK;
            }
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    if (!context_key(&id)) return MOE_ERR_CUDA;  // the lookup above made a context current
    g_static[g_static_next] = {id, p};
    g_static_next = (g_static_next + 1) % kMaxStaticContexts;
    if (g_static_count < kMaxStaticContexts) ++g_static_count;
    *ptr = p;
    return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" size_t moe_static_workspace_bytes(void) { return moe::kStaticWorkspaceBytes; }

extern "C" int moe_ffn_forward_static(const void* x, const float* logits, const void* w13, const void* s13,
                                      const void* w2, const void* s2, int T, int H, int F, int E, int k, int dtype,
                                      void* out, void* stream) {
    // the checks of moe_ffn_forward first, in its order (the workspace pointer
    // is the built-in array, never null), then the size against the array
    alignas(16) static const unsigned char kNonNull[16] = {};
    const int rc_args = moe::check_forward_args(x, logits, w13, s13, w2, s2, T, H, F, E, k, dtype, out, kNonNull);
    if (rc_args != MOE_OK) return rc_args;
    const size_t need = moe_workspace_size(T, H, F, E, k, dtype);
    if (need == 0) return MOE_ERR_INVALID_ARG;
    if (need > moe::kStaticWorkspaceBytes) return MOE_ERR_WORKSPACE;
    void* ws = nullptr;
    const int rc = moe::static_workspace(&ws);
    if (rc != MOE_OK) return rc;
    return moe_ffn_forward(x, logits, w13, s13, w2, s2, T, H, F, E, k, dtype, out, ws, moe::kStaticWorkspaceBytes,
                           stream);
}
