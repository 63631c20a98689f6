// noalloc.cu -- the fixed device scratch behind csa_attend_noalloc.
//
// Some callers cannot give the library device memory: a serving engine that has
// reserved nearly all of HBM for its KV-cache pool, or a host program with no
// device allocator of its own.  For them one attention entry point runs on a
// file-scope device array instead of a caller workspace.  The array lives in this
// translation unit alone, so under lazy module loading only processes that use
// that entry point pay for it.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/lcs.h"
#include "lcs_internal.h"

static __device__ __align__(256) unsigned char g_noalloc_scratch[LCS_NOALLOC_SCRATCH_BYTES];

namespace lcs {

namespace {
constexpr int kMaxDevices = 64;
void* g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mutex;
}  // namespace

int noalloc_scratch(void** ptr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LCS_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        // The symbol's address differs per device; the lookup runs with `dev` current.
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();   // do not leave the lookup's error for the caller's next check
            return LCS_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
    return LCS_OK;
}

}  // namespace lcs
