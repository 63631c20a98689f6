// noalloc.cu -- the fixed device scratch behind csa_attend_noalloc.
//
// Some callers cannot give the library device memory: a serving engine that has
// reserved nearly all of HBM for its KV-cache pool, or a host program with no
// device allocator of its own.  For them one attention entry point runs on a
// file-scope device array instead of a caller workspace.  The array lives in this
// translation unit alone, so under lazy module loading only processes that use
// that entry point pay for it.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/lcs.h"
#include "lcs_internal.h"

static __device__ __align__(256) unsigned char g_noalloc_scratch[LCS_NOALLOC_SCRATCH_BYTES];

namespace lcs {

namespace {
constexpr int kMaxDevices = 64;
// The array's device address per device, and the id of the context it was looked up in:
// a new context on the device (after cudaDeviceReset, say) reloads the module, so the
// address is looked up again.
struct Slot {
    void* ptr;
    unsigned long long ctx_id;
    bool valid;
};
Slot g_noalloc[kMaxDevices];
std::mutex g_noalloc_mutex;

typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

CtxGetIdFn ctx_get_id() {
    static CtxGetIdFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetIdFn>(p);
    });
    return fn;
}

// Unique id of the calling thread's current context, if there is one.
bool current_ctx_id(unsigned long long* id) {
    CtxGetIdFn fn = ctx_get_id();
    return fn != nullptr && fn(nullptr, id) == CUDA_SUCCESS;
}
}  // namespace

int noalloc_scratch(void** ptr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LCS_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    unsigned long long id = 0;
    bool have_id = current_ctx_id(&id);
    Slot& s = g_noalloc[dev];
    if (!(have_id && s.valid && s.ctx_id == id)) {
        // The symbol's address differs per device (and per context); the lookup runs with
        // `dev` current.
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();   // do not leave the lookup's error for the caller's next check
            return LCS_ERR_CUDA;
        }
        if (!have_id) have_id = current_ctx_id(&id);   // the lookup made a context current
        s.ptr = p;
        s.ctx_id = id;
        s.valid = have_id;   // without a context id the address is looked up on every call
    }
    *ptr = s.ptr;
    return LCS_OK;
}

}  // namespace lcs
