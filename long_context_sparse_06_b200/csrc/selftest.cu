// selftest.cu -- exercises the bounded-wait path every pipelined kernel relies on.
//
// Not part of the method: the pages describe no such call.  A kernel that waits on an
// mbarrier nothing will ever complete must give up after its budget, record
// LCS_ERR_TIMEOUT (with where it waited) in the status word and return, leaving the
// CUDA context usable; a later wait in the same grid must give up at once because the
// status word is already set.  lcs_selftest_wait runs exactly that, with the waiting
// code the kernels use and a caller-chosen budget.
#include "lcs_common.cuh"
#include "lcs_internal.h"

namespace lcs {
namespace {

__global__ void selftest_wait_kernel(uint64_t budget_ns, int* status, long long* out) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);   // never arrived on: phase 0 never completes
        fence_barrier_init();
    }
    __syncthreads();
    const uint64_t t0 = globaltimer();
    const bool ok1 = mbar_wait(&bar, 0, status, 901, budget_ns);
    const uint64_t t1 = globaltimer();
    // the grid's status is set now: this wait gives up within two checks
    const bool ok2 = mbar_wait(&bar, 0, status, 902, 1000 * budget_ns);
    const uint64_t t2 = globaltimer();
    __syncthreads();
    if (threadIdx.x == 0) {
        out[0] = ok1;
        out[1] = (long long)(t1 - t0);
        out[2] = ok2;
        out[3] = (long long)(t2 - t1);
    }
}

}  // namespace

cudaError_t launch_selftest_wait(uint64_t budget_ns, int* status, long long* out, cudaStream_t stream) {
    selftest_wait_kernel<<<1, 64, 0, stream>>>(budget_ns, status, out);
    return cudaGetLastError();
}

}  // namespace lcs
