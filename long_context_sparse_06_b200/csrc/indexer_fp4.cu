// indexer_fp4.cu -- FP4 (E2M1 + E4M3 per-32 scale) lightning indexer.
#include <utility>

#include "lcs_common.cuh"
#include "lcs_internal.h"

namespace lcs {

int64_t index_fp4_scratch_bytes(int64_t B, int64_t Q, int d_I) { return B * Q * 64 * (d_I / 2 + d_I / 32); }

cudaError_t launch_index_fp4_tc(const void*, const float*, const void*, int64_t, int64_t, int64_t, int,
                                const int64_t*, int, uint16_t*, uint8_t*, int*, cudaStream_t, bool) {
    return cudaErrorNotSupported;
}

}  // namespace lcs
