// cp.cu -- context parallelism for one long request: the compressed entries of a request
// are split over G ranks (rank r holds entries [r*S, (r+1)*S)).
//
// "DeepSeek V4 深度解析" §2, CSA steps 2-3: the lightning indexer keeps the top-k of all
// compressed entries, and one softmax runs over the selection and the window.  Both split
// exactly over shards of the entries:
//  * every global top-k entry is in the top-k of its own shard, so the top-k of the
//    ranks' local top-k candidates, gathered in rank order (which is global-index order),
//    is the global top-k with the same tie rule (lower index first);
//  * attention over a union of disjoint row sets is the log-sum-exp merge of the parts:
//    o = sum_r exp(lse_r - L) o_r with L = log sum_r exp(lse_r).
// These kernels are the device side of that exchange; the collectives themselves (one
// all-gather of candidates, one of attention partials) are the caller's.
#include <utility>

#include "lcs_common.cuh"
#include "lcs_internal.h"

namespace lcs {

namespace {

// One block per request: (score, global index) of the rank's local selection; -1 entries
// become (-inf, -1).
__global__ void cp_candidates_kernel(const void* __restrict__ scores, int score_dtype, int64_t S,
                                     const int32_t* __restrict__ idx_local, int k, int64_t offset,
                                     float* __restrict__ cand_score, int32_t* __restrict__ cand_idx) {
    const int64_t b = blockIdx.x;
    for (int i = threadIdx.x; i < k; i += blockDim.x) {
        const int32_t li = idx_local[b * k + i];
        float sc = -INFINITY;
        int32_t gi = -1;
        if (li >= 0 && li < S) {
            sc = score_dtype == LCS_BF16 ? bf16_bits_to_f32(static_cast<const uint16_t*>(scores)[b * S + li])
                                         : static_cast<const float*>(scores)[b * S + li];
            gi = (int32_t)(offset + li);
        }
        cand_score[b * k + i] = sc;
        cand_idx[b * k + i] = gi;
    }
}

// Gathered candidates [G, B, k] -> score rows [B, G*k] in rank order.
__global__ void cp_rows_kernel(const float* __restrict__ cand_score, int G, int64_t B, int k,
                               float* __restrict__ rows) {
    const int64_t b = blockIdx.x;
    for (int i = threadIdx.x; i < G * k; i += blockDim.x) {
        const int r = i / k, j = i - r * k;
        rows[b * (int64_t)G * k + i] = cand_score[((int64_t)r * B + b) * k + j];
    }
}

// Selected positions (ascending) -> global indices, valid ones first in ascending order then
// -1; and this rank's share as local indices (ascending, -1 padded).  One block per request.
constexpr int kMapThreads = 256;
__global__ void __launch_bounds__(kMapThreads) cp_map_kernel(const int32_t* __restrict__ pos,
                                                             const int32_t* __restrict__ cand_idx, int G,
                                                             int64_t B, int k, int64_t offset, int64_t S,
                                                             int32_t* __restrict__ idx_global,
                                                             int32_t* __restrict__ idx_local) {
    __shared__ uint32_t wsum[2][kMapThreads / 32];
    __shared__ uint32_t tot[2];
    const int64_t b = blockIdx.x;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    uint32_t base_g = 0, base_l = 0;
    for (int c0 = 0; c0 < k; c0 += kMapThreads) {
        const int i = c0 + t;
        int32_t g = -1;
        if (i < k) {
            const int32_t p = pos[b * k + i];
            if (p >= 0) {
                const int r = p / k, j = p - r * k;
                g = cand_idx[((int64_t)r * B + b) * k + j];
            }
        }
        const bool vg = g >= 0, vl = vg && g >= offset && g < offset + S;
        const uint32_t mg = __ballot_sync(0xffffffffu, vg), ml = __ballot_sync(0xffffffffu, vl);
        if (lane == 0) {
            wsum[0][warp] = __popc(mg);
            wsum[1][warp] = __popc(ml);
        }
        __syncthreads();
        uint32_t bg = base_g, bl = base_l;
        for (int w = 0; w < warp; ++w) {
            bg += wsum[0][w];
            bl += wsum[1][w];
        }
        const uint32_t lt = (1u << lane) - 1u;
        if (vg) idx_global[b * k + bg + __popc(mg & lt)] = g;
        if (vl) idx_local[b * k + bl + __popc(ml & lt)] = (int32_t)(g - offset);
        if (t == 0) {
            uint32_t sg = 0, sl = 0;
            for (int w = 0; w < kMapThreads / 32; ++w) {
                sg += wsum[0][w];
                sl += wsum[1][w];
            }
            tot[0] = sg;
            tot[1] = sl;
        }
        __syncthreads();
        base_g += tot[0];
        base_l += tot[1];
        __syncthreads();
    }
    for (int i = (int)base_g + t; i < k; i += kMapThreads) idx_global[b * k + i] = -1;
    for (int i = (int)base_l + t; i < k; i += kMapThreads) idx_local[b * k + i] = -1;
}

// One block per (request, head) row: o = sum_r exp(lse_r - L) o_r, L = log sum_r exp(lse_r),
// summed in rank order; all lse_r = -inf (an empty row set) gives o = 0, lse = -inf.
__global__ void attn_merge_kernel(const float* __restrict__ o, const float* __restrict__ lse, int G, int64_t rows,
                                  int d_v, void* __restrict__ out, int out_dtype, float* __restrict__ lse_out) {
    const int64_t row = blockIdx.x;
    float M = -INFINITY;
    for (int r = 0; r < G; ++r) M = fmaxf(M, lse[(int64_t)r * rows + row]);
    float L = 0.f;
    for (int r = 0; r < G; ++r) {
        const float l = lse[(int64_t)r * rows + row];
        L += l == -INFINITY ? 0.f : expf(l - M);
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    for (int d = threadIdx.x; d < d_v; d += blockDim.x) {
        float acc = 0.f;
        for (int r = 0; r < G; ++r) {
            const float l = lse[(int64_t)r * rows + row];
            if (l != -INFINITY) acc = fmaf(expf(l - M) * inv, o[((int64_t)r * rows + row) * d_v + d], acc);
        }
        if (out_dtype == LCS_F32) static_cast<float*>(out)[row * d_v + d] = acc;
        else static_cast<uint16_t*>(out)[row * d_v + d] = f32_to_bf16_bits(acc);
    }
    if (threadIdx.x == 0 && lse_out != nullptr) lse_out[row] = L > 0.f ? M + logf(L) : -INFINITY;
}

}  // namespace

cudaError_t launch_cp_candidates(const void* scores, int score_dtype, int64_t B, int64_t S, const int32_t* idx_local,
                                 int k, int64_t offset, float* cand_score, int32_t* cand_idx, cudaStream_t s) {
    if (B == 0 || k == 0) return cudaSuccess;
    cp_candidates_kernel<<<(unsigned)B, 256, 0, s>>>(scores, score_dtype, S, idx_local, k, offset, cand_score,
                                                     cand_idx);
    return cudaGetLastError();
}

int64_t cp_select_scratch_bytes(int G, int64_t B, int k) {
    return align256(B * (int64_t)G * k * 4) + align256(B * (int64_t)k * 4);
}

cudaError_t launch_cp_select(const float* cand_score, const int32_t* cand_idx, int G, int64_t B, int k, int64_t offset,
                             int64_t S, int32_t* idx_global, int32_t* idx_local, void* scratch, int* status,
                             cudaStream_t s) {
    if (B == 0 || k == 0) return cudaSuccess;
    float* rows = static_cast<float*>(scratch);
    int32_t* pos = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(scratch) + align256(B * (int64_t)G * k * 4));
    cp_rows_kernel<<<(unsigned)B, 256, 0, s>>>(cand_score, G, B, k, rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = launch_topk(rows, LCS_F32, B, 1, (int64_t)G * k, nullptr, 1, k, pos, nullptr, status, s, false);
    if (e != cudaSuccess) return e;
    cp_map_kernel<<<(unsigned)B, kMapThreads, 0, s>>>(pos, cand_idx, G, B, k, offset, S, idx_global, idx_local);
    return cudaGetLastError();
}

cudaError_t launch_attn_merge(const float* o, const float* lse, int G, int64_t rows, int d_v, void* out, int out_dtype,
                              float* lse_out, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    attn_merge_kernel<<<(unsigned)rows, 128, 0, s>>>(o, lse, G, rows, d_v, out, out_dtype, lse_out);
    return cudaGetLastError();
}

}  // namespace lcs
