// proj.cu -- the compressor and the lightning indexer with their input projections fused in.
//
// "DeepSeek V4 深度解析" §2, CSA steps 1-2: the KV rows and the index keys that the
// compressor pools, the per-token pooling logits, and the indexer's query heads and per-head
// weights are all linear in the token's hidden state h.  These kernels take h and the weights
// instead of the projected tensors, so the projected rows never leave the chip:
//  * lcs_compress_proj: x_t = h_t . Wx and z_t = h_t . wz for the tokens of a tile of
//    entries, then the pooling p = softmax(z + bias), e = sum p x and RoPE of csa_compress;
//  * csa_index_topk_proj: qI = h_t . W_qI and w = h_t . W_w for the query, then the fp32
//    index scores (fixed fma chains over dims and heads) and the top-k of csa_index_topk.
// Every projected value is the fp32 fma chain over the hidden dims in order, so the scores
// are bit-exact against a reference that defines the projection the same way.  CUDA cores,
// sized for small hidden states (the shared-memory tile holds the tile's hidden rows).
#include <utility>

#include "lcs_common.cuh"
#include "lcs_internal.h"

namespace lcs {

namespace {

constexpr int kPThreads = 256;

template <typename T>
__device__ __forceinline__ float ldf(const T* p, int64_t i) {
    if constexpr (sizeof(T) == 4) return p[i];
    else return __bfloat162float(p[i]);
}

// One CTA per (request, tile of E entries).  Rows r = 0 .. R-1 of the tile are tokens
// t0 - overlap + r (R = E*m + overlap); a token before the chunk comes from h_tail or, with
// none, is left out of the softmax.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kPThreads) compress_proj_kernel(
    const Tin* __restrict__ h, const Tin* __restrict__ h_tail, const Tin* __restrict__ Wx, const float* __restrict__ wz,
    const float* __restrict__ bias, int64_t T, int hidden, int d, int m, int overlap, int d_rope, float theta,
    int64_t pos0, int E, Tout* __restrict__ out) {
    extern __shared__ __align__(16) float psh[];
    const int R = E * m + overlap;
    float* hs = psh;                               // [R, hidden]
    float* xs = hs + (int64_t)R * hidden;          // [R, d]
    float* zs = xs + (int64_t)R * d;               // [R]
    float* es = zs + R;                            // [d]  pooled entry
    float* pw = es + d;                            // [m + overlap]
    __shared__ int present[1024];
    const int64_t n_ent = T / m;
    const int64_t tiles = (n_ent + E - 1) / E;
    const int64_t b = blockIdx.x / tiles, tile = blockIdx.x - b * tiles;
    const int64_t j0 = tile * E;
    const int e_here = (int)((n_ent - j0) < E ? (n_ent - j0) : E);
    const int rows = e_here * m + overlap;
    const int64_t t0 = j0 * m;
    const int tid = threadIdx.x;

    // ---- hidden rows of the tile
    for (int r = tid; r < rows; r += kPThreads) {
        const int64_t t = t0 - overlap + r;
        present[r] = (t >= 0) || (h_tail != nullptr);
    }
    for (int64_t i = tid; i < (int64_t)rows * hidden; i += kPThreads) {
        const int r = (int)(i / hidden), c = (int)(i - (int64_t)r * hidden);
        const int64_t t = t0 - overlap + r;
        float v = 0.f;
        if (t >= 0) v = ldf(h, (b * T + t) * hidden + c);
        else if (h_tail != nullptr) v = ldf(h_tail, (b * overlap + (overlap + t)) * hidden + c);
        hs[i] = v;
    }
    __syncthreads();
    // ---- projections: fp32 fma chains over the hidden dims, in order
    for (int64_t o = tid; o < (int64_t)rows * (d + 1); o += kPThreads) {
        const int r = (int)(o / (d + 1)), c = (int)(o - (int64_t)r * (d + 1));
        const float* hr = hs + (int64_t)r * hidden;
        float acc = 0.f;
        if (c < d) {
            for (int i = 0; i < hidden; ++i) acc = fmaf(hr[i], ldf(Wx, (int64_t)i * d + c), acc);
            xs[(int64_t)r * d + c] = acc;
        } else {
            for (int i = 0; i < hidden; ++i) acc = fmaf(hr[i], wz[i], acc);
            zs[r] = acc;
        }
    }
    __syncthreads();
    // ---- pooling, one entry at a time
    const int Wp = m + overlap;
    for (int j = 0; j < e_here; ++j) {
        if (tid == 0) {
            float mx = -INFINITY;
            for (int i = 0; i < Wp; ++i)
                if (present[j * m + i]) mx = fmaxf(mx, zs[j * m + i] + bias[i]);
            float sum = 0.f;
            for (int i = 0; i < Wp; ++i) {
                const float e = present[j * m + i] ? expf(zs[j * m + i] + bias[i] - mx) : 0.f;
                pw[i] = e;
                sum += e;
            }
            for (int i = 0; i < Wp; ++i) pw[i] /= sum;
        }
        __syncthreads();
        for (int c = tid; c < d; c += kPThreads) {
            float acc = 0.f;
            for (int i = 0; i < Wp; ++i)
                if (present[j * m + i]) acc = fmaf(pw[i], xs[(int64_t)(j * m + i) * d + c], acc);
            es[c] = acc;
        }
        __syncthreads();
        const int half = d_rope / 2, c0 = d - d_rope;
        const int64_t pos = pos0 + (j0 + j) * m + m - 1;
        for (int i = tid; i < half; i += kPThreads) {
            float o1, o2;
            rope_pair(es[c0 + i], es[c0 + i + half], pos, i, d_rope, theta, o1, o2);
            es[c0 + i] = o1;
            es[c0 + i + half] = o2;
        }
        __syncthreads();
        Tout* dst = out + (b * n_ent + j0 + j) * d;
        for (int c = tid; c < d; c += kPThreads) {
            if constexpr (sizeof(Tout) == 4) dst[c] = es[c];
            else dst[c] = __float2bfloat16_rn(es[c]);
        }
        __syncthreads();
    }
}

// One CTA per (query, slice of entries): the query's index heads and head weights from its
// hidden state, then the scores as in the fp32 indexer (fma chain over d per head, fma chain
// over heads of w_h * ReLU).
__global__ void __launch_bounds__(kPThreads) index_proj_f32_kernel(
    const float* __restrict__ h, int hidden, const float* __restrict__ WqI, const float* __restrict__ Ww,
    const float* __restrict__ kI, int64_t Q, int64_t N_c, int H, int dI, const int64_t* __restrict__ q_pos, int m,
    float* __restrict__ scores) {
    extern __shared__ __align__(16) float ish[];
    float* hsv = ish;                 // [hidden]
    float* qs = hsv + hidden;         // [H, dI]
    float* ws = qs + H * dI;          // [H]
    const int64_t g = blockIdx.x;     // (b, q)
    const int64_t b = g / Q;
    for (int i = threadIdx.x; i < hidden; i += blockDim.x) hsv[i] = h[g * hidden + i];
    __syncthreads();
    for (int o = threadIdx.x; o < H * dI + H; o += blockDim.x) {
        float acc = 0.f;
        if (o < H * dI) {
            for (int i = 0; i < hidden; ++i) acc = fmaf(hsv[i], WqI[(int64_t)i * H * dI + o], acc);
            qs[o] = acc;
        } else {
            const int hh = o - H * dI;
            for (int i = 0; i < hidden; ++i) acc = fmaf(hsv[i], Ww[(int64_t)i * H + hh], acc);
            ws[hh] = acc;
        }
    }
    __syncthreads();
    int64_t n = N_c;
    if (q_pos != nullptr) {
        const int64_t a = (q_pos[g] + 1) / m;
        n = a < 0 ? 0 : (a < N_c ? a : N_c);
    }
    const float* kb = kI + b * N_c * dI;
    for (int64_t s = (int64_t)blockIdx.y * blockDim.x + threadIdx.x; s < N_c; s += (int64_t)gridDim.y * blockDim.x) {
        float acc = -INFINITY;
        if (s < n) {
            acc = 0.f;
            const float* kr = kb + s * dI;
            for (int hh = 0; hh < H; ++hh) {
                float dot = 0.f;
                for (int c = 0; c < dI; ++c) dot = fmaf(qs[hh * dI + c], kr[c], dot);
                acc = fmaf(ws[hh], dot > 0.f ? dot : 0.f, acc);
            }
        }
        scores[g * N_c + s] = acc;
    }
}

}  // namespace

// Entries per CTA for the compressor with projections: as many as fit about 150 KB of hidden
// and projected rows (at least one); 0 when one entry's window does not fit.
int compress_proj_tile(int hidden, int d, int m, int overlap) {
    const int64_t per_row = (int64_t)(hidden + d + 1) * 4;
    const int64_t budget = 150 * 1024;
    if ((int64_t)(m + overlap) * per_row + (d + m + overlap) * 4 > budget || m + overlap > 1024) return 0;
    int64_t E = (budget / per_row - overlap) / m;
    if (E > 16) E = 16;
    if ((int64_t)E * m + overlap > 1024) E = (1024 - overlap) / m;
    return E < 1 ? 1 : (int)E;
}

cudaError_t launch_compress_proj(const void* h, int h_dtype, int64_t B, int64_t T, int hidden, const void* h_tail,
                                 const void* Wx, int d, const float* wz, const float* bias, int m, int overlap,
                                 int d_rope, float theta, int64_t pos0, void* out, int out_dtype, cudaStream_t s) {
    const int E = compress_proj_tile(hidden, d, m, overlap);
    const int64_t n_ent = T / m;
    if (B == 0 || n_ent == 0) return cudaSuccess;
    const int R = E * m + overlap;
    const size_t smem = sizeof(float) * ((size_t)R * hidden + (size_t)R * d + R + d + m + overlap);
    const int64_t grid = B * ((n_ent + E - 1) / E);
    auto go = [&](auto kern, auto in_t, auto out_t) -> cudaError_t {
        using Ti = decltype(in_t);
        using To = decltype(out_t);
        cudaError_t e = set_smem_once(reinterpret_cast<const void*>(kern), smem);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)grid, kPThreads, smem, s>>>(static_cast<const Ti*>(h), static_cast<const Ti*>(h_tail),
                                                     static_cast<const Ti*>(Wx), wz, bias, T, hidden, d, m, overlap,
                                                     d_rope, theta, pos0, E, static_cast<To*>(out));
        return cudaGetLastError();
    };
    if (h_dtype == LCS_F32) {
        if (out_dtype == LCS_F32) return go(compress_proj_kernel<float, float>, float(), float());
        return go(compress_proj_kernel<float, __nv_bfloat16>, float(), __nv_bfloat16());
    }
    if (out_dtype == LCS_F32) return go(compress_proj_kernel<__nv_bfloat16, float>, __nv_bfloat16(), float());
    return go(compress_proj_kernel<__nv_bfloat16, __nv_bfloat16>, __nv_bfloat16(), __nv_bfloat16());
}

cudaError_t launch_index_proj_f32(const float* h, int hidden, const float* WqI, const float* Ww, const float* kI,
                                  int64_t B, int64_t Q, int64_t N_c, int H_I, int d_I, const int64_t* q_pos, int m,
                                  float* scores, cudaStream_t s) {
    const int64_t groups = B * Q;
    if (groups == 0 || N_c == 0) return cudaSuccess;
    const size_t smem = sizeof(float) * (hidden + H_I * d_I + H_I);
    cudaError_t e = set_smem_once(reinterpret_cast<const void*>(index_proj_f32_kernel), smem);
    if (e != cudaSuccess) return e;
    const int64_t ychunks = (N_c + kPThreads - 1) / kPThreads;
    dim3 grid((unsigned)groups, (unsigned)(ychunks < 16 ? ychunks : 16));
    index_proj_f32_kernel<<<grid, kPThreads, smem, s>>>(h, hidden, WqI, Ww, kI, Q, N_c, H_I, d_I, q_pos, m, scores);
    return cudaGetLastError();
}

}  // namespace lcs
