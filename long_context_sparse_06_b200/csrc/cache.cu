// cache.cu -- decode-time cache update: one new token per request.
//
// "DeepSeek V4 深度解析" §4 (KV-cache management for the mixed attention): a state cache
// holds the sliding window and the raw tokens not yet enough to compress, and a
// compressed cache holds the CSA and HCA entries.  For the new token t of request b:
//   * its raw (un-rotated) KV row and index-key row go into a ring of the last 128 raw
//     tokens, its three pooling logits into a ring beside it;
//   * its KV row, rotated at position t, goes into the 128-row window ring (slot t % 128);
//   * when t + 1 is a multiple of 4, CSA entry j = t / 4 is pooled from tokens
//     4j-2 .. 4j+3 (those >= 0) with p = softmax(z + bias[0..5]) and rotated at
//     position t; the index key j is pooled the same way with its own logits and bias;
//   * when t + 1 is a multiple of 128, HCA entry h = t / 128 is pooled from tokens
//     128h .. 128h+127 with p = softmax(z_h + bias_h[0..127]) and rotated at position t.
// Entries are written in the caches' storage format: fp32, bf16, the FP8 KV row (E4M3
// content with a power-of-two scale per 128 dims, bf16 RoPE dims) or FP4 index keys (E2M1
// with an E4M3 scale per 32); the quantised writes are those of lcs_quant_kv_fp8 and
// lcs_quant_fp4 applied to the fp32 entry.  One CTA per request.
#include <utility>

#include "lcs_common.cuh"
#include "lcs_internal.h"

namespace lcs {

namespace {

constexpr int kRing = 128;            // raw tokens kept (one HCA block), also the window length
constexpr int kM = 4, kOv = 2, kMh = 128;
constexpr int kThreads = 256;

template <typename Tx>
__device__ __forceinline__ float ld(const Tx* p, int64_t i) {
    if constexpr (sizeof(Tx) == 4) return p[i];
    else return __bfloat162float(p[i]);
}
template <typename Tx>
__device__ __forceinline__ void st(Tx* p, int64_t i, float v) {
    if constexpr (sizeof(Tx) == 4) p[i] = v;
    else p[i] = __float2bfloat16_rn(v);
}

// Block-wide softmax of the logits l[0..n) (n <= kThreads; invalid positions carry -inf) into
// p[0..n), fp32.  red: 2 * (kThreads / 32) floats of scratch.
__device__ void block_softmax(const float* l, int n, float* p, float* red) {
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const float v = t < n ? l[t] : -INFINITY;
    float mx = warp_max(v);
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    mx = red[0];
    for (int w = 1; w < kThreads / 32; ++w) mx = fmaxf(mx, red[w]);
    const float e = (t < n && v != -INFINITY) ? expf(v - mx) : 0.f;
    float sm = warp_sum(e);
    if (lane == 0) red[kThreads / 32 + warp] = sm;
    __syncthreads();
    sm = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) sm += red[kThreads / 32 + w];
    if (t < n) p[t] = e / sm;
    __syncthreads();
}

// Stores the fp32 vector v[0..d) (shared memory) as one row of `dtype` at dst:
// LCS_F32 / LCS_BF16 rows of d, LCS_KV_FP8 rows (content d - d_rope, RoPE d_rope).
__device__ void store_row(const float* v, int d, int d_rope, int dtype, void* dst) {
    if (dtype == LCS_F32) {
        for (int i = threadIdx.x; i < d; i += kThreads) static_cast<float*>(dst)[i] = v[i];
    } else if (dtype == LCS_BF16) {
        for (int i = threadIdx.x; i < d; i += kThreads)
            static_cast<__nv_bfloat16*>(dst)[i] = __float2bfloat16_rn(v[i]);
    } else if (threadIdx.x < 32) {
        quant_kv_fp8_row_warp(v, d - d_rope, d_rope, static_cast<uint8_t*>(dst));
    }
}

// In-place rotate-half RoPE of the last d_rope dims of v[0..d) at position pos.
__device__ void rope_row(float* v, int d, int d_rope, float theta, int64_t pos) {
    const int half = d_rope / 2, c0 = d - d_rope;
    for (int i = threadIdx.x; i < half; i += kThreads) {
        float o1, o2;
        rope_pair(v[c0 + i], v[c0 + i + half], pos, i, d_rope, theta, o1, o2);
        v[c0 + i] = o1;
        v[c0 + i + half] = o2;
    }
    __syncthreads();
}

struct AppendArgs {
    const int64_t* pos;
    const void* x;
    const void* kx;
    const float *z, *zI, *zh, *bias, *biasI, *biash;
    int D, d_rope, dI;
    float theta;
    void* raw;       // [B, 128, D + dI] x dtype
    float* logits;   // [B, 3, 128]
    void* win;       // [B, 128, row]
    int win_dtype;
    void* comp;      // [B, N_c, row]
    void* kI;        // [B, N_c, dI] or FP4 planes
    void* hca;       // [B, N_h, row]
    int64_t B, N_c, N_h;
    int kv_dtype, kI_dtype;
};

__host__ __device__ inline int64_t row_bytes(int dtype, int d, int d_rope) {
    return dtype == LCS_F32 ? 4 * d : dtype == LCS_BF16 ? 2 * d : (d - d_rope) + 2 * d_rope + 4 * ((d - d_rope) / 128);
}

template <typename Tx>
__global__ void __launch_bounds__(kThreads) cache_append_kernel(const AppendArgs a, int* status) {
    extern __shared__ __align__(16) float sh[];
    const int D = a.D, dI = a.dI, DR = D + dI;
    float* cur = sh;                   // [DR] the new token's raw rows, fp32
    float* ent = cur + DR;             // [D]  pooled entry / rotated window row
    float* lg = ent + D;               // [kThreads] logits
    float* pw = lg + kThreads;         // [kThreads] pooling weights
    float* red = pw + kThreads;        // [16]
    const int64_t b = blockIdx.x;
    const int64_t t = a.pos[b];
    if (t < 0) return;                 // no token for this request in this call
    const int slot = (int)(t % kRing);
    const int tid = threadIdx.x;

    // ---- state cache: raw rows and logits into the rings, the rotated row into the window
    const Tx* xb = static_cast<const Tx*>(a.x) + b * D;
    const Tx* kb = static_cast<const Tx*>(a.kx) + b * dI;
    Tx* ring = static_cast<Tx*>(a.raw) + b * kRing * DR;
    for (int i = tid; i < DR; i += kThreads) {
        const float v = i < D ? ld(xb, i) : ld(kb, i - D);
        cur[i] = v;
        st(ring, (int64_t)slot * DR + i, v);
        if (i < D) ent[i] = v;
    }
    float* lring = a.logits + b * 3 * kRing;
    if (tid == 0) {
        lring[slot] = a.z[b];
        lring[kRing + slot] = a.zI[b];
        lring[2 * kRing + slot] = a.zh[b];
    }
    __syncthreads();
    rope_row(ent, D, a.d_rope, a.theta, t);
    const int64_t wrb = row_bytes(a.win_dtype, D, a.d_rope);
    store_row(ent, D, a.d_rope, a.win_dtype, static_cast<uint8_t*>(a.win) + (b * kRing + slot) * wrb);
    __syncthreads();   // ring writes visible to the block; ent free again

    const int64_t crb = row_bytes(a.kv_dtype, D, a.d_rope);
    // ---- CSA entry j = t / 4: tokens 4j-2 .. 4j+3, i.e. t-5 .. t
    if ((t + 1) % kM == 0) {
        const int64_t j = t / kM;
        if (j >= a.N_c) {
            if (tid == 0) set_status(status, LCS_ERR_DEVICE, 401);
        } else {
            constexpr int W = kM + kOv;
            for (int which = 0; which < 2; ++which) {   // 0: KV rows, 1: index-key rows
                const float* bias = which ? a.biasI : a.bias;
                if (tid < W) {
                    const int64_t tok = t - (W - 1) + tid;
                    lg[tid] = tok >= 0 ? lring[which * kRing + (int)(tok % kRing)] + bias[tid] : -INFINITY;
                }
                __syncthreads();
                block_softmax(lg, W, pw, red);
                const int c0 = which ? D : 0, d = which ? dI : D;
                for (int i = tid; i < d; i += kThreads) {
                    float acc = 0.f;
                    for (int w = 0; w < W; ++w) {
                        const int64_t tok = t - (W - 1) + w;
                        if (tok < 0) continue;
                        const float v = tok == t ? cur[c0 + i] : ld(ring, (tok % kRing) * DR + c0 + i);
                        acc = fmaf(pw[w], v, acc);
                    }
                    ent[i] = acc;
                }
                __syncthreads();
                if (which == 0) {
                    rope_row(ent, D, a.d_rope, a.theta, t);
                    store_row(ent, D, a.d_rope, a.kv_dtype, static_cast<uint8_t*>(a.comp) + (b * a.N_c + j) * crb);
                } else if (a.kI_dtype == LCS_FP4) {
                    uint8_t* packed = static_cast<uint8_t*>(a.kI);
                    uint8_t* scales = packed + a.B * a.N_c * (dI / 2);
                    const int64_t r = b * a.N_c + j;
                    const int warp = tid >> 5, lane = tid & 31;
                    for (int blk = warp; blk < dI / 32; blk += kThreads / 32)
                        quant_fp4_block_warp(ent[blk * 32 + lane], packed + r * (dI / 2) + blk * 16,
                                             scales + r * (dI / 32) + blk);
                } else {
                    store_row(ent, dI, 0, a.kI_dtype,
                              static_cast<uint8_t*>(a.kI) + (b * a.N_c + j) * row_bytes(a.kI_dtype, dI, 0));
                }
                __syncthreads();
            }
        }
    }
    // ---- HCA entry h = t / 128: tokens 128h .. t
    if ((t + 1) % kMh == 0) {
        const int64_t h = t / kMh;
        if (h >= a.N_h) {
            if (tid == 0) set_status(status, LCS_ERR_DEVICE, 402);
        } else {
            if (tid < kMh) lg[tid] = lring[2 * kRing + (int)((t - (kMh - 1) + tid) % kRing)] + a.biash[tid];
            __syncthreads();
            block_softmax(lg, kMh, pw, red);
            for (int i = tid; i < D; i += kThreads) {
                float acc = 0.f;
                for (int w = 0; w < kMh; ++w) {
                    const int64_t tok = t - (kMh - 1) + w;
                    const float v = tok == t ? cur[i] : ld(ring, (tok % kRing) * DR + i);
                    acc = fmaf(pw[w], v, acc);
                }
                ent[i] = acc;
            }
            __syncthreads();
            rope_row(ent, D, a.d_rope, a.theta, t);
            store_row(ent, D, a.d_rope, a.kv_dtype, static_cast<uint8_t*>(a.hca) + (b * a.N_h + h) * crb);
        }
    }
}

}  // namespace

cudaError_t launch_cache_append(const int64_t* pos, const void* x, const void* kx, int x_dtype, const float* z,
                                const float* zI, const float* zh, const float* bias, const float* biasI,
                                const float* biash, int D, int d_rope, int d_I, float theta, void* raw,
                                float* logits, void* win, int win_dtype, void* comp, void* kI, void* hca, int64_t B,
                                int64_t N_c, int64_t N_h, int kv_dtype, int kI_dtype, int* status, cudaStream_t s) {
    if (B == 0) return cudaSuccess;
    AppendArgs a{pos, x, kx, z, zI, zh, bias, biasI, biash, D, d_rope, d_I, theta, raw, logits, win, win_dtype,
                 comp, kI, hca, B, N_c, N_h, kv_dtype, kI_dtype};
    const size_t smem = sizeof(float) * ((D + d_I) + D + 2 * kThreads + 16);
    if (x_dtype == LCS_F32) {
        cudaError_t e = set_smem_once(reinterpret_cast<const void*>(cache_append_kernel<float>), smem);
        if (e != cudaSuccess) return e;
        cache_append_kernel<float><<<(unsigned)B, kThreads, smem, s>>>(a, status);
    } else {
        cudaError_t e = set_smem_once(reinterpret_cast<const void*>(cache_append_kernel<__nv_bfloat16>), smem);
        if (e != cudaSuccess) return e;
        cache_append_kernel<__nv_bfloat16><<<(unsigned)B, kThreads, smem, s>>>(a, status);
    }
    return cudaGetLastError();
}

}  // namespace lcs
