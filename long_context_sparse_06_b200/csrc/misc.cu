// misc.cu -- RoPE, the two quantising cache writers and the grouped output
// projection.
//
//  * RoPE: rotate-half pairs on the last d_rope dims (the RoPE dims that
//    "DeepSeek V4 深度解析" §2 keeps in BF16).
//  * lcs_quant_kv_fp8: the mixed-precision KV row of the same paragraph (RoPE
//    dims BF16, the rest FP8 E4M3 with one power-of-two fp32 scale per 128
//    dims, so that code * scale is exact in bf16).
//  * lcs_quant_fp4: FP4 E2M1 with one E4M3 scale per 32 elements, the format of
//    the indexer's QK path ("DeepSeek V4 深度解析" §4, FP4量化感知訓練).
//  * group_oproj: the grouped output projection (§2, HCA paragraph).
#include <utility>

#include "lcs_common.cuh"
#include "lcs_internal.h"

namespace lcs {

namespace {

// One thread per (row, pair).
template <typename T>
__global__ void rope_kernel(T* rows, int64_t n, int d, int d_rope, float theta, const int64_t* __restrict__ pos) {
    const int half = d_rope / 2;
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= n * half) return;
    const int64_t r = g / half;
    const int i = (int)(g - r * half);
    const int c0 = d - d_rope;
    T* x = rows + r * d;
    float o1, o2;
    if constexpr (sizeof(T) == 4) {
        rope_pair(x[c0 + i], x[c0 + i + half], pos[r], i, d_rope, theta, o1, o2);
        x[c0 + i] = o1;
        x[c0 + i + half] = o2;
    } else {
        rope_pair(__bfloat162float(x[c0 + i]), __bfloat162float(x[c0 + i + half]), pos[r], i, d_rope, theta, o1, o2);
        x[c0 + i] = __float2bfloat16_rn(o1);
        x[c0 + i + half] = __float2bfloat16_rn(o2);
    }
}

// One warp per row.  Each 128-dim block: lane l owns elements 4l..4l+3.
__global__ void quant_kv_fp8_kernel(const float* __restrict__ x, int64_t n, int d_c, int d_r,
                                    uint8_t* __restrict__ out) {
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= n) return;
    const int64_t rb = d_c + 2 * d_r + 4 * (d_c / 128);
    quant_kv_fp8_row_warp(x + r * (d_c + d_r), d_c, d_r, out + r * rb);
}

// One warp per 32-element block, lane = element.
__global__ void quant_fp4_kernel(const float* __restrict__ x, int64_t nblk, uint8_t* __restrict__ packed,
                                 uint8_t* __restrict__ scales) {
    const int64_t blk = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (blk >= nblk) return;
    quant_fp4_block_warp(x[blk * 32 + (threadIdx.x & 31)], packed + blk * 16, scales + blk);
}

// One block per token: the group projections into shared memory, then Wo.
__global__ void group_oproj_kernel(const float* __restrict__ o, int H, int d_v, const float* __restrict__ Wg,
                                   int G, int d_g, const float* __restrict__ Wo, int hidden, float* __restrict__ y) {
    extern __shared__ float sh[];
    const int gin = (H / G) * d_v;
    float* ot = sh;                 // [H * d_v]
    float* cat = sh + H * d_v;      // [G * d_g]
    const int64_t t = blockIdx.x;
    for (int i = threadIdx.x; i < H * d_v; i += blockDim.x) ot[i] = o[t * H * d_v + i];
    __syncthreads();
    for (int gc = threadIdx.x; gc < G * d_g; gc += blockDim.x) {
        const int g = gc / d_g, c = gc - g * d_g;
        const float* wg = Wg + (int64_t)g * gin * d_g + c;
        float acc = 0.f;
        for (int i = 0; i < gin; ++i) acc = fmaf(ot[g * gin + i], wg[(int64_t)i * d_g], acc);
        cat[gc] = acc;
    }
    __syncthreads();
    for (int c = threadIdx.x; c < hidden; c += blockDim.x) {
        float acc = 0.f;
        for (int i = 0; i < G * d_g; ++i) acc = fmaf(cat[i], Wo[(int64_t)i * hidden + c], acc);
        y[t * hidden + c] = acc;
    }
}

}  // namespace

cudaError_t launch_rope(void* rows, int dtype, int64_t n, int d, int d_rope, float theta, const int64_t* pos,
                        cudaStream_t s) {
    const int64_t work = n * (d_rope / 2);
    if (work == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((work + 255) / 256);
    if (dtype == LCS_F32)
        rope_kernel<float><<<grid, 256, 0, s>>>(static_cast<float*>(rows), n, d, d_rope, theta, pos);
    else
        rope_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<__nv_bfloat16*>(rows), n, d, d_rope, theta, pos);
    return cudaGetLastError();
}

cudaError_t launch_quant_kv_fp8(const float* x, int64_t n, int d_c, int d_r, void* out, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    quant_kv_fp8_kernel<<<(unsigned)((n + 7) / 8), 256, 0, s>>>(x, n, d_c, d_r, static_cast<uint8_t*>(out));
    return cudaGetLastError();
}

cudaError_t launch_quant_fp4(const float* x, int64_t n, int d, void* out, cudaStream_t s) {
    const int64_t nblk = n * (d / 32);
    if (nblk == 0) return cudaSuccess;
    uint8_t* packed = static_cast<uint8_t*>(out);
    uint8_t* scales = packed + n * (d / 2);
    quant_fp4_kernel<<<(unsigned)((nblk + 7) / 8), 256, 0, s>>>(x, nblk, packed, scales);
    return cudaGetLastError();
}

cudaError_t launch_group_oproj(const float* o, int64_t T, int H, int d_v, const float* Wg, int G, int d_g,
                               const float* Wo, int hidden, float* y, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const size_t smem = sizeof(float) * (H * d_v + G * d_g);
    cudaError_t err = set_smem_once(reinterpret_cast<const void*>(group_oproj_kernel), smem);
    if (err != cudaSuccess) return err;
    group_oproj_kernel<<<(unsigned)T, 256, smem, s>>>(o, H, d_v, Wg, G, d_g, Wo, hidden, y);
    return cudaGetLastError();
}

}  // namespace lcs
