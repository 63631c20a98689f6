// compress.cu -- streaming token compressor (CSA m=4 with overlap; HCA m'=128).
//
// "DeepSeek V4 深度解析" §2, CSA step 1: every m raw tokens' KV pooled into one
// entry with learned per-token weights plus a position bias, softmax-normalised,
// neighbouring blocks overlapping; HCA paragraph: the same with m' = 128.
//
// One warp per output entry.  The warp computes the window's softmax with
// shuffles (each lane owns positions lane, lane+32, ...), then streams the
// window's rows with 16-byte vector loads (lane c owns 16-byte chunks c, c+32,
// ... of every row, so each row read is coalesced), accumulates in fp32, stages
// the pooled row in shared memory, applies RoPE to the last d_rope dims and
// writes the entry with 16-byte stores.
#include <utility>

#include "lcs_common.cuh"
#include "lcs_internal.h"

namespace lcs {

namespace {

constexpr int kWarps = 8;

template <typename T>
struct Vec;
template <>
struct Vec<float> {
    static constexpr int N = 4;
    __device__ static void load(const float* p, float (&v)[8]) {
        float4 a = __ldg(reinterpret_cast<const float4*>(p));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    }
};
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void load(const __nv_bfloat16* p, float (&v)[8]) {
        uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
        uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kWarps * 32) compress_kernel(const Tin* __restrict__ x,
                                                              const Tin* __restrict__ x_tail,
                                                              const float* __restrict__ z_tail,
                                                              const float* __restrict__ z,
                                                              const float* __restrict__ bias, int64_t B, int64_t T,
                                                              int d, int m, int overlap, int d_rope, float theta,
                                                              int64_t pos0, Tout* __restrict__ out) {
    extern __shared__ float sh[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wp = m + overlap;
    const int wp_pad = (wp + 3) & ~3;
    float* pw = sh + warp * (wp_pad + d);   // softmax weights
    float* row = pw + wp_pad;               // pooled row (fp32)

    const int64_t n_out = T / m;
    const int64_t e = (int64_t)blockIdx.x * kWarps + warp;
    if (e >= B * n_out) return;
    const int64_t b = e / n_out, j = e - b * n_out;
    const int64_t t0 = m * j - overlap;   // token of window position 0

    // ---- softmax over the window (positions before the chunk are left out without a tail)
    float mx = -INFINITY;
    for (int i = lane; i < wp; i += 32) {
        const int64_t t = t0 + i;
        float l = -INFINITY;
        if (t >= 0) l = z[b * T + t] + bias[i];
        else if (x_tail != nullptr) l = z_tail[b * overlap + (overlap + t)] + bias[i];
        pw[i] = l;
        mx = fmaxf(mx, l);
    }
    mx = warp_max(mx);
    float sum = 0.f;
    for (int i = lane; i < wp; i += 32) {
        const float p = (pw[i] == -INFINITY) ? 0.f : expf(pw[i] - mx);
        pw[i] = p;
        sum += p;
    }
    sum = warp_sum(sum);
    const float inv = 1.f / sum;
    __syncwarp();

    // ---- weighted sum of the window rows, 16-byte chunks per lane
    constexpr int VN = Vec<Tin>::N;
    const int nchunk = d / VN;
    const Tin* xb = x + b * T * d;
    const Tin* tb = x_tail ? x_tail + b * overlap * d : nullptr;
    for (int c = lane; c < nchunk; c += 32) {
        float acc[VN];
#pragma unroll
        for (int v = 0; v < VN; ++v) acc[v] = 0.f;
        int i = 0;
        for (; i + 4 <= wp; i += 4) {
            float vals[4][8];
            float p[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t t = t0 + i + u;
                p[u] = pw[i + u];
                const Tin* src = (t >= 0) ? xb + t * d : (tb ? tb + (overlap + t) * d : nullptr);
                if (src != nullptr && p[u] != 0.f) Vec<Tin>::load(src + c * VN, vals[u]);
                else {
#pragma unroll
                    for (int v = 0; v < 8; ++v) vals[u][v] = 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < VN; ++v) acc[v] = fmaf(p[u], vals[u][v], acc[v]);
        }
        for (; i < wp; ++i) {
            const int64_t t = t0 + i;
            const float p = pw[i];
            const Tin* src = (t >= 0) ? xb + t * d : (tb ? tb + (overlap + t) * d : nullptr);
            if (src == nullptr || p == 0.f) continue;
            float vals[8];
            Vec<Tin>::load(src + c * VN, vals);
#pragma unroll
            for (int v = 0; v < VN; ++v) acc[v] = fmaf(p, vals[v], acc[v]);
        }
#pragma unroll
        for (int v = 0; v < VN; ++v) row[c * VN + v] = acc[v] * inv;
    }
    __syncwarp();

    // ---- RoPE on the last d_rope dims at the entry's last token position
    if (d_rope > 0) {
        const int half = d_rope / 2, c0 = d - d_rope;
        const double pos = (double)(pos0 + m * j + m - 1);
        for (int i = lane; i < half; i += 32) {
            const double freq = pow((double)theta, -2.0 * i / (double)d_rope);
            double a = pos * freq;
            a -= 6.283185307179586 * rint(a * 0.15915494309189535);   // reduce to [-pi, pi]
            float sn, cs;
            sincosf((float)a, &sn, &cs);
            const float x1 = row[c0 + i], x2 = row[c0 + i + half];
            row[c0 + i] = x1 * cs - x2 * sn;
            row[c0 + i + half] = x2 * cs + x1 * sn;
        }
        __syncwarp();
    }

    // ---- store
    Tout* o = out + e * d;
    if constexpr (sizeof(Tout) == 4) {
        for (int c = lane; c < d / 4; c += 32)
            reinterpret_cast<float4*>(o)[c] = make_float4(row[4 * c], row[4 * c + 1], row[4 * c + 2], row[4 * c + 3]);
    } else {
        for (int c = lane; c < d / 8; c += 32) {
            const float* r = row + 8 * c;
            uint4 v = make_uint4(pack_bf16x2(r[0], r[1]), pack_bf16x2(r[2], r[3]), pack_bf16x2(r[4], r[5]),
                                 pack_bf16x2(r[6], r[7]));
            reinterpret_cast<uint4*>(o)[c] = v;
        }
    }
}

template <typename Tin, typename Tout>
cudaError_t launch_t(const void* x, int64_t B, int64_t T, int d, const void* x_tail, const float* z_tail,
                     const float* z, const float* bias, int m, int overlap, int d_rope, float theta, int64_t pos0,
                     void* out, cudaStream_t s) {
    const size_t smem = sizeof(float) * kWarps * (((m + overlap + 3) & ~3) + d);
    auto kern = compress_kernel<Tin, Tout>;
    cudaError_t err = set_smem_once(reinterpret_cast<const void*>(kern), smem);
    if (err != cudaSuccess) return err;
    const int64_t n = B * (T / m);
    if (n == 0) return cudaSuccess;
    dim3 grid((unsigned)((n + kWarps - 1) / kWarps));
    kern<<<grid, kWarps * 32, smem, s>>>(static_cast<const Tin*>(x), static_cast<const Tin*>(x_tail), z_tail, z,
                                         bias, B, T, d, m, overlap, d_rope, theta, pos0, static_cast<Tout*>(out));
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_compress(const void* x, int x_dtype, int64_t B, int64_t T, int d, const void* x_tail,
                            const float* z_tail, const float* z, const float* bias, int m, int overlap, int d_rope,
                            float theta, int64_t pos0, void* out, int out_dtype, cudaStream_t s) {
    if (x_dtype == LCS_F32 && out_dtype == LCS_F32)
        return launch_t<float, float>(x, B, T, d, x_tail, z_tail, z, bias, m, overlap, d_rope, theta, pos0, out, s);
    if (x_dtype == LCS_F32 && out_dtype == LCS_BF16)
        return launch_t<float, __nv_bfloat16>(x, B, T, d, x_tail, z_tail, z, bias, m, overlap, d_rope, theta, pos0,
                                              out, s);
    if (x_dtype == LCS_BF16 && out_dtype == LCS_F32)
        return launch_t<__nv_bfloat16, float>(x, B, T, d, x_tail, z_tail, z, bias, m, overlap, d_rope, theta, pos0,
                                              out, s);
    return launch_t<__nv_bfloat16, __nv_bfloat16>(x, B, T, d, x_tail, z_tail, z, bias, m, overlap, d_rope, theta,
                                                  pos0, out, s);
}

}  // namespace lcs
