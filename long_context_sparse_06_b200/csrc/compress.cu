// compress.cu -- streaming token compressor (CSA m=4 with overlap; HCA m'=128).
//
// "DeepSeek V4 深度解析" §2, CSA step 1: every m raw tokens' KV pooled into one
// entry with learned per-token weights plus a position bias, softmax-normalised,
// neighbouring blocks overlapping; HCA paragraph: the same with m' = 128.
//
// bf16 rows (d a multiple of 64): the TMA-staged tile kernel below.  Otherwise one warp
// per output entry.  The warp computes the window's softmax with
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

// ------------------------------------------------------------------------------
// TMA-staged path: bf16 rows, d a multiple of 64, m + overlap <= 256, d_rope <= 64.
// A CTA pools a tile of E consecutive entries of one request (E a power of two, E*m +
// overlap <= 256 rows): the tile's rows are contiguous, so each 64-column block of them
// arrives with one 3-D TMA load (rows before the sequence start read as zeros), double-
// buffered.  Item (entry, 8-column group, row slice) -- E * 8 * S = 256 of them, S row
// slices summed with shuffles -- forms the pooled values; RoPE rotates the last d_rope
// dims (all in the last column block) in shared memory; the stores are 16-byte.
constexpr int kTThreads = 256;
constexpr int kTMaxRows = 256;

template <typename Tout>
__global__ void __launch_bounds__(kTThreads) compress_tma_kernel(
    const __grid_constant__ CUtensorMap map_x, const __nv_bfloat16* __restrict__ x_tail,
    const float* __restrict__ z_tail, const float* __restrict__ z, const float* __restrict__ bias, int64_t T, int d,
    int m, int overlap, int d_rope, float theta, int64_t pos0, int E, int S, int64_t tiles_per,
    Tout* __restrict__ out) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full[2];
    uint8_t* stage = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int R = E * m + overlap;   // stage rows
    const int wp = m + overlap;
    float* p_s = reinterpret_cast<float*>(stage + 2 * R * 128);   // [E][wp] pooling weights
    float* pool = p_s + E * wp;                                    // [E][64] pooled column block
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int64_t b = blockIdx.x / tiles_per;
    const int64_t j0 = (blockIdx.x - b * tiles_per) * E;   // first entry of the tile
    const int64_t n_out = T / m;
    const int ne = (int)((n_out - j0) < E ? (n_out - j0) : E);
    const int64_t t0 = m * j0 - overlap;   // token of stage row 0
    const int ncb = d / 64;

    if (t == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        fence_barrier_init();
        prefetch_tmap(&map_x);
    }
    __syncthreads();
    if (t == 0)
        for (int cb = 0; cb < 2 && cb < ncb; ++cb) {
            mbar_arrive_expect_tx(&full[cb], (uint32_t)(R * 128));
            tma_load_3d(stage + cb * R * 128, &map_x, &full[cb], 64 * cb, (int)t0, (int)b);
        }
    // ---- pooling weights, one warp per entry (positions before the sequence start are
    // left out unless a tail is given)
    for (int e = warp; e < ne; e += kTThreads / 32) {
        const int64_t te = t0 + (int64_t)e * m;
        float mx = -INFINITY;
        for (int i = lane; i < wp; i += 32) {
            const int64_t tt = te + i;
            float l = -INFINITY;
            if (tt >= 0) l = z[b * T + tt] + bias[i];
            else if (x_tail != nullptr) l = z_tail[b * overlap + (overlap + tt)] + bias[i];
            p_s[e * wp + i] = l;
            mx = fmaxf(mx, l);
        }
        mx = warp_max(mx);
        float sum = 0.f;
        for (int i = lane; i < wp; i += 32) {
            const float p = (p_s[e * wp + i] == -INFINITY) ? 0.f : expf(p_s[e * wp + i] - mx);
            p_s[e * wp + i] = p;
            sum += p;
        }
        sum = warp_sum(sum);
        const float inv = 1.f / sum;
        __syncwarp();
        for (int i = lane; i < wp; i += 32) p_s[e * wp + i] *= inv;
    }
    __syncthreads();
    const int ntail = (t0 < 0 && x_tail != nullptr) ? (int)(-t0) : 0;   // stage rows taken from the tail
    const int sl = t % S, rest = t / S, cg = rest & 7, ie = rest >> 3;
    const int per = (wp + S - 1) / S;
    const int i0 = sl * per, i1 = (i0 + per < wp) ? i0 + per : wp;
    for (int cb = 0; cb < ncb; ++cb) {
        const int st = cb & 1;
        uint8_t* sb = stage + st * R * 128;
        mbar_wait(&full[st], (uint32_t)((cb >> 1) & 1), nullptr, 401);
        if (ntail > 0) {
            for (int i = t; i < ntail * 8; i += kTThreads) {
                const int r = i >> 3, c = i & 7;
                const __nv_bfloat16* src = x_tail + (b * overlap + overlap + (t0 + r)) * d + 64 * cb + 8 * c;
                *reinterpret_cast<uint4*>(sb + r * 128 + c * 16) = __ldg(reinterpret_cast<const uint4*>(src));
            }
            __syncthreads();
        }
        float acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = 0.f;
        if (ie < ne)
            for (int i = i0; i < i1; ++i) {
                const float pw = p_s[ie * wp + i];
                const uint4 v = *reinterpret_cast<const uint4*>(sb + (ie * m + i) * 128 + cg * 16);
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    acc[2 * k] = fmaf(pw, __uint_as_float(w4[k] << 16), acc[2 * k]);
                    acc[2 * k + 1] = fmaf(pw, __uint_as_float(w4[k] & 0xFFFF0000u), acc[2 * k + 1]);
                }
            }
        for (int o = 1; o < S; o <<= 1)
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], o);
        if (sl == 0 && ie < ne)
#pragma unroll
            for (int k = 0; k < 8; ++k) pool[ie * 64 + cg * 8 + k] = acc[k];
        __syncthreads();   // stage st is read; the pooled block is complete
        if (t == 0 && cb + 2 < ncb) {
            mbar_arrive_expect_tx(&full[st], (uint32_t)(R * 128));
            tma_load_3d(sb, &map_x, &full[st], 64 * (cb + 2), (int)t0, (int)b);
        }
        if (cb == ncb - 1 && d_rope > 0) {
            // RoPE at each entry's last token position; the angle reduced in fp64
            const int half = d_rope / 2, c0 = 64 - d_rope;
            for (int i = t; i < ne * half; i += kTThreads) {
                const int e = i / half, k = i - e * half;
                const double pos = (double)(pos0 + m * (j0 + e) + m - 1);
                const double freq = pow((double)theta, -2.0 * k / (double)d_rope);
                double a = pos * freq;
                a -= 6.283185307179586 * rint(a * 0.15915494309189535);
                float sn, cs;
                sincosf((float)a, &sn, &cs);
                float* r = pool + e * 64 + c0;
                const float x1 = r[k], x2 = r[k + half];
                r[k] = x1 * cs - x2 * sn;
                r[k + half] = x2 * cs + x1 * sn;
            }
            __syncthreads();
        }
        for (int i = t; i < ne * 8; i += kTThreads) {
            const int e = i >> 3, c = i & 7;
            const float* r = pool + e * 64 + c * 8;
            Tout* o = out + (b * n_out + j0 + e) * d + 64 * cb + 8 * c;
            if constexpr (sizeof(Tout) == 4) {
                reinterpret_cast<float4*>(o)[0] = make_float4(r[0], r[1], r[2], r[3]);
                reinterpret_cast<float4*>(o)[1] = make_float4(r[4], r[5], r[6], r[7]);
            } else {
                reinterpret_cast<uint4*>(o)[0] = make_uint4(pack_bf16x2(r[0], r[1]), pack_bf16x2(r[2], r[3]),
                                                            pack_bf16x2(r[4], r[5]), pack_bf16x2(r[6], r[7]));
            }
        }
        __syncthreads();   // the pooled block is reused
    }
}

// Entries per tile for the TMA path (0: not applicable).
int tma_tile_entries(int d, int m, int overlap, int d_rope) {
    if (d % 64 || d_rope > 64 || m + overlap > kTMaxRows) return 0;
    int e = 32;
    while (e > 1 && e * m + overlap > kTMaxRows) e >>= 1;
    return e;
}

template <typename Tout>
cudaError_t launch_tma(const void* x, int64_t B, int64_t T, int d, const void* x_tail, const float* z_tail,
                       const float* z, const float* bias, int m, int overlap, int d_rope, float theta, int64_t pos0,
                       void* out, int E, cudaStream_t s) {
    const int R = E * m + overlap;
    const int S = kTThreads / (8 * E);
    CUtensorMap map;
    if (T >= (int64_t(1) << 31) || B >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
    if (!encode_tmap_3d(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)d, (uint64_t)T, (uint64_t)B,
                        (uint64_t)d * 2, (uint64_t)T * d * 2, 64, (uint32_t)R))
        return cudaErrorInvalidValue;
    const size_t smem = 128 + 2 * (size_t)R * 128 + sizeof(float) * ((size_t)E * (m + overlap) + (size_t)E * 64);
    auto kern = compress_tma_kernel<Tout>;
    cudaError_t err = set_smem_once(reinterpret_cast<const void*>(kern), smem);
    if (err != cudaSuccess) return err;
    const int64_t n_out = T / m;
    const int64_t tiles_per = (n_out + E - 1) / E;
    if (B * tiles_per == 0) return cudaSuccess;
    kern<<<(unsigned)(B * tiles_per), kTThreads, smem, s>>>(map, static_cast<const __nv_bfloat16*>(x_tail), z_tail, z,
                                                            bias, T, d, m, overlap, d_rope, theta, pos0, E, S,
                                                            tiles_per, static_cast<Tout*>(out));
    return cudaGetLastError();
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
    if (x_dtype == LCS_BF16) {
        const int E = tma_tile_entries(d, m, overlap, d_rope);
        if (E > 0) {
            if (out_dtype == LCS_F32)
                return launch_tma<float>(x, B, T, d, x_tail, z_tail, z, bias, m, overlap, d_rope, theta, pos0, out, E,
                                         s);
            return launch_tma<__nv_bfloat16>(x, B, T, d, x_tail, z_tail, z, bias, m, overlap, d_rope, theta, pos0, out,
                                             E, s);
        }
    }
    if (x_dtype == LCS_BF16 && out_dtype == LCS_F32)
        return launch_t<__nv_bfloat16, float>(x, B, T, d, x_tail, z_tail, z, bias, m, overlap, d_rope, theta, pos0,
                                              out, s);
    return launch_t<__nv_bfloat16, __nv_bfloat16>(x, B, T, d, x_tail, z_tail, z, bias, m, overlap, d_rope, theta,
                                                  pos0, out, s);
}

}  // namespace lcs
