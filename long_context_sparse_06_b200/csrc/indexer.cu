// indexer.cu -- lightning-indexer scoring.
//
// "DeepSeek V4 深度解析" §2, CSA step 2: a light, low-rank indexer scores every
// compressed entry against the query; "V3 vs V4" page, "V4 改进一" (闪电索引器).
// Adopted form (the pages print none):
//   score[s] = sum_{h < H_I} w_h * ReLU(qI_h . kI_s)
// with the per-head dot in fp32 and the head sum as a fixed-order fma chain
// (h = 0, 1, ...), so that the score of an entry does not depend on where it
// sits in the batch or in the tile.
//
// Two paths:
//  * fp32 inputs: CUDA cores, the dot itself a fixed-order fma chain over d.
//  * bf16 inputs: tcgen05 tensor cores.  A CTA is persistent over (query group,
//    128-key tile) work items.  Warp 0 streams key tiles [128 x 128] with TMA
//    (128-byte swizzle) through a 4-stage ring and the group's query heads
//    [64 x 128] into one of two slots; warp 1 issues tcgen05.mma (M = 128 keys,
//    N = 64 heads, K = 128) into one of four TMEM accumulators; warps 2-5 read
//    the accumulator rows (one key per thread) with tcgen05.ld and apply the
//    ReLU / weighted head sum in fp32, writing one score per key.  The prefill form
//    (four queries per group, N = 256, two accumulators) has a second epilogue group,
//    warps 6-9: the groups take alternate work items, one accumulator each, since the
//    head chains of four queries take longer than the MMA of an item.
#include <utility>

#include "lcs_common.cuh"
#include "lcs_internal.h"

namespace lcs {

namespace {

__device__ __forceinline__ int64_t avail(const int64_t* q_pos, int64_t g, int m, int64_t N_c) {
    if (q_pos == nullptr) return N_c;
    const int64_t a = (q_pos[g] + 1) / m;
    return a < 0 ? 0 : (a < N_c ? a : N_c);
}

// ------------------------------------------------------------------ fp32 path
__global__ void index_f32_kernel(const float* __restrict__ qI, const float* __restrict__ w,
                                 const float* __restrict__ kI, int64_t Q, int64_t N_c, int H, int dI,
                                 const int64_t* __restrict__ q_pos, int m, float* __restrict__ scores) {
    extern __shared__ float sh[];
    float* qs = sh;            // [H, dI]
    float* ws = sh + H * dI;   // [H]
    const int64_t g = blockIdx.x;   // (b, q)
    const int64_t b = g / Q;
    for (int i = threadIdx.x; i < H * dI; i += blockDim.x) qs[i] = qI[g * H * dI + i];
    for (int i = threadIdx.x; i < H; i += blockDim.x) ws[i] = w[g * H + i];
    __syncthreads();
    const int64_t n = avail(q_pos, g, m, N_c);
    const float* kb = kI + b * N_c * dI;
    for (int64_t s = (int64_t)blockIdx.y * blockDim.x + threadIdx.x; s < N_c; s += (int64_t)gridDim.y * blockDim.x) {
        float acc = -INFINITY;
        if (s < n) {
            acc = 0.f;
            const float* kr = kb + s * dI;
            for (int h = 0; h < H; ++h) {
                float dot = 0.f;
                for (int c = 0; c < dI; ++c) dot = fmaf(qs[h * dI + c], kr[c], dot);
                const float r = dot > 0.f ? dot : 0.f;
                acc = fmaf(ws[h], r, acc);
            }
        }
        scores[g * N_c + s] = acc;
    }
}

// ------------------------------------------------------------- bf16 tcgen05 path
// 32 lanes x 32 bits, 32 consecutive columns (thread i: lane base + i, register j: column
// base + j).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// QB queries of one request share a group: their 64 x QB heads are the MMA's N, so each
// key tile is read once per QB queries (decode: QB = 1; prefill: QB = 4, N = 256).
constexpr int kBM = 128;        // keys per tile (MMA M)
constexpr int kHeads = 64;      // index heads per query
constexpr int kDI = 128;        // index dim (MMA K)
constexpr int kATile = kBM * kDI * 2;        // 32 KB
template <int QB>
struct IxCfg {
    static constexpr int kEpiGroups = QB == 1 ? 1 : 2;     // epilogue groups of four warps
    static constexpr int kQG = QB / kEpiGroups;            // queries per epilogue group
    static constexpr int kHStep = QB == 1 ? 16 : 32;       // heads per TMEM load round
    static constexpr int kThreads = 64 + 128 * kEpiGroups;
    static constexpr int kN = kHeads * QB;                 // MMA N
    static constexpr int kStages = QB == 1 ? 4 : 3;
    static constexpr int kAcc = QB == 1 ? 4 : 2;
    static constexpr int kBTile = kN * kDI * 2;            // 16 KB x QB
    static constexpr int kTmemCols = kAcc * kN;            // 256 or 512
    static constexpr size_t kSmem = 1024 + kStages * kATile + 2 * kBTile;
};

template <int QB>
struct IxBars {
    uint64_t full[IxCfg<QB>::kStages], empty[IxCfg<QB>::kStages];
    uint64_t bfull[2], bempty[2];
    uint64_t afull[IxCfg<QB>::kAcc], aempty[IxCfg<QB>::kAcc];
    uint32_t tmem_base;
};

// Entries of group gb (request b, queries QB*qb ...) available to its last query.
template <int QB>
__device__ __forceinline__ int64_t group_avail(const int64_t* q_pos, int64_t b, int64_t qb, int64_t Q, int m,
                                               int64_t N_c) {
    if (q_pos == nullptr) return N_c;
    int64_t n = 0;
#pragma unroll
    for (int qi = 0; qi < QB; ++qi) {
        const int64_t q = qb * QB + qi;
        if (q < Q) {
            const int64_t a = avail(q_pos, b * Q + q, m, N_c);
            n = a > n ? a : n;
        }
    }
    return n;
}

template <int QB>
__global__ void __launch_bounds__(IxCfg<QB>::kThreads, 1)
    index_bf16_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                         const float* __restrict__ w, int64_t Q, int64_t N_c, const int64_t* __restrict__ q_pos,
                         int m, int64_t n_groups, float* __restrict__ scores, int* status) {
    using C = IxCfg<QB>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ IxBars<QB> bars;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* a_tiles = smem;
    uint8_t* b_tiles = smem + C::kStages * kATile;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t nqb = (Q + QB - 1) / QB;   // groups per request
    const int64_t tiles_per = (N_c + kBM - 1) / kBM;
    const int64_t total = n_groups * tiles_per;
    const int64_t per = (total + gridDim.x - 1) / gridDim.x;
    const int64_t it0 = (int64_t)blockIdx.x * per;
    const int64_t it1 = (it0 + per < total) ? it0 + per : total;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kStages; ++i) { mbar_init(&bars.full[i], 1); mbar_init(&bars.empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&bars.bfull[i], 1); mbar_init(&bars.bempty[i], 1); }
        for (int i = 0; i < C::kAcc; ++i) { mbar_init(&bars.afull[i], 1); mbar_init(&bars.aempty[i], 4 * C::kEpiGroups); }
        fence_barrier_init();
        prefetch_tmap(&map_k);
        prefetch_tmap(&map_q);
    }
    if (warp == 1) {
        tmem_alloc(&bars.tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem_base;

#if defined(__CUDA_ARCH__)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer
            int64_t prev_g = -1, gseq = -1, n_it = 0;
            TileIt ti(it0, (int)tiles_per, (int)nqb);
            int64_t av_g = -1, av_n = 0;
            for (int64_t it = it0; it < it1; ++it, ti.next((int)tiles_per, (int)nqb)) {
                const int64_t g = ti.g, tile = ti.tile;
                if (g != av_g) {   // availability of the group, formed once per group
                    av_g = g;
                    av_n = group_avail<QB>(q_pos, ti.b, ti.q, Q, m, N_c);
                }
                if (tile * kBM >= av_n) continue;
                if (g != prev_g) {
                    ++gseq;
                    const int slot = (int)(gseq & 1);
                    if (!mbar_wait(&bars.bempty[slot], (uint32_t)(((gseq >> 1) & 1) ^ 1), status, 101)) break;
                    mbar_arrive_expect_tx(&bars.bfull[slot], C::kBTile);
                    for (int kb = 0; kb < 2; ++kb)
                        tma_load_2d(b_tiles + slot * C::kBTile + kb * (C::kBTile / 2), &map_q, &bars.bfull[slot],
                                    kb * 64, (int)((ti.b * Q + ti.q * QB) * kHeads));
                    prev_g = g;
                }
                const int st = (int)(n_it % C::kStages);
                if (!mbar_wait(&bars.empty[st], (uint32_t)(((n_it / C::kStages) & 1) ^ 1), status, 102)) break;
                mbar_arrive_expect_tx(&bars.full[st], kATile);
                for (int kb = 0; kb < 2; ++kb)
                    tma_load_2d(a_tiles + st * kATile + kb * (kATile / 2), &map_k, &bars.full[st], kb * 64,
                                (int)(ti.b * N_c + tile * kBM));
                ++n_it;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            constexpr uint32_t idesc = idesc_bf16(kBM, C::kN, false, false);
            int64_t prev_g = -1, gseq = -1, n_it = 0;
            int slot = 0;
            bool ok = true;
            TileIt ti(it0, (int)tiles_per, (int)nqb);
            int64_t av_g = -1, av_n = 0;
            for (int64_t it = it0; it < it1 && ok; ++it, ti.next((int)tiles_per, (int)nqb)) {
                const int64_t g = ti.g, tile = ti.tile;
                if (g != av_g) {   // availability of the group, formed once per group
                    av_g = g;
                    av_n = group_avail<QB>(q_pos, ti.b, ti.q, Q, m, N_c);
                }
                if (tile * kBM >= av_n) continue;
                if (g != prev_g) {
                    if (prev_g >= 0) mma_commit(&bars.bempty[slot]);   // previous group's heads are free
                    ++gseq;
                    slot = (int)(gseq & 1);
                    if (!mbar_wait(&bars.bfull[slot], (uint32_t)((gseq >> 1) & 1), status, 103)) { ok = false; break; }
                    prev_g = g;
                }
                const int st = (int)(n_it % C::kStages);
                const int ac = (int)(n_it % C::kAcc);
                if (!mbar_wait(&bars.aempty[ac], (uint32_t)(((n_it / C::kAcc) & 1) ^ 1), status, 104)) { ok = false; break; }
                if (!mbar_wait(&bars.full[st], (uint32_t)((n_it / C::kStages) & 1), status, 105)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a_base = smem_u32(a_tiles + st * kATile);
                const uint32_t b_base = smem_u32(b_tiles + slot * C::kBTile);
#pragma unroll
                for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = sw128_desc(a_base + kb * (kATile / 2) + kk * 32, 16, 1024);
                        const uint64_t bd = sw128_desc(b_base + kb * (C::kBTile / 2) + kk * 32, 16, 1024);
                        mma_bf16_ss(tmem + ac * C::kN, ad, bd, idesc, (kb | kk) ? 1u : 0u);
                    }
                mma_commit(&bars.empty[st]);
                mma_commit(&bars.afull[ac]);
                ++n_it;
            }
            if (prev_g >= 0) mma_commit(&bars.bempty[slot]);
        }
    } else {
        // ---------------- epilogue: warps 2..5 (and 6..9, the second group); TMEM lane
        // quarter = warp % 4, thread = key.  Every group takes every work item, group e the
        // queries e * kQG ... of the QB, so that an item's accumulator is released after
        // half the head chains a thread would otherwise run.  A thread's kQG head chains run
        // interleaved (each in its own fixed order h = 0..63), so that their fused
        // multiply-adds hide one another's latency.
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int egroup = (warp - 2) >> 2;
        const int q0 = egroup * C::kQG;
        int64_t n_it = 0, av_g = -1, av_n = 0;
        int64_t nq[C::kQG];
        const float4* wq[C::kQG];
        TileIt ti(it0, (int)tiles_per, (int)nqb);
        for (int64_t it = it0; it < it1; ++it, ti.next((int)tiles_per, (int)nqb)) {
            const int64_t tile = ti.tile;
            if (ti.g != av_g) {   // the group's queries: availability and head weights
                av_g = ti.g;
                av_n = group_avail<QB>(q_pos, ti.b, ti.q, Q, m, N_c);
#pragma unroll
                for (int qi = 0; qi < C::kQG; ++qi) {
                    const int64_t q = ti.q * QB + q0 + qi;
                    const int64_t gq = ti.b * Q + (q < Q ? q : ti.q * QB);
                    nq[qi] = q < Q ? avail(q_pos, gq, m, N_c) : -1;
                    wq[qi] = reinterpret_cast<const float4*>(w + gq * kHeads);   // L1-resident
                }
            }
            if (tile * kBM >= av_n) continue;
            const int ac = (int)(n_it % C::kAcc);
            if (!mbar_wait(&bars.afull[ac], (uint32_t)((n_it / C::kAcc) & 1), status, 106)) break;
            tc_fence_after();
            float acc[C::kQG];
#pragma unroll
            for (int qi = 0; qi < C::kQG; ++qi) acc[qi] = 0.f;
#pragma unroll 1
            for (int h0 = 0; h0 < kHeads; h0 += C::kHStep) {
                uint32_t d[C::kQG][C::kHStep];
#pragma unroll
                for (int qi = 0; qi < C::kQG; ++qi) {
                    const uint32_t ta = tmem_addr(tmem, quarter * 32, ac * C::kN + (q0 + qi) * kHeads + h0);
                    if constexpr (C::kHStep == 32) tmem_ld32(ta, d[qi]);
                    else tmem_ld16(ta, d[qi]);
                }
                tmem_ld_wait();
#pragma unroll
                for (int j4 = 0; j4 < C::kHStep / 4; ++j4) {
                    float4 wv[C::kQG];
#pragma unroll
                    for (int qi = 0; qi < C::kQG; ++qi) wv[qi] = __ldg(wq[qi] + h0 / 4 + j4);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
#pragma unroll
                        for (int qi = 0; qi < C::kQG; ++qi) {
                            const float ww = u == 0 ? wv[qi].x : u == 1 ? wv[qi].y : u == 2 ? wv[qi].z : wv[qi].w;
                            const float dot = __uint_as_float(d[qi][4 * j4 + u]);
                            acc[qi] = fmaf(ww, dot > 0.f ? dot : 0.f, acc[qi]);
                        }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.aempty[ac]);
            const int64_t s = tile * kBM + row;
            if (s < N_c)
#pragma unroll
                for (int qi = 0; qi < C::kQG; ++qi)
                    if (nq[qi] >= 0)
                        scores[(ti.b * Q + ti.q * QB + q0 + qi) * N_c + s] = (s < nq[qi]) ? acc[qi] : -INFINITY;
            ++n_it;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace

cudaError_t launch_index_f32(const float* qI, const float* w, const float* kI, int64_t B, int64_t Q, int64_t N_c,
                             int H_I, int d_I, const int64_t* q_pos, int m, float* scores, cudaStream_t s) {
    const int64_t groups = B * Q;
    if (groups == 0 || N_c == 0) return cudaSuccess;
    const size_t smem = sizeof(float) * (H_I * d_I + H_I);
    cudaError_t e = set_smem_once(reinterpret_cast<const void*>(index_f32_kernel), smem);
    if (e != cudaSuccess) return e;
    const int64_t ychunks = (N_c + 255) / 256;
    dim3 grid((unsigned)groups, (unsigned)(ychunks < 16 ? ychunks : 16));
    index_f32_kernel<<<grid, 256, smem, s>>>(qI, w, kI, Q, N_c, H_I, d_I, q_pos, m, scores);
    return cudaGetLastError();
}

cudaError_t launch_index_bf16_tc(const void* qI, const float* w, const void* kI, int64_t B, int64_t Q,
                                 int64_t N_c, int d_I, const int64_t* q_pos, int m, float* scores, int* status,
                                 cudaStream_t s, bool pdl) {
    const int64_t groups = B * Q;
    if (groups == 0 || N_c == 0) return cudaSuccess;
    (void)d_I;
    CUtensorMap mk, mq;
    if (!encode_tmap_2d(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kI, kDI, (uint64_t)(B * N_c), kDI * 2, 64, kBM,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const bool batched = Q >= 4;   // prefill: four queries per group
    const int qb = batched ? 4 : 1;
    if (!encode_tmap_2d(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, qI, kDI, (uint64_t)(groups * kHeads), kDI * 2, 64,
                        (uint32_t)(kHeads * qb), CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const int64_t n_groups = B * ((Q + qb - 1) / qb);
    const int64_t total = n_groups * ((N_c + kBM - 1) / kBM);
    const int64_t grid = total < num_sms() ? total : num_sms();
    if (batched) {
        cudaError_t e = set_smem_once(reinterpret_cast<const void*>(index_bf16_tc_kernel<4>), IxCfg<4>::kSmem);
        if (e != cudaSuccess) return e;
        return launch_k(index_bf16_tc_kernel<4>, dim3((unsigned)grid), dim3(IxCfg<4>::kThreads), IxCfg<4>::kSmem, s, pdl, mk,
                        mq, w, Q, N_c, q_pos, m, n_groups, scores, status);
    }
    cudaError_t e = set_smem_once(reinterpret_cast<const void*>(index_bf16_tc_kernel<1>), IxCfg<1>::kSmem);
    if (e != cudaSuccess) return e;
    return launch_k(index_bf16_tc_kernel<1>, dim3((unsigned)grid), dim3(IxCfg<1>::kThreads), IxCfg<1>::kSmem, s, pdl, mk, mq,
                    w, Q, N_c, q_pos, m, n_groups, scores, status);
}

}  // namespace lcs
