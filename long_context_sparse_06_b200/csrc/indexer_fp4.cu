// indexer_fp4.cu -- lightning indexer with the FP4 QK path.
//
// "DeepSeek V4 深度解析" §4 (FP4量化感知訓練): the indexer's Q and K paths are FP4;
// "V3 vs V4" page, "FP4 为什么能无损": index scores in BF16.  Keys are E2M1 with
// one E4M3 scale per 32 elements; the query (bf16) is quantised the same way.
//
// Per key s and head h, with D_b the block dot of the E2M1 codes, the score is
//   dot_h = fixed-order fma over blocks b of D_b * (sq_{h,b} * sk_{s,b}),
//   score = fma chain over heads of w_h * ReLU(dot_h), rounded to bf16.
//
// The block dots come from the FP4 tensor cores (tcgen05.mma kind::f8f6f4, E2M1 x E2M1,
// fp32 accumulate), one K = 32 MMA per block into an accumulator of its own.  E2M1
// values are multiples of 1/2 below 6 in magnitude, so a block dot is a multiple of 1/4
// below 1152: exact in fp32 whatever the accumulation order.  The scale product
// sq*sk (4 + 4 significant bits) and D_b * sq*sk (at most 21 bits) are exact too, so the
// epilogue's fma chain over the blocks rounds exactly where the definition does.
//
// Operands reach shared memory in the form the MMA reads: a TMA tensor map of type
// 16U4_ALIGN16B expands every 8 bytes of packed codes into a 16-byte slot (the FP4 form
// of kind::f8f6f4), with the 128-byte swizzle; a key row of 128 codes is one 128-byte
// swizzle row and the block b of a row starts 32 bytes after block b-1.
//
// Kernel layout (persistent, one CTA per SM, 320 threads):
//   warp 0     TMA: key tiles [128 keys x 128 codes] into an 8-stage ring, and the
//              group's quantised query heads [64 x 128 codes] into one of 2 slots
//   warp 1     tcgen05.mma (M = 128 keys, N = 64 heads, K = 32 per block) into one of two
//              256-column accumulator sets (4 blocks x 64 heads)
//   warps 2-9  epilogue, two groups of 4 warps taking alternate tiles (one accumulator
//              set each): one key row per thread; block combine and the ReLU-weighted
//              head chain in packed fp32x2 arithmetic (each lane rounds as the scalar
//              fma does), bf16 score
#include <utility>

#include "lcs_common.cuh"
#include "lcs_internal.h"

namespace lcs {

namespace {

constexpr int kBM = 128, kHeads = 64, kDI = 128;
constexpr int kKStages = 8;
constexpr int kKTile = kBM * 128;           // 16 KB in shared memory (codes + gaps)
constexpr int kQTile = kHeads * 128;        // 8 KB
// A 16U4_ALIGN16B copy counts the packed bytes it reads toward the mbarrier's transaction
// count, half of what it writes to shared memory.
constexpr uint32_t kKTx = kKTile / 2, kQTx = kQTile / 2;
constexpr int kThreads = 320;
constexpr size_t kSmem = 1024 + kKStages * kKTile + 2 * kQTile;

struct Bars {
    uint64_t kfull[kKStages], kempty[kKStages];
    uint64_t qfull[2], qempty[2];
    uint64_t cfull[2], cempty[2];
    uint32_t tmem_base;
};

__device__ __forceinline__ int64_t avail(const int64_t* q_pos, int64_t g, int m, int64_t N_c) {
    if (q_pos == nullptr) return N_c;
    const int64_t a = (q_pos[g] + 1) / m;
    return a < 0 ? 0 : (a < N_c ? a : N_c);
}

// Packed fp32x2 arithmetic (sm_100): each lane is rounded as the scalar instruction is.
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "mul.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 a, b, c, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 c, {%6, %7};\n\t"
        "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// Query quantiser: one warp per (group, head, 32-block), lane = element.  Writes the codes
// in the keys' packed layout (row = group*64 + head, 64 bytes, element 2j in the low
// nibble of byte j) and the scale as fp32 at qscale[(group*4 + block)*64 + head].
__global__ void quant_q_fp4_kernel(const __nv_bfloat16* __restrict__ qI, int64_t nblk, uint8_t* __restrict__ codes,
                                   float* __restrict__ qscale) {
    const int lane = threadIdx.x & 31;
    const int64_t blk = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (blk >= nblk) return;
    const float v = __bfloat162float(qI[blk * 32 + lane]);
    const float amax = warp_max(fabsf(v));
    uint8_t sc_code = f32_to_e4m3(amax / 6.0f);
    if ((sc_code & 0x7F) == 0) sc_code = 0x38;   // 1.0
    const float sc = e4m3_to_f32(sc_code);
    const uint32_t q = f32_to_e2m1(v / sc);
    const uint32_t other = __shfl_down_sync(0xffffffffu, q, 1);
    if ((lane & 1) == 0) codes[blk * 16 + lane / 2] = (uint8_t)(q | (other << 4));
    if (lane == 0) {
        const int64_t gh = blk >> 2;              // group * 64 + head
        const int64_t g = gh / kHeads;
        qscale[(g * 4 + (blk & 3)) * kHeads + (gh - g * kHeads)] = sc;
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    index_fp4_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                        const uint8_t* __restrict__ k_scales, const float* __restrict__ qscale,
                        const float* __restrict__ w, int64_t Q, int64_t N_c, const int64_t* __restrict__ q_pos,
                        int m, int64_t groups, uint16_t* __restrict__ scores, int* status) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ Bars bars;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* k_tiles = smem;                              // 8 x 16 KB
    uint8_t* q_tiles = k_tiles + kKStages * kKTile;       // 2 x 8 KB

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tiles_per = (N_c + kBM - 1) / kBM;
    const int64_t total = groups * tiles_per;
    const int64_t per = (total + gridDim.x - 1) / gridDim.x;
    const int64_t it0 = (int64_t)blockIdx.x * per;
    const int64_t it1 = (it0 + per < total) ? it0 + per : total;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kKStages; ++i) { mbar_init(&bars.kfull[i], 1); mbar_init(&bars.kempty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars.qfull[i], 1);
            mbar_init(&bars.qempty[i], 1);
            mbar_init(&bars.cfull[i], 1);
            mbar_init(&bars.cempty[i], 4);
        }
        fence_barrier_init();
        prefetch_tmap(&map_k);
        prefetch_tmap(&map_q);
    }
    if (warp == 1) {
        tmem_alloc(&bars.tmem_base, 512);
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
            TileIt ti(it0, (int)tiles_per, (int)Q);
            for (int64_t it = it0; it < it1; ++it, ti.next((int)tiles_per, (int)Q)) {
                const int64_t g = ti.g, tile = ti.tile;
                if (tile * kBM >= avail(q_pos, g, m, N_c)) continue;
                if (g != prev_g) {
                    ++gseq;
                    const int slot = (int)(gseq & 1);
                    if (!mbar_wait(&bars.qempty[slot], (uint32_t)(((gseq >> 1) & 1) ^ 1), status, 111)) break;
                    mbar_arrive_expect_tx(&bars.qfull[slot], kQTx);
                    tma_load_2d(q_tiles + slot * kQTile, &map_q, &bars.qfull[slot], 0, (int)(g * kHeads));
                    prev_g = g;
                }
                const int st = (int)(n_it % kKStages);
                if (!mbar_wait(&bars.kempty[st], (uint32_t)(((n_it / kKStages) & 1) ^ 1), status, 112)) break;
                mbar_arrive_expect_tx(&bars.kfull[st], kKTx);
                tma_load_2d(k_tiles + st * kKTile, &map_k, &bars.kfull[st], 0, (int)(ti.b * N_c + tile * kBM));
                ++n_it;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer: block b of the K dim -> accumulator (set, b)
            constexpr uint32_t idesc = idesc_e2m1(kBM, kHeads);
            const uint64_t k_desc0 = sw128_desc(smem_u32(k_tiles), 16, 1024);
            const uint64_t q_desc0 = sw128_desc(smem_u32(q_tiles), 16, 1024);
            int64_t prev_g = -1, gseq = -1, n_it = 0;
            int slot = 0;
            TileIt ti(it0, (int)tiles_per, (int)Q);
            for (int64_t it = it0; it < it1; ++it, ti.next((int)tiles_per, (int)Q)) {
                const int64_t g = ti.g, tile = ti.tile;
                if (tile * kBM >= avail(q_pos, g, m, N_c)) continue;
                if (g != prev_g) {
                    if (prev_g >= 0) mma_commit(&bars.qempty[slot]);
                    ++gseq;
                    slot = (int)(gseq & 1);
                    if (!mbar_wait(&bars.qfull[slot], (uint32_t)((gseq >> 1) & 1), status, 113)) break;
                    prev_g = g;
                }
                const int st = (int)(n_it % kKStages), cb = (int)(n_it & 1);
                if (!mbar_wait(&bars.cempty[cb], (uint32_t)(((n_it >> 1) & 1) ^ 1), status, 114)) break;
                if (!mbar_wait(&bars.kfull[st], (uint32_t)((n_it / kKStages) & 1), status, 115)) break;
                tc_fence_after();
                const uint64_t kd = k_desc0 + (uint64_t)((st * kKTile) >> 4);
                const uint64_t qd = q_desc0 + (uint64_t)((slot * kQTile) >> 4);
#pragma unroll
                for (int blk = 0; blk < 4; ++blk)   // block blk: 32 codes = 32 bytes further along the row
                    mma_f8f6f4_ss(tmem + cb * 256 + blk * 64, kd + (uint64_t)((32 * blk) >> 4),
                                  qd + (uint64_t)((32 * blk) >> 4), idesc, 0u);
                mma_commit(&bars.kempty[st]);
                mma_commit(&bars.cfull[cb]);
                ++n_it;
            }
            if (prev_g >= 0) mma_commit(&bars.qempty[slot]);
        }
    } else {
        // ---------------- epilogue: warps 2..9 in two groups of 4 (group e takes the tiles
        // with n_it % 2 == e, i.e. accumulator set e); TMEM lane quarter = warp % 4, thread =
        // key row.
        const int e = (warp - 2) >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        int64_t n_it = 0;   // tiles of this group so far
        // The key scales of this group's tile are prefetched two of its tiles early (tile
        // it + 4 of the sequence, when no tile is skipped); a mismatch loads them directly.
        auto load_sk = [&](int64_t b, int64_t tile) -> uint32_t {
            const int64_t ss = tile * kBM + row;
            return ss < N_c ? __ldg(reinterpret_cast<const uint32_t*>(k_scales + (b * N_c + ss) * 4)) : 0u;
        };
        int64_t pf_id[2] = {-1, -1};
        uint32_t pf_val[2] = {0u, 0u};
        int64_t nv = 0;   // valid tiles of the sequence so far (both groups)
        TileIt ti(it0, (int)tiles_per, (int)Q);
        for (int64_t it = it0; it < it1; ++it, ti.next((int)tiles_per, (int)Q)) {
            const int64_t g = ti.g, tile = ti.tile;
            const int64_t n = avail(q_pos, g, m, N_c);
            if (tile * kBM >= n) continue;
            if (((nv++) & 1) != e) continue;
            const uint32_t skw = (pf_id[0] == it) ? pf_val[0] : load_sk(ti.b, tile);
            pf_id[0] = pf_id[1];
            pf_val[0] = pf_val[1];
            pf_id[1] = -1;
            if (it + 4 < it1) {
                TileIt t4 = ti;
#pragma unroll
                for (int u = 0; u < 4; ++u) t4.next((int)tiles_per, (int)Q);
                pf_id[1] = it + 4;
                pf_val[1] = load_sk(t4.b, t4.tile);
            }
            // the group's query scales [4][64] and head weights [64] (L1-resident broadcasts)
            const float4* sq4 = reinterpret_cast<const float4*>(qscale + g * 4 * kHeads);
            const float4* w4 = reinterpret_cast<const float4*>(w + g * kHeads);
            const int64_t s = tile * kBM + row;
            float2 sk2[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float v = e4m3_to_f32((uint8_t)(skw >> (8 * i)));
                sk2[i] = make_float2(v, v);
            }
            // the k-th tile of this group is the k-th use of accumulator set e
            if (!mbar_wait(&bars.cfull[e], (uint32_t)(n_it & 1), status, 118)) break;
            tc_fence_after();
            float acc = 0.f;
#pragma unroll 2
            for (int h0 = 0; h0 < kHeads; h0 += 8) {
                uint32_t dv[4][8];
#pragma unroll
                for (int blk = 0; blk < 4; ++blk)
                    tmem_ld8(tmem_addr(tmem, quarter * 32, e * 256 + blk * 64 + h0), dv[blk]);
                float4 sq[4][2];
#pragma unroll
                for (int blk = 0; blk < 4; ++blk) {
                    sq[blk][0] = __ldg(sq4 + blk * (kHeads / 4) + h0 / 4);
                    sq[blk][1] = __ldg(sq4 + blk * (kHeads / 4) + h0 / 4 + 1);
                }
                const float4 wa = __ldg(w4 + h0 / 4), wb = __ldg(w4 + h0 / 4 + 1);
                const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 4; ++j) {   // heads h0 + 2j, h0 + 2j + 1
                    float2 c[4];
#pragma unroll
                    for (int blk = 0; blk < 4; ++blk) {
                        const float4 q4 = sq[blk][j >> 1];
                        c[blk] = mul2((j & 1) ? make_float2(q4.z, q4.w) : make_float2(q4.x, q4.y), sk2[blk]);
                    }
                    auto dd = [&](int blk) {
                        return make_float2(__uint_as_float(dv[blk][2 * j]), __uint_as_float(dv[blk][2 * j + 1]));
                    };
                    float2 dot = mul2(dd(0), c[0]);
                    dot = fma2(dd(1), c[1], dot);
                    dot = fma2(dd(2), c[2], dot);
                    dot = fma2(dd(3), c[3], dot);
                    acc = fmaf(wv[2 * j], dot.x > 0.f ? dot.x : 0.f, acc);
                    acc = fmaf(wv[2 * j + 1], dot.y > 0.f ? dot.y : 0.f, acc);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.cempty[e]);
            if (s < N_c) scores[g * N_c + s] = (s < n) ? f32_to_bf16_bits(acc) : (uint16_t)0xFF80u;   // -inf
            ++n_it;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Query codes [groups*64, 64 B] then, 256-byte aligned, scales fp32 [groups, 4, 64].
int64_t q_codes_bytes(int64_t groups) { return align256(groups * kHeads * (kDI / 2)); }

}  // namespace

int64_t index_fp4_scratch_bytes(int64_t B, int64_t Q, int d_I) {
    (void)d_I;
    return q_codes_bytes(B * Q) + B * Q * 4 * kHeads * 4;
}

cudaError_t launch_index_fp4_tc(const void* qI, const float* w, const void* kI, int64_t B, int64_t Q, int64_t N_c,
                                int d_I, const int64_t* q_pos, int m, uint16_t* scores, uint8_t* q_scratch,
                                int* status, cudaStream_t s, bool pdl) {
    (void)d_I;
    const int64_t groups = B * Q;
    if (groups == 0 || N_c == 0) return cudaSuccess;
    uint8_t* qcodes = q_scratch;
    float* qscale = reinterpret_cast<float*>(q_scratch + q_codes_bytes(groups));
    const int64_t nblk = groups * kHeads * (kDI / 32);
    quant_q_fp4_kernel<<<(unsigned)((nblk + 7) / 8), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(qI), nblk, qcodes,
                                                                   qscale);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const uint8_t* packed = static_cast<const uint8_t*>(kI);
    const uint8_t* k_scales = packed + B * N_c * (kDI / 2);
    CUtensorMap mk, mq;
    // packed codes, 128 per row (64 bytes); each 8 bytes land in a 16-byte slot
    if (!encode_tmap_2d(&mk, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, packed, kDI, (uint64_t)(B * N_c), kDI / 2, kDI,
                        kBM, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!encode_tmap_2d(&mq, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, qcodes, kDI, (uint64_t)(groups * kHeads), kDI / 2,
                        kDI, kHeads, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    e = set_smem_once(reinterpret_cast<const void*>(index_fp4_tc_kernel), kSmem);
    if (e != cudaSuccess) return e;
    const int64_t total = groups * ((N_c + kBM - 1) / kBM);
    const int64_t grid = total < num_sms() ? total : num_sms();
    return launch_k(index_fp4_tc_kernel, dim3((unsigned)grid), dim3(kThreads), kSmem, s, pdl, mk, mq, k_scales, qscale,
                    w, Q, N_c, q_pos, m, groups, scores, status);
}

}  // namespace lcs
