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
// Exact on tensor cores without a sub-byte MMA:
//  * every E2M1 value is a bf16 value, and so is code * sq (<= 6 significant
//    bits); the query operand is therefore the dequantised query in bf16 and the
//    key operand the key codes in bf16 (converted in shared memory);
//  * one bf16 MMA per 32-block, each into its own TMEM accumulator, gives
//    E_{h,b} = sq_{h,b} * D_b exactly: every partial sum is an integer multiple of
//    one unit and below 2^17 of them, whatever the accumulation order;
//  * E_{h,b} * sk_{s,b} equals D_b * sq_{h,b} * sk_{s,b} exactly, so the epilogue
//    fma(E, sk, acc) chain reproduces the fma(D, sq*sk, acc) chain bit for bit.
//
// Kernel layout (persistent, one CTA per SM, 448 threads):
//   warp 0     TMA: packed key tiles [128 keys x 64 B] into a 6-stage raw ring, and
//              the group's dequantised query heads [64 x 128 bf16] into one of 2 slots
//   warp 1     tcgen05.mma (M = 128 keys, N = 64 heads, K = 32 per block) into one of
//              two 256-column accumulator sets (4 blocks x 64 heads)
//   warps 2-5  converters: one key row per thread, packed bytes -> bf16 codes through a
//              lane-replicated 256-entry table, into a 3-stage 128-byte-swizzled ring
//   warps 6-13 epilogue, two groups of 4 warps taking alternate tiles (one accumulator
//              set each): one key row per thread, block/heads combine, ReLU-weighted
//              head chain, bf16 score
#include <utility>

#include "lcs_common.cuh"
#include "lcs_internal.h"

namespace lcs {

namespace {

constexpr int kBM = 128, kHeads = 64, kDI = 128;
constexpr int kRawStages = 6, kAStages = 3;
constexpr int kRawTile = kBM * kDI / 2;           // 8 KB packed
constexpr int kATile = kBM * kDI * 2;             // 32 KB bf16
constexpr int kBTile = kHeads * kDI * 2;          // 16 KB bf16
constexpr int kLutBytes = 256 * 32 * 4;           // byte -> 2 bf16, one copy per lane
constexpr int kThreads = 448;
constexpr size_t kSmem = 1024 + kAStages * kATile + 2 * kBTile + kRawStages * kRawTile + kLutBytes;

struct Bars {
    uint64_t rfull[kRawStages], rempty[kRawStages];
    uint64_t afull[kAStages], aempty[kAStages];
    uint64_t bfull[2], bempty[2];
    uint64_t cfull[2], cempty[2];
    uint32_t tmem_base;
};

__device__ __forceinline__ int64_t avail(const int64_t* q_pos, int64_t g, int m, int64_t N_c) {
    if (q_pos == nullptr) return N_c;
    const int64_t a = (q_pos[g] + 1) / m;
    return a < 0 ? 0 : (a < N_c ? a : N_c);
}

// bf16 bits of an E2M1 code (value table of the OCP MX spec).
__device__ __forceinline__ uint32_t e2m1_bf16_bits(uint32_t nib) {
    constexpr uint32_t mag[8] = {0x0000, 0x3F00, 0x3F80, 0x3FC0, 0x4000, 0x4040, 0x4080, 0x40C0};
    return mag[nib & 7] | ((nib & 8) ? 0x8000u : 0u);
}

// Query quantiser: one warp per (group, head, 32-block); writes the dequantised values
// (code * scale, exact in bf16) as the B operand rows [groups * 64, 128].
__global__ void quant_q_fp4_kernel(const __nv_bfloat16* __restrict__ qI, int64_t nblk, uint16_t* __restrict__ qdq) {
    const int lane = threadIdx.x & 31;
    const int64_t blk = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (blk >= nblk) return;
    const float v = __bfloat162float(qI[blk * 32 + lane]);
    const float amax = warp_max(fabsf(v));
    uint8_t sc_code = f32_to_e4m3(amax / 6.0f);
    if ((sc_code & 0x7F) == 0) sc_code = 0x38;   // 1.0
    const float sc = e4m3_to_f32(sc_code);
    const uint32_t q = f32_to_e2m1(v / sc);
    const float val = __uint_as_float(e2m1_bf16_bits(q) << 16) * sc;   // exact
    qdq[blk * 32 + lane] = f32_to_bf16_bits(val);
}

__global__ void __launch_bounds__(kThreads, 1)
    index_fp4_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                        const uint8_t* __restrict__ k_scales, const float* __restrict__ w, int64_t Q, int64_t N_c,
                        const int64_t* __restrict__ q_pos, int m, int64_t groups, uint16_t* __restrict__ scores,
                        int* status) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ Bars bars;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* a_tiles = smem;                                   // 3 x 32 KB, SW128 bf16 codes
    uint8_t* b_tiles = a_tiles + kAStages * kATile;            // 2 x 16 KB, SW128 bf16 query
    uint8_t* raw = b_tiles + 2 * kBTile;                       // 6 x 8 KB packed keys
    uint32_t* lut = reinterpret_cast<uint32_t*>(raw + kRawStages * kRawTile);   // [256][32]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tiles_per = (N_c + kBM - 1) / kBM;
    const int64_t total = groups * tiles_per;
    const int64_t per = (total + gridDim.x - 1) / gridDim.x;
    const int64_t it0 = (int64_t)blockIdx.x * per;
    const int64_t it1 = (it0 + per < total) ? it0 + per : total;

    // byte -> (bf16 of the low nibble) | (bf16 of the high nibble) << 16, replicated per lane
    for (int i = threadIdx.x; i < 256 * 32; i += kThreads) {
        const uint32_t byte = (uint32_t)(i >> 5);
        lut[i] = e2m1_bf16_bits(byte & 15) | (e2m1_bf16_bits(byte >> 4) << 16);
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < kRawStages; ++i) { mbar_init(&bars.rfull[i], 1); mbar_init(&bars.rempty[i], 128); }
        for (int i = 0; i < kAStages; ++i) { mbar_init(&bars.afull[i], 128); mbar_init(&bars.aempty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars.bfull[i], 1);
            mbar_init(&bars.bempty[i], 1);
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
                    if (!mbar_wait(&bars.bempty[slot], (uint32_t)(((gseq >> 1) & 1) ^ 1), status, 111)) break;
                    mbar_arrive_expect_tx(&bars.bfull[slot], kBTile);
                    for (int kb = 0; kb < 2; ++kb)
                        tma_load_2d(b_tiles + slot * kBTile + kb * (kBTile / 2), &map_q, &bars.bfull[slot], kb * 64,
                                    (int)(g * kHeads));
                    prev_g = g;
                }
                const int rs = (int)(n_it % kRawStages);
                if (!mbar_wait(&bars.rempty[rs], (uint32_t)(((n_it / kRawStages) & 1) ^ 1), status, 112)) break;
                mbar_arrive_expect_tx(&bars.rfull[rs], kRawTile);
                tma_load_2d(raw + rs * kRawTile, &map_k, &bars.rfull[rs], 0, (int)(ti.b * N_c + tile * kBM));
                ++n_it;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer: block b of the K dim -> accumulator set (buf, b)
            constexpr uint32_t idesc = idesc_bf16(kBM, kHeads, false, false);
            const uint64_t a_desc0 = sw128_desc(smem_u32(a_tiles), 16, 1024);
            const uint64_t b_desc0 = sw128_desc(smem_u32(b_tiles), 16, 1024);
            int64_t prev_g = -1, gseq = -1, n_it = 0;
            int slot = 0;
            TileIt ti(it0, (int)tiles_per, (int)Q);
            for (int64_t it = it0; it < it1; ++it, ti.next((int)tiles_per, (int)Q)) {
                const int64_t g = ti.g, tile = ti.tile;
                if (tile * kBM >= avail(q_pos, g, m, N_c)) continue;
                if (g != prev_g) {
                    if (prev_g >= 0) mma_commit(&bars.bempty[slot]);
                    ++gseq;
                    slot = (int)(gseq & 1);
                    if (!mbar_wait(&bars.bfull[slot], (uint32_t)((gseq >> 1) & 1), status, 113)) break;
                    prev_g = g;
                }
                const int as = (int)(n_it % kAStages), cb = (int)(n_it & 1);
                if (!mbar_wait(&bars.cempty[cb], (uint32_t)(((n_it >> 1) & 1) ^ 1), status, 114)) break;
                if (!mbar_wait(&bars.afull[as], (uint32_t)((n_it / kAStages) & 1), status, 115)) break;
                tc_fence_after();
                const uint64_t ad = a_desc0 + (uint64_t)((as * kATile) >> 4);
                const uint64_t bd = b_desc0 + (uint64_t)((slot * kBTile) >> 4);
#pragma unroll
                for (int blk = 0; blk < 4; ++blk)
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        // K offset of block blk, step kk: column block blk/2, byte (blk%2)*64 + kk*32
                        const uint32_t off_a = (blk >> 1) * (kATile / 2) + (blk & 1) * 64 + kk * 32;
                        const uint32_t off_b = (blk >> 1) * (kBTile / 2) + (blk & 1) * 64 + kk * 32;
                        mma_bf16_ss(tmem + cb * 256 + blk * 64, ad + (off_a >> 4), bd + (off_b >> 4), idesc,
                                    kk ? 1u : 0u);
                    }
                mma_commit(&bars.aempty[as]);
                mma_commit(&bars.cfull[cb]);
                ++n_it;
            }
            if (prev_g >= 0) mma_commit(&bars.bempty[slot]);
        }
    } else if (warp < 6) {
        // ---------------- converters: thread = key row of the tile
        const int row = threadIdx.x - 64;
        int64_t n_it = 0;
        TileIt ti(it0, (int)tiles_per, (int)Q);
        for (int64_t it = it0; it < it1; ++it, ti.next((int)tiles_per, (int)Q)) {
            if (ti.tile * kBM >= avail(q_pos, ti.g, m, N_c)) continue;
            const int rs = (int)(n_it % kRawStages), as = (int)(n_it % kAStages);
            if (!mbar_wait(&bars.rfull[rs], (uint32_t)((n_it / kRawStages) & 1), status, 116)) break;
            if (!mbar_wait(&bars.aempty[as], (uint32_t)(((n_it / kAStages) & 1) ^ 1), status, 117)) break;
            const uint4* src = reinterpret_cast<const uint4*>(raw + rs * kRawTile + row * 64);
            uint8_t* dst = a_tiles + as * kATile;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {         // 32 codes per 16 bytes
                // rows 64 B apart: rotating the piece order by row/2 keeps the 8 rows of a
                // shared-memory phase on distinct banks
                const int q = (qq + (row >> 1)) & 3;
                const uint4 v = src[q];
                const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
                uint32_t o[16];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) o[4 * i + j] = lut[(((wv[i] >> (8 * j)) & 0xFF) << 5) + lane];
#pragma unroll
                for (int c = 0; c < 4; ++c) {        // 4 chunks of 8 bf16
                    const int ch = 4 * q + c;        // chunk 0..15 of the 256-byte row
                    *reinterpret_cast<uint4*>(dst + (ch >> 3) * (kATile / 2) + sw128_off(row, ch & 7)) =
                        make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&bars.rempty[rs]);
            mbar_arrive(&bars.afull[as]);
            ++n_it;
        }
    } else {
        // ---------------- epilogue: warps 6..13 in two groups of 4 (group e takes the tiles
        // with n_it % 2 == e, i.e. accumulator set e); TMEM lane quarter = warp % 4, thread =
        // key row.
        const int e = (warp - 6) >> 2;
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
            const float4* wg4 = reinterpret_cast<const float4*>(w + g * kHeads);   // L1-resident
            const int64_t s = tile * kBM + row;
            float sk[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) sk[i] = e4m3_to_f32((uint8_t)(skw >> (8 * i)));
            // the k-th tile of this group is the k-th use of accumulator set e
            if (!mbar_wait(&bars.cfull[e], (uint32_t)(n_it & 1), status, 118)) break;
            tc_fence_after();
            float acc = 0.f;
#pragma unroll
            for (int h0 = 0; h0 < kHeads; h0 += 8) {
                uint32_t ev[4][8];
#pragma unroll
                for (int blk = 0; blk < 4; ++blk)
                    tmem_ld8(tmem_addr(tmem, quarter * 32, e * 256 + blk * 64 + h0), ev[blk]);
                tmem_ld_wait();
#pragma unroll
                for (int j4 = 0; j4 < 2; ++j4) {
                    const float4 w4 = __ldg(wg4 + h0 / 4 + j4);
                    const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int j = 4 * j4 + jj;
                        float dot = __uint_as_float(ev[0][j]) * sk[0];
                        dot = fmaf(__uint_as_float(ev[1][j]), sk[1], dot);
                        dot = fmaf(__uint_as_float(ev[2][j]), sk[2], dot);
                        dot = fmaf(__uint_as_float(ev[3][j]), sk[3], dot);
                        acc = fmaf(wv[jj], dot > 0.f ? dot : 0.f, acc);
                    }
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

}  // namespace

int64_t index_fp4_scratch_bytes(int64_t B, int64_t Q, int d_I) { return B * Q * kHeads * d_I * 2; }

cudaError_t launch_index_fp4_tc(const void* qI, const float* w, const void* kI, int64_t B, int64_t Q, int64_t N_c,
                                int d_I, const int64_t* q_pos, int m, uint16_t* scores, uint8_t* q_scratch,
                                int* status, cudaStream_t s, bool pdl) {
    (void)d_I;
    const int64_t groups = B * Q;
    if (groups == 0 || N_c == 0) return cudaSuccess;
    // dequantised FP4 query -> q_scratch [groups * 64, 128] bf16
    const int64_t nblk = groups * kHeads * (kDI / 32);
    quant_q_fp4_kernel<<<(unsigned)((nblk + 7) / 8), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(qI), nblk,
                                                                   reinterpret_cast<uint16_t*>(q_scratch));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const uint8_t* packed = static_cast<const uint8_t*>(kI);
    const uint8_t* k_scales = packed + B * N_c * (kDI / 2);
    CUtensorMap mk, mq;
    if (!encode_tmap_2d(&mk, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, kDI / 2, (uint64_t)(B * N_c), kDI / 2, kDI / 2,
                        kBM, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    if (!encode_tmap_2d(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q_scratch, kDI, (uint64_t)(groups * kHeads), kDI * 2, 64,
                        kHeads, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    e = set_smem_once(reinterpret_cast<const void*>(index_fp4_tc_kernel), kSmem);
    if (e != cudaSuccess) return e;
    const int64_t total = groups * ((N_c + kBM - 1) / kBM);
    const int64_t grid = total < num_sms() ? total : num_sms();
    return launch_k(index_fp4_tc_kernel, dim3((unsigned)grid), dim3(kThreads), kSmem, s, pdl, mk, mq, k_scales, w, Q,
                    N_c, q_pos, m, groups, scores, status);
}

}  // namespace lcs
