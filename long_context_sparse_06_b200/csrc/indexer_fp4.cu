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
// The scaled block dots E_b = D_b * sq_b * sk_b come from the block-scaled FP4 tensor cores
// (tcgen05.mma kind::mxf4nvf4, E2M1 x E2M1, one UE4M3 scale per 16 elements and operand),
// one MMA per block b into an accumulator of its own: the MMA covers the 64 codes of the
// block pair holding b, with b's two 16-element scales set to sk_b (keys) and sq_b (query)
// and the partner block's set to 0.  Every term of that MMA then carries the same scale
// product, and D_b is a multiple of 1/4 below 1152 in magnitude, so E_b (at most 21
// significant bits) comes out exact; the hardware rounds sums of differently scaled terms
// with limited precision, which is why each block gets its own MMA.  With E_b exact,
//   fma(D_b, sq_b*sk_b, dot) = dot + E_b rounded once,
// so the epilogue forms the definition's chain with three fp32 additions per head.
//
// Operands reach shared memory packed (two codes per byte, low nibble first) by TMA with
// the 64-byte swizzle: a key row of 128 codes is one 64-byte swizzle row, and the block
// pair p starts 32 bytes after pair p-1.  Scale factors live in tensor memory, each row's
// four 16-element scales of one MMA packed into a 32-bit column, in every 32-lane quarter.
//
// Kernel layout (persistent, one CTA per SM, 320 threads):
//   warp 0     TMA: key tiles [128 keys x 64 B] into a 12-stage ring, and the group's
//              quantised query heads [64 x 64 B] into one of 2 slots
//   warp 1     tcgen05.mma (M = 128 keys, N = 32 heads, K = 64): per tile, for heads
//              0-31 then 32-63, one MMA per block into a 128-column accumulator slot (the
//              two slots alternate, so one half-tile's MMAs run under the other's epilogue)
//   warps 2-5  scale factors: per tile the keys' (16 columns, up to 4 tiles ahead), per
//              query group the heads' (16 columns), read from global memory and written to
//              tensor memory with tcgen05.st
//   warps 6-9  epilogue: one key row per thread; the half-tiles in order (heads 0-31, then
//              32-63); three fp32 additions, ReLU and the head chain per head, bf16 score
#include <utility>

#include "lcs_common.cuh"
#include "lcs_internal.h"

namespace lcs {

namespace {

constexpr int kBM = 128, kHeads = 64, kDI = 128;
constexpr int kKStages = 12;
constexpr int kKTile = kBM * (kDI / 2);     // 8 KB of packed key codes
constexpr int kQTile = kHeads * (kDI / 2);  // 4 KB
constexpr int kSfSlots = 4;                 // key scale-factor slots in tensor memory
constexpr int kThreads = 320;
constexpr size_t kSmem = 1024 + kKStages * kKTile + 2 * kQTile;
// Tensor memory columns: accumulator slots [3][block] (32 heads each), key scale factors
// [slot][block][4], query scale factors [group slot][half][block][2].
constexpr int kAccSlots = 2;
constexpr uint32_t kColAcc = 0, kColSfa = kAccSlots * 128, kColSfb = kColSfa + kSfSlots * 16;
static_assert(kColSfb + 2 * 16 <= 512, "tensor memory columns");

struct Bars {
    uint64_t kfull[kKStages], kempty[kKStages];
    uint64_t qfull[2], qempty[2];
    uint64_t sffull[kSfSlots], sfempty[kSfSlots];
    uint64_t cfull[kAccSlots], cempty[kAccSlots];   // accumulator slots (half-tiles)
    uint32_t tmem_base;
};

__device__ __forceinline__ int64_t avail(const int64_t* q_pos, int64_t g, int m, int64_t N_c) {
    if (q_pos == nullptr) return N_c;
    const int64_t a = (q_pos[g] + 1) / m;
    return a < 0 ? 0 : (a < N_c ? a : N_c);
}

// D(tmem) = A * B with per-16-element scales from tensor memory (E2M1 x E2M1, UE4M3).
__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, 0, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Instruction descriptor, kind::mxf4nvf4: E2M1 x E2M1, UE4M3 scales, K = 64, K-major.
__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N) {
    return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// The 32-bit scale-factor column word of block b for one row with block scale byte s: the
// MMA covering b spans blocks 2(b/2), 2(b/2)+1 as four 16-element groups; b's two get s,
// the partner's two get 0.
__device__ __forceinline__ uint32_t sf_word(uint32_t s, int b) {
    const uint32_t pair = s | (s << 8);
    return (b & 1) ? (pair << 16) : pair;
}

// Query quantiser: one warp per (group, head, 32-block), lane = element.  Writes the codes
// in the keys' packed layout (row = group*64 + head, 64 bytes, element 2j in the low
// nibble of byte j) and the scale's E4M3 byte at qsb[(group*64 + head)*4 + block].
__global__ void quant_q_fp4_kernel(const __nv_bfloat16* __restrict__ qI, int64_t nblk, uint8_t* __restrict__ codes,
                                   uint8_t* __restrict__ qsb) {
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
    if (lane == 0) qsb[blk] = sc_code;
}

__global__ void __launch_bounds__(kThreads, 1)
    index_fp4_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                        const uint8_t* __restrict__ k_scales, const uint8_t* __restrict__ qsb,
                        const float* __restrict__ w, int64_t Q, int64_t N_c, const int64_t* __restrict__ q_pos,
                        int m, int64_t groups, uint16_t* __restrict__ scores, int* status) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ Bars bars;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* k_tiles = smem;                              // 12 x 8 KB
    uint8_t* q_tiles = k_tiles + kKStages * kKTile;       // 2 x 4 KB

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tiles_per = (N_c + kBM - 1) / kBM;
    const int64_t total = groups * tiles_per;
    const int64_t per = (total + gridDim.x - 1) / gridDim.x;
    const int64_t it0 = (int64_t)blockIdx.x * per;
    const int64_t it1 = (it0 + per < total) ? it0 + per : total;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kKStages; ++i) {
            mbar_init(&bars.kfull[i], 1);
            mbar_init(&bars.kempty[i], 1);
        }
        for (int i = 0; i < kSfSlots; ++i) {
            mbar_init(&bars.sffull[i], 128);   // the four scale-factor warps
            mbar_init(&bars.sfempty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars.qfull[i], 1);
            mbar_init(&bars.qempty[i], 1);
        }
        for (int i = 0; i < kAccSlots; ++i) {
            mbar_init(&bars.cfull[i], 1);
            mbar_init(&bars.cempty[i], 4);    // the four epilogue warps
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
                    mbar_arrive_expect_tx(&bars.qfull[slot], kQTile);
                    tma_load_2d(q_tiles + slot * kQTile, &map_q, &bars.qfull[slot], 0, (int)(g * kHeads));
                    prev_g = g;
                }
                const int st = (int)(n_it % kKStages);
                if (!mbar_wait(&bars.kempty[st], (uint32_t)(((n_it / kKStages) & 1) ^ 1), status, 112)) break;
                mbar_arrive_expect_tx(&bars.kfull[st], kKTile);
                tma_load_2d(k_tiles + st * kKTile, &map_k, &bars.kfull[st], 0, (int)(ti.b * N_c + tile * kBM));
                ++n_it;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer: (head half, block b) -> accumulator (half, b)
            constexpr uint32_t idesc = idesc_nvf4(kBM, kHeads / 2);
            const uint64_t k_desc0 = sw64_desc(smem_u32(k_tiles), 512);
            const uint64_t q_desc0 = sw64_desc(smem_u32(q_tiles), 512);
            int64_t prev_g = -1, gseq = -1, n_it = 0;
            int slot = 0;
            bool ok = true;
            TileIt ti(it0, (int)tiles_per, (int)Q);
            for (int64_t it = it0; it < it1 && ok; ++it, ti.next((int)tiles_per, (int)Q)) {
                const int64_t g = ti.g, tile = ti.tile;
                if (tile * kBM >= avail(q_pos, g, m, N_c)) continue;
                if (g != prev_g) {
                    if (prev_g >= 0) mma_commit(&bars.qempty[slot]);
                    ++gseq;
                    slot = (int)(gseq & 1);
                    if (!mbar_wait(&bars.qfull[slot], (uint32_t)((gseq >> 1) & 1), status, 113)) break;
                    prev_g = g;
                }
                const int st = (int)(n_it % kKStages), sf = (int)(n_it % kSfSlots);
                if (!mbar_wait(&bars.kfull[st], (uint32_t)((n_it / kKStages) & 1), status, 115)) break;
                if (!mbar_wait(&bars.sffull[sf], (uint32_t)((n_it / kSfSlots) & 1), status, 116)) break;
                const uint64_t kd = k_desc0 + (uint64_t)((st * kKTile) >> 4);
                for (int hh = 0; hh < 2; ++hh) {
                    const int64_t j = 2 * n_it + hh;   // half-tile sequence number
                    const int as = (int)(j % kAccSlots);
                    if (!mbar_wait(&bars.cempty[as], (uint32_t)(((j / kAccSlots) & 1) ^ 1), status, 114)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // heads 32*hh .. 32*hh+31: 32 rows of 64 B further into the query tile
                    const uint64_t qd = q_desc0 + (uint64_t)((slot * kQTile + hh * 32 * 64) >> 4);
#pragma unroll
                    for (int blk = 0; blk < 4; ++blk)   // block pair blk/2: 32 bytes further along the row
                        mma_nvf4(tmem + kColAcc + as * 128 + blk * 32, kd + (uint64_t)((32 * (blk >> 1)) >> 4),
                                 qd + (uint64_t)((32 * (blk >> 1)) >> 4), idesc,
                                 tmem + kColSfa + sf * 16 + blk * 4, tmem + kColSfb + slot * 16 + (hh * 4 + blk) * 2);
                    mma_commit(&bars.cfull[as]);
                }
                if (!ok) break;
                mma_commit(&bars.kempty[st]);
                mma_commit(&bars.sfempty[sf]);
                ++n_it;
            }
            if (prev_g >= 0) mma_commit(&bars.qempty[slot]);
        }
    } else if (warp < 6) {
        // ---------------- scale factors: warp w writes the lanes of TMEM quarter w % 4 (the
        // MMA reads every quarter); lane i holds key rows i, 32+i, 64+i, 96+i and heads i,
        // 32+i.  Key scales (4 bytes per key, block b in byte b) come from the key plane's
        // scale plane, query scales from qsb; keys at or beyond N_c get 0.
        const uint32_t lanes = (uint32_t)((warp & 3) * 32) << 16;
        // the key scales of the valid tiles are loaded three tiles ahead of their use
        auto valid = [&](const TileIt& t) { return (int64_t)t.tile * kBM < avail(q_pos, t.g, m, N_c); };
        auto fetch = [&](const TileIt& t, int64_t itx, uint32_t (&dst)[4]) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int64_t sk = (int64_t)t.tile * kBM + c * 32 + lane;
                dst[c] = (itx < it1 && sk < N_c)
                             ? __ldg(reinterpret_cast<const uint32_t*>(k_scales + (t.b * N_c + sk) * 4))
                             : 0u;
            }
        };
        TileIt la(it0, (int)tiles_per, (int)Q);   // lookahead position
        int64_t ila = it0;
        auto advance = [&]() {   // la to the next valid tile (or past the end)
            do {
                ++ila;
                la.next((int)tiles_per, (int)Q);
            } while (ila < it1 && !valid(la));
        };
        while (ila < it1 && !valid(la)) {
            ++ila;
            la.next((int)tiles_per, (int)Q);
        }
        uint32_t p0[4], p1[4], p2[4];
        fetch(la, ila, p0);
        advance();
        fetch(la, ila, p1);
        advance();
        fetch(la, ila, p2);
        int64_t prev_g = -1, gseq = -1, n_it = 0;
        TileIt ti(it0, (int)tiles_per, (int)Q);
        for (int64_t it = it0; it < it1; ++it, ti.next((int)tiles_per, (int)Q)) {
            const int64_t g = ti.g;
            if (!valid(ti)) continue;
            if (g != prev_g) {
                ++gseq;
                const int slot = (int)(gseq & 1);
                // the slot's previous group is done with (its last MMA complete)
                if (!mbar_wait(&bars.qempty[slot], (uint32_t)(((gseq >> 1) & 1) ^ 1), status, 117)) break;
                const uint32_t* qw = reinterpret_cast<const uint32_t*>(qsb + g * kHeads * 4);
                uint32_t v[16];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const uint32_t s4 = __ldg(qw + hh * 32 + lane);   // head hh*32 + lane, blocks 0..3
#pragma unroll
                    for (int blk = 0; blk < 4; ++blk) {
                        v[(hh * 4 + blk) * 2] = sf_word((s4 >> (8 * blk)) & 0xFF, blk);
                        v[(hh * 4 + blk) * 2 + 1] = 0u;
                    }
                }
                tmem_st16(tmem + lanes + kColSfb + slot * 16, v);
                prev_g = g;
            }
            uint32_t cur[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                cur[c] = p0[c];
                p0[c] = p1[c];
                p1[c] = p2[c];
            }
            advance();
            fetch(la, ila, p2);
            const int sf = (int)(n_it % kSfSlots);
            if (!mbar_wait(&bars.sfempty[sf], (uint32_t)(((n_it / kSfSlots) & 1) ^ 1), status, 118)) break;
            uint32_t v[16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint32_t s4 = cur[c];   // key row c*32 + lane, blocks 0..3
#pragma unroll
                for (int blk = 0; blk < 4; ++blk) v[blk * 4 + c] = sf_word((s4 >> (8 * blk)) & 0xFF, blk);
            }
            tmem_st16(tmem + lanes + kColSfa + sf * 16, v);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars.sffull[sf]);
            ++n_it;
        }
    } else {
        // ---------------- epilogue: warps 6..9; TMEM lane quarter = warp % 4, thread = key row.
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        int64_t n_it = 0;
        TileIt ti(it0, (int)tiles_per, (int)Q);
        for (int64_t it = it0; it < it1; ++it, ti.next((int)tiles_per, (int)Q)) {
            const int64_t g = ti.g, tile = ti.tile;
            const int64_t n = avail(q_pos, g, m, N_c);
            if (tile * kBM >= n) continue;
            const float4* w4 = reinterpret_cast<const float4*>(w + g * kHeads);
            const int64_t s = tile * kBM + row;
            float acc = 0.f;
            bool ok = true;
            for (int hh = 0; hh < 2; ++hh) {
                const int64_t j = 2 * n_it + hh;
                const int as = (int)(j % kAccSlots);
                if (!mbar_wait(&bars.cfull[as], (uint32_t)((j / kAccSlots) & 1), status, 120)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll 2
                for (int h0 = 0; h0 < 32; h0 += 8) {
                    uint32_t dv[4][8];
#pragma unroll
                    for (int blk = 0; blk < 4; ++blk)
                        tmem_ld8(tmem_addr(tmem, quarter * 32, kColAcc + as * 128 + blk * 32 + h0), dv[blk]);
                    const float4 wa = __ldg(w4 + (hh * 32 + h0) / 4), wb = __ldg(w4 + (hh * 32 + h0) / 4 + 1);
                    const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        // fma(D_b, sq_b*sk_b, dot) with E_b = D_b*sq_b*sk_b exact: dot + E_b, rounded
                        float dot = __uint_as_float(dv[0][j]);
                        dot = __fadd_rn(dot, __uint_as_float(dv[1][j]));
                        dot = __fadd_rn(dot, __uint_as_float(dv[2][j]));
                        dot = __fadd_rn(dot, __uint_as_float(dv[3][j]));
                        acc = fmaf(wv[j], dot > 0.f ? dot : 0.f, acc);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.cempty[as]);
            }
            if (!ok) break;
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

// Query codes [groups*64, 64 B] then, 256-byte aligned, scale bytes [groups, 64, 4].
int64_t q_codes_bytes(int64_t groups) { return align256(groups * kHeads * (kDI / 2)); }

}  // namespace

int64_t index_fp4_scratch_bytes(int64_t B, int64_t Q, int d_I) {
    (void)d_I;
    return q_codes_bytes(B * Q) + B * Q * kHeads * 4;
}

cudaError_t launch_index_fp4_tc(const void* qI, const float* w, const void* kI, int64_t B, int64_t Q, int64_t N_c,
                                int d_I, const int64_t* q_pos, int m, uint16_t* scores, uint8_t* q_scratch,
                                int* status, cudaStream_t s, bool pdl) {
    (void)d_I;
    const int64_t groups = B * Q;
    if (groups == 0 || N_c == 0) return cudaSuccess;
    uint8_t* qcodes = q_scratch;
    uint8_t* qsb = q_scratch + q_codes_bytes(groups);
    const int64_t nblk = groups * kHeads * (kDI / 32);
    quant_q_fp4_kernel<<<(unsigned)((nblk + 7) / 8), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(qI), nblk, qcodes,
                                                                   qsb);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const uint8_t* packed = static_cast<const uint8_t*>(kI);
    const uint8_t* k_scales = packed + B * N_c * (kDI / 2);
    CUtensorMap mk, mq;
    // packed codes as bytes, 64 per row, 64-byte swizzle
    if (!encode_tmap_2d(&mk, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, kDI / 2, (uint64_t)(B * N_c), kDI / 2, kDI / 2,
                        kBM, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    if (!encode_tmap_2d(&mq, CU_TENSOR_MAP_DATA_TYPE_UINT8, qcodes, kDI / 2, (uint64_t)(groups * kHeads), kDI / 2,
                        kDI / 2, kHeads, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    e = set_smem_once(reinterpret_cast<const void*>(index_fp4_tc_kernel), kSmem);
    if (e != cudaSuccess) return e;
    const int64_t total = groups * ((N_c + kBM - 1) / kBM);
    const int64_t grid = total < num_sms() ? total : num_sms();
    return launch_k(index_fp4_tc_kernel, dim3((unsigned)grid), dim3(kThreads), kSmem, s, pdl, mk, mq, k_scales, qsb,
                    w, Q, N_c, q_pos, m, groups, scores, status);
}

}  // namespace lcs
