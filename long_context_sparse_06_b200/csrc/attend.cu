// attend.cu -- shared-KV MQA over a gathered row set (CSA sparse; HCA dense).
//
// "DeepSeek V4 深度解析" §2, CSA step 3: the selected compressed entries and the
// most recent 128 raw tokens are attended together; HCA paragraph: dense
// attention over every compressed entry plus the window; both use shared-KV
// multi-query attention.  For query (b,q) and head h:
//   o_h = sum_r softmax_r(scale * q_h . K_r) V_r,  V_r = first d_v dims of K_r,
// one softmax over the union of the selected (or all available) compressed
// rows and the window rows.
//
// Tensor-core path (H = 64, D = 576, d_v = 512; bf16 rows or FP8 rows), 448 threads:
//  * one CTA per (query, split of its row list); the row list is the window rows
//    (padded to whole chunks of 64) followed by the selected (CSA) or available (HCA)
//    compressed rows;
//  * warp 12 loads the 64 query heads once (TMA, 128-byte swizzle) and issues
//    tcgen05.mma with the query heads as M = 64:
//      S [64 heads x 64 rows] = Q [64 x 576] . K_chunk^T        (K-major x K-major)
//    warp 13 issues
//      O [64 heads x 512]    += P [64 x 64 rows] . V_chunk       (K-major x MN-major)
//    with P in bf16: for FP8 rows P = P_hi + P_lo, two bf16 parts (two MMAs per K step);
//    for bf16 rows a single part, and the softmax of chunk c+1 then runs under the P.V of
//    chunk c (it waits for that P.V only to rescale O).  O lives in
//    TMEM as two interleaved M=64 accumulators (dims 0-255 in lanes 0-15 of each
//    32-lane quarter, dims 256-511 in lanes 16-31), S double-buffered beside it;
//  * warps 4-11 fill a 2-stage ring, four warps per stage, writing the SW128 layout that
//    both MMAs read (the same bytes are the K-major B of Q.K^T and the MN-major B of
//    P.V): contiguous bf16 chunks (window rows, HCA's compressed rows) with one TMA tile
//    load per 128-byte column block; selected rows with 16-byte cp.async (row gathers
//    scale with the number of issuing warps, not with TMA); FP8 rows with
//    load-convert-store (E4M3 x power-of-two block scale -> bf16, exact).  A stage is
//    released in two halves (column blocks 0-3 after P.V's first 256 output dims, the
//    rest after all of it), and a TMA-filled stage lands in the same two halves, so the
//    next chunk's load and Q.K^T start under the current P.V.  Q and the
//    window chunks are fetched before the kernel waits for the preceding kernel
//    (programmatic dependent launch): they do not depend on it;
//  * warps 0-3 run the online softmax on S (fp32, exp2), write P_hi into the chunk's
//    RoPE column block (dead once Q.K^T has read it) and, for FP8 rows, P_lo into a block of
//    its own, rescale O in TMEM only when a head's running max grows by more than 2^8
//    in weight, and write O / l out through shared memory (coalesced);
//  * with several splits each CTA writes its unnormalised O and (m, l) to the
//    workspace, and attend_combine_kernel merges them in split order.
// F32 path (C1-sized problems): CUDA cores, fp32 online softmax.
#include <utility>

#include "lcs_common.cuh"
#include "lcs_internal.h"

namespace lcs {

namespace {

constexpr int kH = 64, kD = 576, kDv = 512, kChunk = 64;
constexpr int kBlk = kChunk * 128;            // one SW128 column block of a chunk: 64 rows x 128 B
constexpr int kStageBytes = 9 * kBlk;         // 72 KB
constexpr int kQBytes = 9 * (kH * 128);       // 72 KB
constexpr int kAtThreads = 448;   // 4 softmax, 8 producers, 1 Q.K^T issuer, 1 P.V issuer
constexpr int kWarpQK = 12, kWarpPV = 13;
constexpr int kProdWarps = 8, kProdThreads = kProdWarps * 32;
constexpr int kRowsPerWarp = kChunk / kProdWarps;   // gathered rows per producer warp and chunk
constexpr size_t kAtSmem = 1024 + kQBytes + 2 * kStageBytes + kBlk;   // + the low part of P
constexpr int kMaxSplits = 16;                // row-list splits per query (merged by attend_combine_kernel)
constexpr int kOPitchF32 = kDv * 4 + 16;      // staged O rows (padded)
constexpr int kOPitchBF16 = kDv * 2 + 16;
static_assert(kH * kOPitchF32 <= 2 * kStageBytes, "staged O fits in the stages");
static_assert(kH * kOPitchF32 + 4 * (2 * kH + kH / 2 * (kMaxSplits + 2)) <= 2 * kStageBytes,
              "staged O, (m, l) and the merge weights fit in the stages");

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.0f;              // log2 of the tolerated growth before O is rescaled

// Each stage is two halves with barriers of their own: column blocks 0-3 (dims 0-255) and
// blocks 4-8 (dims 256-575; block 8 also carries P after Q.K^T).  P.V releases the first half
// after its first 256 output dims, and Q.K^T starts on a first half that has landed, so a
// stage's next load overlaps the rest of its P.V and the next Q.K^T.
constexpr int kHalfBlocks = 4;   // blocks of the first half
struct AtBars {
    uint64_t qfull;
    uint64_t kfull[2][2], kempty[2][2];   // [stage][half]
    uint64_t sfull[2], sempty[2];
    uint64_t pfull[2];
    uint64_t ofull[2];   // P.V of chunk c done (per chunk parity)
    uint64_t odone;      // every P.V of this CTA done
    uint64_t rawfull[2]; // FP8 chunk codes landed (TMA), before widening
    uint32_t tmem_base;
    int nsel;
};

struct RowPlan {
    int64_t nsel;        // selected / available compressed rows
    int64_t win_lo;      // first window row index in win[b]
    int64_t nwin;
};

// Named barrier of the `count` threads of one producer group.
__device__ __forceinline__ void group_bar(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// AND of v over the `count` threads of one producer group (every thread reaches it once),
// so that the group takes one decision after per-thread bounded waits.
__device__ __forceinline__ bool group_all(int id, int count, bool v) {
    int r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 q, %1, 0;\n\tbar.red.and.pred p, %2, %3, q;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((int)v), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

// Two E4M3 codes (low byte first) times the power-of-two block scale s -> two bf16, exact:
// one conversion instruction per pair to f16 (exact: every E4M3 value is a normal f16),
// f16 -> fp32 exact, the product with a power of two exact in fp32 and representable in
// bf16, so the final rounding changes nothing.
__device__ __forceinline__ uint32_t widen_e4m3x2(uint32_t two, float s) {
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xFFFFu), __NV_E4M3);
    const float2 f = __half22float2(*reinterpret_cast<__half2*>(&h));
    return pack_bf16x2(f.x * s, f.y * s);
}

// 16 E4M3 codes (a uint4, low byte first) -> 16 bf16 (8 packed pairs).
__device__ __forceinline__ void widen16(uint4 v, float s, uint32_t (&o)[8]) {
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        o[2 * q] = widen_e4m3x2(w4[q], s);
        o[2 * q + 1] = widen_e4m3x2(w4[q] >> 16, s);
    }
}

// 16 codes of one row (a uint4) -> 16 bf16 written as the row's 16-byte chunks ch, ch+1
// of a SW128 column block.
__device__ __forceinline__ void widen_piece(uint8_t* blk, int r, int ch, uint4 v, float s) {
    uint32_t o[8];
    widen16(v, s, o);
    *reinterpret_cast<uint4*>(blk + sw128_off(r, ch)) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4*>(blk + sw128_off(r, ch + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
}

__device__ __forceinline__ RowPlan plan_rows(const AttendArgs& a, int64_t g, int nsel) {
    RowPlan p;
    const int64_t b = g / a.Q;
    p.nsel = nsel;
    if (a.q_pos == nullptr) {
        p.win_lo = 0;
        p.nwin = a.Tw;
    } else {
        const int64_t t = a.q_pos[g];
        const int64_t wp0 = a.win_pos0[b];
        int64_t lo = t - a.W + 1 - wp0, hi = t - wp0;
        if (lo < 0) lo = 0;
        if (hi > a.Tw - 1) hi = a.Tw - 1;
        p.win_lo = lo;
        p.nwin = hi >= lo ? hi - lo + 1 : 0;
    }
    return p;
}

// Row pointer of row position r of query g (bf16 rows: D elements; FP8: 656 B).
// sel = the query's selection (CSA; its first nsel entries are valid) or null (HCA).
__device__ __forceinline__ const uint8_t* row_ptr(const AttendArgs& a, int64_t b, const RowPlan& p,
                                                  const int32_t* sel, int64_t r, int row_bytes) {
    if (r < p.nsel) {
        const int64_t e = sel ? sel[r] : r;   // sel may be global (tensor-core path) or shared (fp32 path)
        return static_cast<const uint8_t*>(a.comp) + (b * a.N_c + e) * row_bytes;
    }
    return static_cast<const uint8_t*>(a.win) + (b * a.Tw + p.win_lo + (r - p.nsel)) * row_bytes;
}

// Window rows of query g: the rows r of win[b] with win_pos0[b] + r in [t-W+1, t]
// (decode, q_pos == NULL: every row).  They come first in the tensor-core path's row list.
struct WinPlan {
    int64_t win_lo, nwin;
};
__device__ __forceinline__ WinPlan plan_window(const AttendArgs& a, int64_t g) {
    WinPlan p;
    if (a.q_pos == nullptr) {
        p.win_lo = 0;
        p.nwin = a.Tw;
    } else {
        const int64_t b = g / a.Q;
        const int64_t t = a.q_pos[g];
        const int64_t wp0 = a.win_pos0[b];
        int64_t lo = t - a.W + 1 - wp0, hi = t - wp0;
        if (lo < 0) lo = 0;
        if (hi > a.Tw - 1) hi = a.Tw - 1;
        p.win_lo = lo;
        p.nwin = hi >= lo ? hi - lo + 1 : 0;
    }
    return p;
}
// HCA: compressed entries available to query g.
__device__ __forceinline__ int64_t hca_avail(const AttendArgs& a, int64_t g) {
    if (a.q_pos == nullptr) return a.N_c;
    const int64_t av = (a.q_pos[g] + 1) / a.m;
    return av < 0 ? 0 : (av < a.N_c ? av : a.N_c);
}

template <bool FP8>
__global__ void __launch_bounds__(kAtThreads, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_c,
                     const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_cr,
                     const __grid_constant__ CUtensorMap map_wr, const AttendArgs a, int splits, int cmerge,
                     float* __restrict__ part_o, float* __restrict__ part_ml, int* status) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ AtBars bars;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* q_s = smem;
    uint8_t* stage_s = smem + kQBytes;
    uint8_t* plo_s = stage_s + 2 * kStageBytes;   // low bf16 part of P (one block)
    // with the in-cluster split merge: this split's (m, l) per head beside its staged O
    float* ml_s = reinterpret_cast<float*>(stage_s + kH * kOPitchF32);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t g = blockIdx.x / splits;
    const int sp = blockIdx.x - (int)(g * splits);
    const int64_t b = g / a.Q;
    constexpr int row_bytes = FP8 ? 656 : kD * 2;

    if (threadIdx.x == 0) {
        mbar_init(&bars.qfull, 1);
        for (int i = 0; i < 2; ++i) {
            for (int hf = 0; hf < 2; ++hf) {
                mbar_init(&bars.kfull[i][hf], kProdThreads);   // every producer thread
                mbar_init(&bars.kempty[i][hf], 1);
            }
            mbar_init(&bars.pfull[i], 128);
            mbar_init(&bars.sfull[i], 1);
            mbar_init(&bars.sempty[i], 128);
            mbar_init(&bars.ofull[i], 1);
            mbar_init(&bars.rawfull[i], 1);
        }
        mbar_init(&bars.odone, 1);
        fence_barrier_init();
        prefetch_tmap(&map_q);
        prefetch_tmap(&map_c);
        prefetch_tmap(&map_w);
        if constexpr (FP8) {
            prefetch_tmap(&map_cr);
            prefetch_tmap(&map_wr);
        }
    }
    if (warp == kWarpQK) {
        tmem_alloc(&bars.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem_base;

    // ---- what does not depend on the preceding kernel: the window rows, which fill the
    // first chunks of the row list (the last one padded), and Q.
    const WinPlan wp = plan_window(a, g);
    const int64_t nwc = (wp.nwin + kChunk - 1) / kChunk;
    const int64_t comp_max = (a.idx != nullptr) ? a.k : hca_avail(a, g);
    const int64_t nch_max = nwc + (comp_max + kChunk - 1) / kChunk;
    // chunks are dealt to the splits round-robin: local chunk c is global chunk sp + splits*c
    // (the window chunks, loaded by TMA, and the gathered ones spread over the splits)
    auto gcof = [&](int c) -> int64_t { return sp + (int64_t)splits * c; };
    const bool q_wanted = sp < nch_max;
    if (warp == kWarpQK && lane == 0 && q_wanted) {
        mbar_arrive_expect_tx(&bars.qfull, kQBytes);
        for (int blk = 0; blk < 9; ++blk)
            tma_load_2d(q_s + blk * (kH * 128), &map_q, &bars.qfull, blk * 64, (int)(g * kH));
    }
    const int32_t* sel = (a.idx != nullptr) ? a.idx + g * a.k : nullptr;
    int nsel = 0;   // valid after the selection scan
    // Global chunk gc: window chunk (gc < nwc) or compressed chunk; rows beyond the valid
    // count are padding (masked in the softmax).
    auto chunk_valid = [&](int64_t gc) -> int {
        const int64_t v = gc < nwc ? wp.nwin - gc * kChunk : (int64_t)nsel - (gc - nwc) * kChunk;
        return (int)(v < kChunk ? v : kChunk);
    };

    // ---- producers: warps 4-7 fill stage 0 (local chunks 0, 2, ...), warps 8-11 stage 1.
    // All eight producer warps fill each chunk, chunks in order (a gather runs at about 60
    // GB/s per SM from eight issuing warps, 39 from four).  A whole chunk of consecutive rows
    // (window rows; HCA's compressed rows) comes by TMA, issued by the first producer thread:
    // bf16 rows as one tile load per 128-byte column block; FP8 rows as their codes, which
    // the producers then widen to bf16 in shared memory.  Other chunks are gathered row by
    // row, warp pw owning rows pw, pw+8, ..., pw+56 (lane i < 8 resolves row pw+8i): bf16
    // rows with 16-byte cp.async, FP8 rows
    // loaded, converted (exact with the power-of-two block scale) and stored.  The gathers
    // write zeros for rows past the chunk's valid count, so a partial chunk never reads
    // rows outside the query's row set (they may hold anything, NaN included).  All write
    // the SW128 layout both MMAs read.
    const bool producer = warp >= 4 && warp < 12;
    const int pw = warp - 4;   // producer warp 0..7
    auto contiguous = [&](int64_t gc) { return (gc < nwc || sel == nullptr) && chunk_valid(gc) == kChunk; };
    uint32_t raw_par = 0;     // FP8 TMA fills: bit st = phase parity of rawfull[st]
    auto row_src = [&](int64_t gc, int rr) -> const uint8_t* {
        if (rr >= chunk_valid(gc)) return nullptr;
        if (gc < nwc)
            return static_cast<const uint8_t*>(a.win) + (b * a.Tw + wp.win_lo + gc * kChunk + rr) * row_bytes;
        const int64_t j = (gc - nwc) * kChunk + rr;
        const int64_t e = sel ? (int64_t)__ldg(sel + j) : j;
        return static_cast<const uint8_t*>(a.comp) + (b * a.N_c + e) * row_bytes;
    };
    auto my_row_src = [&](int64_t gc) -> const uint8_t* {
        return (lane < kRowsPerWarp && !contiguous(gc)) ? row_src(gc, pw + kProdWarps * lane) : nullptr;
    };
    // Fills stage st with global chunk gc (its u-th use; u >= 1 waits for the P.V of the
    // previous use to release the halves) and arrives on both halves' kfull (the TMA bytes
    // complete them).  Returns false when a wait ran out.
    auto wait_half = [&](int u, int hf, int st) -> bool {
        return u < 1 ||
               group_all(1, kProdThreads, mbar_wait(&bars.kempty[st][hf], (uint32_t)((u - 1) & 1), status, 310 + hf));
    };
    auto fill = [&](int64_t gc, const uint8_t* my_src, int u, int st) -> bool {
        uint8_t* dst = stage_s + st * kStageBytes;
        if (contiguous(gc) && !FP8) {
            // bf16 rows by TMA, half by half: the first half's load starts as soon as P.V has
            // released it
            const bool w = gc < nwc;
            const int row0 = w ? (int)(b * a.Tw + wp.win_lo + gc * kChunk) : (int)(b * a.N_c + (gc - nwc) * kChunk);
            for (int hf = 0; hf < 2; ++hf) {
                if (!wait_half(u, hf, st)) return false;
                const int b0 = hf ? kHalfBlocks : 0, b1 = hf ? 9 : kHalfBlocks;
                if (pw == 0 && lane == 0) {
                    mbar_arrive_expect_tx(&bars.kfull[st][hf], (b1 - b0) * kBlk);
                    for (int blk = b0; blk < b1; ++blk)
                        tma_load_2d(dst + blk * kBlk, w ? &map_w : &map_c, &bars.kfull[st][hf], blk * 64, row0);
                } else {
                    mbar_arrive(&bars.kfull[st][hf]);
                }
            }
            return true;
        }
        if constexpr (!FP8) {
            // gathered bf16 rows, half by half like the TMA fills: column blocks 0-3 (lane l
            // copies 16-byte chunk l of each of the warp's rows) as soon as P.V has released
            // them, then blocks 4-8; each half is announced once its copies have landed
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                if (!wait_half(u, hf, st)) return false;
#pragma unroll
                for (int i = 0; i < kRowsPerWarp; ++i) {
                    const int rr = pw + kProdWarps * i;
                    const uint8_t* src = reinterpret_cast<const uint8_t*>(
                        __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(my_src), i));
                    const bool valid = src != nullptr;
                    const uint8_t* base = valid ? src : static_cast<const uint8_t*>(a.comp);
                    for (int ch = hf ? 32 + lane : lane; ch < (hf ? 72 : 32); ch += 32)
                        cp_async_16(dst + (ch >> 3) * kBlk + sw128_off(rr, ch & 7), base + (valid ? ch * 16 : 0),
                                    valid);
                }
                cp_async_commit();
            }
            cp_async_wait<1>();
            fence_proxy_async_smem();
            mbar_arrive(&bars.kfull[st][0]);
            cp_async_wait<0>();
            fence_proxy_async_smem();
            mbar_arrive(&bars.kfull[st][1]);
            return true;
        }
        // every other fill writes the whole stage: wait for both halves first
        if (!wait_half(u, 0, st) || !wait_half(u, 1, st)) return false;
        if (FP8 && contiguous(gc)) {
            const bool w = gc < nwc;
            const int row0 = w ? (int)(b * a.Tw + wp.win_lo + gc * kChunk) : (int)(b * a.N_c + (gc - nwc) * kChunk);
            {
                // the codes of column block j (64 rows x 64 B) land in the upper half of
                // block j, the RoPE dims (bf16, 128-byte swizzle) in block 8; producer thread
                // tg then widens 16 codes of row tg/4 per block (piece tg%4), reading block
                // j+1's codes before the producers' barrier that lets block j+1 be written
                const int tg = pw * 32 + lane;
                if (tg == 0) {
                    mbar_arrive_expect_tx(&bars.rawfull[st], 8 * (kBlk / 2) + kBlk);
                    for (int j = 0; j < 8; ++j)
                        tma_load_2d(dst + j * kBlk + kBlk / 2, w ? &map_w : &map_c, &bars.rawfull[st], j * 64, row0);
                    tma_load_2d(dst + 8 * kBlk, w ? &map_wr : &map_cr, &bars.rawfull[st], 512, row0);
                }
                const int r1 = tg >> 2, piece = tg & 3;
                const uint8_t* scales = static_cast<const uint8_t*>(w ? a.win : a.comp) + (int64_t)row0 * 656 + 640;
                const float4 s1 = __ldg(reinterpret_cast<const float4*>(scales + (int64_t)r1 * 656));
                const bool landed = group_all(1, kProdThreads,
                                              mbar_wait(&bars.rawfull[st], (raw_par >> st) & 1u, status, 311));
                raw_par ^= 1u << st;
                if (landed) {
                    const uint4* raw0 = reinterpret_cast<const uint4*>(dst + kBlk / 2);
                    uint4 c1 = raw0[tg];
                    group_bar(1, kProdThreads);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        uint4 n1 = c1;
                        if (j < 7) n1 = reinterpret_cast<const uint4*>(dst + (j + 1) * kBlk + kBlk / 2)[tg];
                        const int sj = j >> 1;
                        const float f1 = sj == 0 ? s1.x : sj == 1 ? s1.y : sj == 2 ? s1.z : s1.w;
                        widen_piece(dst + j * kBlk, r1, 2 * piece, c1, f1);
                        if (j < 7) group_bar(1, kProdThreads);
                        c1 = n1;
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(&bars.kfull[st][0]);
                mbar_arrive(&bars.kfull[st][1]);
                return true;
            }
        }
        {
            // FP8 row: 32 content pieces of 16 codes (-> 32 bf16) and 8 RoPE pieces of 8 bf16;
            // the warp's 8 rows' loads in flight per lane
            for (int i0 = 0; i0 < kRowsPerWarp; i0 += 8) {
                uint4 cv[8], rv[8];
                float sc[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint8_t* src = reinterpret_cast<const uint8_t*>(
                        __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(my_src), i0 + u));
                    cv[u] = make_uint4(0, 0, 0, 0);
                    rv[u] = make_uint4(0, 0, 0, 0);
                    sc[u] = 0.f;
                    if (src != nullptr) {
                        cv[u] = __ldg(reinterpret_cast<const uint4*>(src + lane * 16));
                        sc[u] = __ldg(reinterpret_cast<const float*>(src + 640) + (lane >> 3));
                        if (lane < 8) rv[u] = __ldg(reinterpret_cast<const uint4*>(src + 512 + lane * 16));
                    }
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int rr = pw + kProdWarps * (i0 + u);
                    // lane's 16 codes are the row's chunks 2*lane, 2*lane+1: block lane/4
                    widen_piece(dst + (lane >> 2) * kBlk, rr, (lane & 3) * 2, cv[u], sc[u]);
                    if (lane < 8) *reinterpret_cast<uint4*>(dst + 8 * kBlk + sw128_off(rr, lane)) = rv[u];
                }
            }
        }
        fence_proxy_async_smem();
        mbar_arrive(&bars.kfull[st][0]);
        mbar_arrive(&bars.kfull[st][1]);
        return true;
    };
    // Window chunks need no selection: the producers fill them (up to both stages) before
    // the wait for the preceding kernel.
    int pre = 0;   // local chunks filled before the wait
    if (producer)
        while (pre < 2 && gcof(pre) < nwc && fill(gcof(pre), my_row_src(gcof(pre)), 0, pre)) ++pre;
#if defined(__CUDA_ARCH__)
    asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
    // ---- selection length (CSA: the valid prefix of idx, as top-k emits it; HCA: n_avail).
    // An index >= N_c ends the prefix and is reported through the status word.
    if (a.idx != nullptr) {
        // every thread checks a few entries (one load round), then a block minimum
        if (threadIdx.x == 0) bars.nsel = a.k;
        __syncthreads();
        int first_bad = a.k;
        for (int i = threadIdx.x; i < a.k; i += kAtThreads) {
            const int32_t v = __ldg(sel + i);
            if (v < 0 || v >= a.N_c) {
                if (v >= a.N_c) set_status(status, LCS_ERR_DEVICE, 201);
                first_bad = min(first_bad, i);
            }
        }
        first_bad = __reduce_min_sync(0xffffffffu, first_bad);
        if (lane == 0 && first_bad < a.k) atomicMin(&bars.nsel, first_bad);
    } else if (threadIdx.x == 0) {
        bars.nsel = (int)comp_max;
    }
    __syncthreads();
    nsel = bars.nsel;
    const int64_t nch_all = nwc + (nsel + kChunk - 1) / kChunk;
    const int nch = sp < nch_all ? (int)((nch_all - sp + splits - 1) / splits) : 0;

    constexpr uint32_t idesc_qk = idesc_bf16(64, kChunk, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16(64, 256, false, true);
    // TMEM: O in columns 0..255 (dims 0-255 at lane offset 0, dims 256-511 at lane
    // offset 16: two interleaved M=64 accumulators), S double-buffered in 256..383.
    auto t_s = [&](int buf) { return tmem + 256u + 64u * (uint32_t)buf; };

    if (warp == kWarpQK) {
        if (lane == 0 && q_wanted) {
            // ---------------- Q.K^T issue
            bool ok = mbar_wait(&bars.qfull, 0, status, 300);
            const uint64_t q_desc = sw128_desc(smem_u32(q_s), 16, 1024);
            const uint64_t k_desc0 = sw128_desc(smem_u32(stage_s), 16, 1024);
            for (int c = 0; c < nch && ok; ++c) {
                const int st = c & 1;
                if (c >= 2 && !mbar_wait(&bars.sempty[st], (uint32_t)(((c - 2) >> 1) & 1), status, 302)) break;
                const uint64_t kd = k_desc0 + (uint64_t)((st * kStageBytes) >> 4);
                for (int hf = 0; hf < 2 && ok; ++hf) {   // each half as soon as it has landed
                    if (!mbar_wait(&bars.kfull[st][hf], (uint32_t)((c >> 1) & 1), status, 301)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int b0 = hf ? kHalfBlocks : 0, b1 = hf ? 9 : kHalfBlocks;
                    for (int blk = b0; blk < b1; ++blk)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_bf16_ss(t_s(st), q_desc + (uint64_t)((blk * (kH * 128) + kk * 32) >> 4),
                                        kd + (uint64_t)((blk * kBlk + kk * 32) >> 4), idesc_qk, (blk | kk) ? 1u : 0u);
                }
                if (!ok) break;
                mma_commit(&bars.sfull[st]);
            }
        }
    } else if (warp == kWarpPV) {
        if (lane == 0 && nch > 0) {
            // ---------------- P.V issue (its own thread, so that it never waits behind the
            // next chunk's Q.K^T, which waits for that chunk's gather); P = P_hi + P_lo
            const uint64_t k_desc0 = sw128_desc(smem_u32(stage_s), 16, 1024);
            const uint64_t v_desc0 = sw128_desc(smem_u32(stage_s), kBlk, 1024);
            for (int c = 0; c < nch; ++c) {
                const int st = c & 1;
                if (!mbar_wait(&bars.pfull[st], (uint32_t)((c >> 1) & 1), status, 303)) break;
                tc_fence_after();
                const uint64_t pd = k_desc0 + (uint64_t)((st * kStageBytes + 8 * kBlk) >> 4);
                const uint64_t pld = k_desc0 + (uint64_t)((2 * kStageBytes) >> 4);
                const uint64_t vd = v_desc0 + (uint64_t)((st * kStageBytes) >> 4);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t od = tmem + (half ? (16u << 16) : 0u);
                        const uint64_t vk = vd + (uint64_t)((half * 4 * kBlk + kk * 2048) >> 4);
                        mma_bf16_ss(od, pd + (uint64_t)((kk * 32) >> 4), vk, idesc_pv, (c | kk) ? 1u : 0u);
                        if constexpr (FP8) mma_bf16_ss(od, pld + (uint64_t)((kk * 32) >> 4), vk, idesc_pv, 1u);
                    }
                    // dims 0-255 read blocks 0-3; the second half (blocks 4-7, and P in block 8)
                    // is released after the rest
                    mma_commit(&bars.kempty[st][half]);
                }
                mma_commit(&bars.ofull[st]);
            }
            mma_commit(&bars.odone);
        }
    } else if (producer) {
        // ---------------- producer loop: local chunks pre, pre+1, ... in order, stage c & 1;
        // a stage is refilled once the P.V that read it is complete.  The next chunk's row
        // sources are resolved while this chunk's copies are in flight.
        const uint8_t* nxt = (pre < nch) ? my_row_src(gcof(pre)) : nullptr;
        for (int c = pre; c < nch; ++c) {
            const uint8_t* my_src = nxt;
            if (c + 1 < nch) nxt = my_row_src(gcof(c + 1));
            // the producers leave together (their waits are group decisions)
            if (!fill(gcof(c), my_src, c >> 1, c & 1)) break;
        }
    } else if (warp < 4) {
        // ---------------- softmax / correction / epilogue: warps 0..3.  Warp q owns heads
        // 16q..16q+15; lane l works on head 16q + (l & 15) and, with the 16x32bx2 TMEM
        // load, on S columns 0-31 (lanes 0-15) or 32-63 (lanes 16-31).
        const int quarter = warp;
        const int hl = lane & 15;
        const int head = quarter * 16 + hl;
        const int cbase = (lane < 16) ? 0 : 32;   // this lane's S columns
        float m_used = -INFINITY;                 // log2-domain running max used for exponentials
        float l_sum = 0.f;                        // sum of the weights (both lane halves)
        const float sl2 = a.scale * kLog2e;
        for (int c = 0; c < nch; ++c) {
            const int st = c & 1;
            if (!mbar_wait(&bars.sfull[st], (uint32_t)((c >> 1) & 1), status, 320)) break;
            tc_fence_after();
            uint32_t sv[32];
            tmem_ld16x2_32(tmem_addr(t_s(st), quarter * 32, 0), sv);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&bars.sempty[st]);
            const int nvalid = chunk_valid(gcof(c));
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (cbase + j < nvalid) mx = fmaxf(mx, __uint_as_float(sv[j]) * sl2);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            float alpha = 1.f;
            bool rescale = false;
            if (mx > m_used + kRescale || m_used == -INFINITY) {
                const float m_new = fmaxf(mx, m_used);
                alpha = (m_used == -INFINITY) ? 0.f : exp2f(m_used - m_new);
                rescale = (c > 0);
                m_used = m_new;
            }
            // p = exp2(scale*log2e*s - m) in bf16 for P.V.  FP8 rows: two bf16 parts, p ~ hi +
            // lo (relative error about 2^-17; a single bf16 P costs 2^-9 per weight, which the
            // heavy-tailed values of that format turn into output errors near 2e-2 of the output
            // RMS).  bf16 rows: the single part hi, and l sums the same rounded weights.  hi goes
            // into the chunk's RoPE column block (dead once Q.K^T has read it), lo into the one
            // P_lo block; both are K-major SW128 rows of 128 B per head.
            uint8_t* pblk = stage_s + st * kStageBytes + 8 * kBlk;
            float psum = 0.f;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t pk[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int j = ch * 8 + 2 * q;
                    const float p0 = (cbase + j < nvalid) ? exp2f(__uint_as_float(sv[j]) * sl2 - m_used) : 0.f;
                    const float p1 = (cbase + j + 1 < nvalid) ? exp2f(__uint_as_float(sv[j + 1]) * sl2 - m_used) : 0.f;
                    pk[q] = pack_bf16x2(p0, p1);
                    const float h0 = bf16_bits_to_f32((uint16_t)(pk[q] & 0xFFFF));
                    const float h1 = bf16_bits_to_f32((uint16_t)(pk[q] >> 16));
                    if constexpr (FP8) {
                        sv[j] = __float_as_uint(p0 - h0);      // exact residuals
                        sv[j + 1] = __float_as_uint(p1 - h1);
                        psum += p0 + p1;
                    } else {
                        psum += h0 + h1;
                    }
                }
                *reinterpret_cast<uint4*>(pblk + sw128_off(head, (cbase >> 3) + ch)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
            // The previous chunk's P.V must be complete before P_lo (single-buffered) or O is
            // written: for FP8 rows every chunk, for bf16 rows only when O is rescaled.  (P.V of
            // chunk c-3 is complete here -- chunk c-1 was gathered after it -- so the
            // per-chunk-parity barrier cannot be two phases behind.)
            const bool any_rescale = __any_sync(0xffffffffu, rescale);
            if (c > 0 && (FP8 || any_rescale)) {
                if (!mbar_wait(&bars.ofull[(c - 1) & 1], (uint32_t)(((c - 1) >> 1) & 1), status, 321)) break;
                tc_fence_after();
            }
            if constexpr (FP8) {
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    uint32_t pk[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int j = ch * 8 + 2 * q;
                        pk[q] = pack_bf16x2(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1]));
                    }
                    *reinterpret_cast<uint4*>(plo_s + sw128_off(head, (cbase >> 3) + ch)) =
                        make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
            psum += __shfl_xor_sync(0xffffffffu, psum, 16);
            l_sum = l_sum * alpha + psum;
            if (any_rescale) {
                // O is stable (the previous chunk's P.V is complete, waited for above).
                const float f = rescale ? alpha : 1.f;
                for (int j = 0; j < 256 / 16; ++j) {
                    uint32_t ov[16];
                    const uint32_t ta = tmem_addr(tmem, quarter * 32, j * 16);
                    tmem_ld16(ta, ov);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 16; ++q) ov[q] = __float_as_uint(__uint_as_float(ov[q]) * f);
                    tmem_st16(ta, ov);
                }
                tmem_st_wait();
                tc_fence_before();
            }
            fence_proxy_async_smem();
            mbar_arrive(&bars.pfull[st]);
        }
        // ---- epilogue: O (normalised when this is the only split; else the partial O and
        // (m, l) for the split combine) staged through shared memory, coalesced global
        // writes.  Lane l of warp q holds the O row of head 16q + (l & 15), dims 0-255
        // (lanes 0-15) or 256-511 (lanes 16-31).
        if (nch > 0) mbar_wait(&bars.odone, 0, status, 322);
        tc_fence_after();
        const bool final_out = splits == 1;
        const float fs = final_out ? ((l_sum > 0.f) ? 1.f / l_sum : 0.f) : 1.f;
        const int dim0 = (lane < 16) ? 0 : 256;
        const bool f32 = !final_out || a.out_dtype == LCS_F32;
        const int row_pitch = f32 ? kOPitchF32 : kOPitchBF16;   // padded rows: fewer bank conflicts
        uint8_t* ostage = stage_s;                               // stages are free after the last P.V
        uint8_t* rowp = ostage + head * row_pitch;
        for (int j0 = 0; j0 < 256 / 16; j0 += 4) {
            uint32_t ov[4][16];
            if (nch > 0) {
#pragma unroll
                for (int u = 0; u < 4; ++u) tmem_ld16(tmem_addr(tmem, quarter * 32, (j0 + u) * 16), ov[u]);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int q = 0; q < 16; ++q) ov[u][q] = 0;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = j0 + u;
                if (f32) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        reinterpret_cast<float4*>(rowp + (dim0 + j * 16) * 4)[q] =
                            make_float4(__uint_as_float(ov[u][4 * q]) * fs, __uint_as_float(ov[u][4 * q + 1]) * fs,
                                        __uint_as_float(ov[u][4 * q + 2]) * fs, __uint_as_float(ov[u][4 * q + 3]) * fs);
                } else {
                    uint32_t pk[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        pk[q] = pack_bf16x2(__uint_as_float(ov[u][2 * q]) * fs, __uint_as_float(ov[u][2 * q + 1]) * fs);
                    reinterpret_cast<uint4*>(rowp + (dim0 + j * 16) * 2)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    reinterpret_cast<uint4*>(rowp + (dim0 + j * 16) * 2)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
        }
        if (lane < 16) {
            if (final_out) {
                if (a.lse != nullptr)
                    a.lse[g * kH + head] = (l_sum > 0.f) ? (m_used + log2f(l_sum)) / kLog2e : -INFINITY;
            } else {
                float* ml = cmerge ? ml_s + 2 * head : part_ml + ((g * splits + sp) * kH + head) * 2;
                ml[0] = (l_sum > 0.f) ? m_used : -INFINITY;
                ml[1] = l_sum;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (cmerge) {
        // ---- split merge inside the query's cluster: split sp (= cluster rank) merges the
        // heads sp, sp + splits, ... from every split's staged fp32 O and (m, l), read over
        // distributed shared memory, weights exp2(m_s - M) / L summed in split order.
        cluster_sync_all();   // every split has staged its partial
        constexpr int kW = kMaxSplits + 2;
        float* wt = ml_s + 2 * kH;   // [heads of this split][f_0 .. f_{splits-1}, 1/L]
        const int nh = (kH - sp + splits - 1) / splits;
        if ((int)threadIdx.x < nh) {
            const int h = sp + (int)threadIdx.x * splits;
            float M = -INFINITY;
            for (int r = 0; r < splits; ++r) {
                const float m = ld_dsmem_f32(dsmem_addr(ml_s + 2 * h, (uint32_t)r));
                const float l = ld_dsmem_f32(dsmem_addr(ml_s + 2 * h + 1, (uint32_t)r));
                if (l > 0.f) M = fmaxf(M, m);
            }
            float L = 0.f;
            for (int r = 0; r < splits; ++r) {
                const float m = ld_dsmem_f32(dsmem_addr(ml_s + 2 * h, (uint32_t)r));
                const float l = ld_dsmem_f32(dsmem_addr(ml_s + 2 * h + 1, (uint32_t)r));
                const float f = l > 0.f ? exp2f(m - M) : 0.f;
                wt[threadIdx.x * kW + r] = f;
                L += l * f;
            }
            wt[threadIdx.x * kW + kMaxSplits] = L > 0.f ? 1.f / L : 0.f;
            if (a.lse != nullptr) a.lse[g * kH + h] = L > 0.f ? (M + log2f(L)) / kLog2e : -INFINITY;
        }
        __syncthreads();
        for (int it = (int)threadIdx.x; it < nh * (kDv / 4); it += kAtThreads) {
            const int i = it / (kDv / 4), q4 = it - i * (kDv / 4);
            const int h = sp + i * splits;
            const float* rw = wt + i * kW;
            const uint8_t* src = stage_s + h * kOPitchF32 + q4 * 16;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int r = 0; r < splits; ++r) {
                const float4 v = ld_dsmem_f4(dsmem_addr(src, (uint32_t)r));
                const float f = rw[r];
                acc.x += v.x * f;
                acc.y += v.y * f;
                acc.z += v.z * f;
                acc.w += v.w * f;
            }
            const float iv = rw[kMaxSplits];
            const int64_t o4 = (g * kH + h) * (kDv / 4) + q4;
            if (a.out_dtype == LCS_F32)
                reinterpret_cast<float4*>(a.out)[o4] = make_float4(acc.x * iv, acc.y * iv, acc.z * iv, acc.w * iv);
            else
                reinterpret_cast<uint2*>(a.out)[o4] =
                    make_uint2(pack_bf16x2(acc.x * iv, acc.y * iv), pack_bf16x2(acc.z * iv, acc.w * iv));
        }
        cluster_sync_all();   // no CTA leaves while a peer still reads its staged partial
    } else {
        // the staged O rows (normalised output, or this split's fp32 partial) go out with
        // coalesced 16-byte stores from every thread of the CTA
        const bool f32 = splits > 1 || a.out_dtype == LCS_F32;
        const int row_pitch = f32 ? kOPitchF32 : kOPitchBF16;
        const int row_bytes_out = f32 ? kDv * 4 : kDv * 2;
        uint8_t* gout = splits == 1 ? static_cast<uint8_t*>(a.out) + g * kH * row_bytes_out
                                    : reinterpret_cast<uint8_t*>(part_o + (g * splits + sp) * kH * kDv);
        for (int off = (int)threadIdx.x * 16; off < kH * row_bytes_out; off += kAtThreads * 16) {
            const int h = off / row_bytes_out, cb = off - h * row_bytes_out;
            *reinterpret_cast<uint4*>(gout + off) = *reinterpret_cast<const uint4*>(stage_s + h * row_pitch + cb);
        }
    }
#if defined(__CUDA_ARCH__)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");   // the split combine
#endif
    if (warp == kWarpQK) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Merges the split partials of one (query, head) per CTA: 128 threads, one float4 of the
// 512 output dims each.  The split weights exp2(m_s - M) and 1/L are formed once; every
// split's float4 is loaded before any is used; the sum runs in split order.
__global__ void __launch_bounds__(128) attend_combine_kernel(const float* __restrict__ part_o,
                                                             const float* __restrict__ part_ml, int splits,
                                                             void* __restrict__ out, int out_dtype,
                                                             float* __restrict__ lse) {
    __shared__ float fac[kMaxSplits];
    __shared__ float inv_l;
    const int64_t gh = blockIdx.x;   // query * 64 + head
    const int64_t g = gh / kH;
    const int h = (int)(gh - g * kH);
    const int t = threadIdx.x;
#if defined(__CUDA_ARCH__)
    asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
    if (t < 32) {
        float2 ml = make_float2(-INFINITY, 0.f);
        if (t < splits) ml = __ldcg(reinterpret_cast<const float2*>(part_ml) + (g * splits + t) * kH + h);
        float M = ml.x;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float e = (t < splits && ml.y > 0.f) ? exp2f(ml.x - M) : 0.f;
        if (t < splits) fac[t] = e;
        // L summed in split order by lane 0
        float L = 0.f;
        for (int s = 0; s < splits; ++s) L += __shfl_sync(0xffffffffu, ml.y * e, s);
        if (t == 0) {
            inv_l = L > 0.f ? 1.f / L : 0.f;
            if (lse != nullptr) lse[gh] = L > 0.f ? (M + log2f(L)) / kLog2e : -INFINITY;
        }
    }
    __syncthreads();
    const float4* src = reinterpret_cast<const float4*>(part_o) + (g * splits * kH + h) * (kDv / 4) + t;
    float4 v[kMaxSplits];
#pragma unroll
    for (int s = 0; s < kMaxSplits; ++s)
        if (s < splits) v[s] = __ldcg(src + (int64_t)s * kH * (kDv / 4));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < kMaxSplits; ++s)
        if (s < splits) {
            const float e = fac[s];
            acc.x += v[s].x * e;
            acc.y += v[s].y * e;
            acc.z += v[s].z * e;
            acc.w += v[s].w * e;
        }
    const float iv = inv_l;
    if (out_dtype == LCS_F32) {
        reinterpret_cast<float4*>(out)[gh * (kDv / 4) + t] = make_float4(acc.x * iv, acc.y * iv, acc.z * iv, acc.w * iv);
    } else {
        reinterpret_cast<uint2*>(out)[gh * (kDv / 4) + t] =
            make_uint2(pack_bf16x2(acc.x * iv, acc.y * iv), pack_bf16x2(acc.z * iv, acc.w * iv));
    }
}

// --------------------------------------------------------------- fp32 path
constexpr int kF32Chunk = 64;

__global__ void attend_f32_kernel(const AttendArgs a, int* status) {
    extern __shared__ float sh[];
    const int H = a.H, D = a.D, dv = a.d_v;
    float* qs = sh;                          // [H, D]
    float* rows = qs + H * D;                // [chunk, D]
    float* s = rows + kF32Chunk * D;         // [H, chunk]
    float* o = s + H * kF32Chunk;            // [H, dv]
    float* mh = o + H * dv;                  // [H]
    float* lh = mh + H;                      // [H]
    float* al = lh + H;                      // [H]
    int* sel = reinterpret_cast<int*>(al + H);   // [k]
    __shared__ int nsel_s;

    const int64_t g = blockIdx.x, b = g / a.Q;
    const float* qg = static_cast<const float*>(a.q) + g * H * D;
    for (int i = threadIdx.x; i < H * D; i += blockDim.x) qs[i] = qg[i];
    for (int i = threadIdx.x; i < H * dv; i += blockDim.x) o[i] = 0.f;
    for (int i = threadIdx.x; i < H; i += blockDim.x) { mh[i] = -INFINITY; lh[i] = 0.f; }
    if (threadIdx.x == 0) {
        int n = 0;
        if (a.idx != nullptr) {
            for (int i = 0; i < a.k; ++i) {
                int v = a.idx[g * a.k + i];
                if (v >= a.N_c) { set_status(status, LCS_ERR_DEVICE, 202); v = -1; }
                if (v >= 0) sel[n++] = v;
            }
        } else {
            int64_t av = a.N_c;
            if (a.q_pos != nullptr) {
                av = (a.q_pos[g] + 1) / a.m;
                av = av < 0 ? 0 : (av < a.N_c ? av : a.N_c);
            }
            n = (int)av;
        }
        nsel_s = n;
    }
    __syncthreads();
    const RowPlan plan = plan_rows(a, g, nsel_s);
    const int64_t R = plan.nsel + plan.nwin;
    const int* selp = a.idx != nullptr ? sel : nullptr;
    for (int64_t r0 = 0; r0 < R; r0 += kF32Chunk) {
        const int nr = (int)((R - r0) < kF32Chunk ? (R - r0) : kF32Chunk);
        for (int i = threadIdx.x; i < nr * D; i += blockDim.x) {
            const int rr = i / D, c = i - rr * D;
            rows[i] = reinterpret_cast<const float*>(row_ptr(a, b, plan, selp, r0 + rr, D * 4))[c];
        }
        __syncthreads();
        for (int i = threadIdx.x; i < H * nr; i += blockDim.x) {
            const int h = i / nr, rr = i - h * nr;
            float acc = 0.f;
            for (int c = 0; c < D; ++c) acc = fmaf(qs[h * D + c], rows[rr * D + c], acc);
            s[h * kF32Chunk + rr] = acc * a.scale;
        }
        __syncthreads();
        for (int h = threadIdx.x; h < H; h += blockDim.x) {
            float mx = mh[h];
            for (int rr = 0; rr < nr; ++rr) mx = fmaxf(mx, s[h * kF32Chunk + rr]);
            const float alpha = (mh[h] == -INFINITY) ? 0.f : expf(mh[h] - mx);
            float l = lh[h] * alpha;
            for (int rr = 0; rr < nr; ++rr) {
                const float p = expf(s[h * kF32Chunk + rr] - mx);
                s[h * kF32Chunk + rr] = p;
                l += p;
            }
            mh[h] = mx;
            lh[h] = l;
            al[h] = alpha;
        }
        __syncthreads();
        for (int i = threadIdx.x; i < H * dv; i += blockDim.x) {
            const int h = i / dv, c = i - h * dv;
            float acc = o[i] * al[h];
            for (int rr = 0; rr < nr; ++rr) acc = fmaf(s[h * kF32Chunk + rr], rows[rr * D + c], acc);
            o[i] = acc;
        }
        __syncthreads();
    }
    float* og = static_cast<float*>(a.out) + g * H * dv;
    for (int i = threadIdx.x; i < H * dv; i += blockDim.x) {
        const int h = i / dv;
        og[i] = lh[h] > 0.f ? o[i] / lh[h] : 0.f;
    }
    if (a.lse != nullptr)
        for (int h = threadIdx.x; h < H; h += blockDim.x)
            a.lse[g * H + h] = lh[h] > 0.f ? mh[h] + logf(lh[h]) : -INFINITY;
}

int64_t max_chunks(const AttendArgs& a) {
    const int64_t nw = (a.q_pos == nullptr ? a.Tw : (a.W < a.Tw ? a.W : a.Tw));
    return (nw + kChunk - 1) / kChunk + ((a.idx != nullptr ? a.k : a.N_c) + kChunk - 1) / kChunk;
}

// Splits per query: every CTA of the launch resident at once (queries x splits <= SMs, one
// CTA per SM), at least two chunks per split; picks the count that minimises the chunks per
// CTA plus a fixed per-CTA cost of about two chunks (prologue, pipeline fill, epilogue) and,
// with splits, one more for the combine.
int choose_splits(const AttendArgs& a) {
    const int64_t queries = a.B * a.Q;
    const int64_t chunks = max_chunks(a);
    int best = 1;
    double best_cost = (double)chunks + 2.0;
    for (int s = 2; s <= kMaxSplits; ++s) {
        if ((chunks + s - 1) / s < 2 || queries * s > num_sms()) break;
        const double cost = (double)((chunks + s - 1) / s) + 3.0;
        if (cost < best_cost) {
            best = s;
            best_cost = cost;
        }
    }
    return best;
}

// The in-cluster split merge is used when a query's splits fit one portable cluster and all
// of the launch's clusters can be resident at once (checked once per kernel and split count).
bool cluster_merge_ok(const void* kern, int splits, int64_t queries) {
    if (splits < 2 || splits > 8) return false;
    static std::mutex mu;
    static const void* kerns[2] = {nullptr, nullptr};
    static int cache[2][9];
    std::lock_guard<std::mutex> lock(mu);
    int slot = kerns[0] == kern ? 0 : kerns[1] == kern ? 1 : (kerns[0] == nullptr ? 0 : 1);
    if (kerns[slot] != kern) {
        kerns[slot] = kern;
        for (int i = 0; i < 9; ++i) cache[slot][i] = 0;
    }
    if (cache[slot][splits] == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)splits);
        cfg.blockDim = dim3(kAtThreads);
        cfg.dynamicSmemBytes = kAtSmem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)splits;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
        cudaGetLastError();
        cache[slot][splits] = n > 0 ? n : -1;
    }
    return cache[slot][splits] >= queries;
}

}  // namespace

// Split partials: fp32 O [queries, splits, 64, 512] and (m, l) [queries, splits, 64, 2].
int64_t attend_scratch_bytes(const AttendArgs& a) {
    if (a.kv_dtype == LCS_F32) return 0;
    const int s = choose_splits(a);
    if (s == 1) return 0;
    const int64_t queries = a.B * a.Q;
    return align256(queries * s * kH * kDv * 4) + align256(queries * s * kH * 2 * 4);
}

cudaError_t launch_attend(const AttendArgs& a, void* scratch, int* status, cudaStream_t s, bool pdl) {
    const int64_t queries = a.B * a.Q;
    if (queries == 0) return cudaSuccess;
    if (a.kv_dtype == LCS_F32) {
        const size_t smem = sizeof(float) * (a.H * a.D + kF32Chunk * a.D + a.H * kF32Chunk + a.H * a.d_v + 3 * a.H) +
                            sizeof(int) * (a.k > 0 ? a.k : 1);
        cudaError_t e = set_smem_once(reinterpret_cast<const void*>(attend_f32_kernel), smem);
        if (e != cudaSuccess) return e;
        return launch_k(attend_f32_kernel, dim3((unsigned)queries), dim3(256), smem, s, pdl, a, status);
    }
    CUtensorMap mq, mc, mw, mcr, mwr;
    if (!encode_tmap_2d(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.q, kD, (uint64_t)(queries * kH), kD * 2, 64, kH,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (a.kv_dtype == LCS_BF16) {
        // contiguous-row maps: boxes of 64 rows x 64 columns (128 B), 128-byte swizzle;
        // row coordinates are int32
        if (a.B * a.N_c >= (int64_t(1) << 31) || a.B * a.Tw >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
        if (!encode_tmap_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.comp, kD, (uint64_t)(a.B * a.N_c), kD * 2, 64,
                            kChunk, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        if (a.Tw > 0) {
            if (!encode_tmap_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.win, kD, (uint64_t)(a.B * a.Tw), kD * 2, 64,
                                kChunk, CU_TENSOR_MAP_SWIZZLE_128B))
                return cudaErrorInvalidValue;
        } else {
            mw = mc;
        }
        mcr = mc;   // unused by the bf16 kernel
        mwr = mc;
    } else {
        // FP8 rows (656 B) as bytes: the 512 codes in boxes of 64 rows x 64 B (no swizzle),
        // the RoPE dims (bf16, bytes 512-639) in boxes of 64 rows x 128 B (128-byte swizzle)
        if (a.B * a.N_c >= (int64_t(1) << 31) || a.B * a.Tw >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
        if (!encode_tmap_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.comp, 656, (uint64_t)(a.B * a.N_c), 656, 64,
                            kChunk, CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !encode_tmap_2d(&mcr, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.comp, 656, (uint64_t)(a.B * a.N_c), 656, 128,
                            kChunk, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        if (a.Tw > 0) {
            if (!encode_tmap_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.win, 656, (uint64_t)(a.B * a.Tw), 656, 64,
                                kChunk, CU_TENSOR_MAP_SWIZZLE_NONE) ||
                !encode_tmap_2d(&mwr, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.win, 656, (uint64_t)(a.B * a.Tw), 656, 128,
                                kChunk, CU_TENSOR_MAP_SWIZZLE_128B))
                return cudaErrorInvalidValue;
        } else {
            mw = mc;
            mwr = mcr;
        }
    }
    auto kern = (a.kv_dtype == LCS_KV_FP8) ? attend_tc_kernel<true> : attend_tc_kernel<false>;
    cudaError_t e = set_smem_once(reinterpret_cast<const void*>(kern), kAtSmem);
    if (e != cudaSuccess) return e;
    const int splits = choose_splits(a);
    float* part_o = nullptr;
    float* part_ml = nullptr;
    if (splits > 1) {
        part_o = static_cast<float*>(scratch);
        part_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + align256(queries * splits * kH * kDv * 4));
    }
    const int cmerge = cluster_merge_ok(reinterpret_cast<const void*>(kern), splits, queries) ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(queries * splits));
    cfg.blockDim = dim3(kAtThreads);
    cfg.dynamicSmemBytes = kAtSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (cmerge) {   // a query's splits form one cluster and merge their partials in shared memory
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)splits;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    e = cudaLaunchKernelEx(&cfg, kern, mq, mc, mw, mcr, mwr, a, splits, cmerge, part_o, part_ml, status);
    if (e != cudaSuccess || splits == 1 || cmerge) return e;
    return launch_k(attend_combine_kernel, dim3((unsigned)(queries * kH)), dim3(128), 0, s, true, part_o, part_ml,
                    splits, a.out, a.out_dtype, a.lse);
}

}  // namespace lcs
