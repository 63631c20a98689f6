// topk.cu -- per-query top-k selection over index scores.
//
// "DeepSeek V4 深度解析" §2, CSA step 2: each query keeps the top-k compressed
// entries (1024 for Pro, 512 for Flash); "V3 vs V4" page, "FP4 为什么能无损":
// index scores in BF16 make this selection cheaper.
//
// Selection = the k largest scores of the row (ties -> lower index), returned in
// ascending index order, padded with -1 when the row has fewer than k entries.
// Scores are compared through order-preserving unsigned keys (-0 == +0), and an
// element is ranked by the 64-bit composite (key << 32 | ~index), so "larger
// composite" is exactly "larger score, then lower index".
//
// One CTA of 512 threads per query row:
//  1. Lower bound: a fixed strided sample of 512 keys is histogrammed over the
//     top 14 key bits (sign, exponent, top mantissa bits); the lower edge of the
//     bin holding the sample's rank-r element, r about 1.5 k x sample/row + 8,
//     bounds the k-th score from below with overwhelming probability.
//  2. One pass over the row: each lane loads 32 consecutive keys with 16-byte
//     vector loads and appends those >= the bound to its warp's buffer; slots
//     come from per-lane counts and a warp scan, so candidates stay in index
//     order.
//  3. The candidates (about 1.5 k) are histogrammed on the same 14 bits; a
//     suffix scan finds the bin holding the k-th largest; that bin's members are
//     ranked exactly by counting on the composite key; an ordered compaction over
//     the candidate list (warp slices, __ballot_sync / __popc for the slots) writes
//     the ascending selection.
// Shared-memory atomics: ~1024 + ~1.5 k per row instead of one per entry.  If
// the bound misses (fewer than k candidates, a full buffer, a crowded bin) the
// row falls back to an exact MSB-first radix select (8-bit digits) followed by
// an ordered ballot compaction.  Nothing depends on the order of the atomics,
// so every step is deterministic.
#include <utility>

#include "lcs_common.cuh"
#include "lcs_internal.h"

namespace lcs {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBinBits = 14;
constexpr int kBins = 1 << kBinBits;
constexpr int kCandCap = 2048;                 // threshold-bin elements ranked by counting
constexpr int kWarpCap = 512;                  // per-warp candidate buffer
constexpr int kListCap = kWarps * kWarpCap;    // all candidates

struct TopkSmem {
    uint32_t bins[kBins + kBins / 32];          // 64 KB histogram, one pad word per 32 bins
    unsigned long long wbuf[kListCap];          // per-warp candidate buffers (64 KB)
    unsigned long long list[kListCap];          // compacted candidates, index order (64 KB)
    uint8_t take[kListCap];                     // candidate selected?
    uint16_t mpos[kCandCap];                    // list positions of the threshold bin's members
    uint32_t hist[256], scan[256];              // radix fallback
    uint32_t warp_cnt[kWarps], warp_off[kWarps], warp_gt[kWarps], warp_sel[kWarps];
    uint32_t wsum[kWarps];
    uint32_t digit, krem, tbin, above, fail, total;
};

// Histogram slot of bin b: one pad word after every 32 bins, so that threads owning
// 32 consecutive bins read different banks.
__device__ __forceinline__ uint32_t hb(uint32_t b) { return b + (b >> 5); }

template <bool BF16>
__device__ __forceinline__ uint32_t load_key(const void* row, int64_t i) {
    if constexpr (BF16) return bf16_key(static_cast<const uint16_t*>(row)[i]);
    else return f32_key(static_cast<const float*>(row)[i]);
}

// ---------------------------------------------------------- exact fallback
__device__ void pick_digit(TopkSmem& sm) {
    const int t = threadIdx.x;
    if (t < 256) sm.scan[t] = sm.hist[255 - t];
    __syncthreads();
    for (int off = 1; off < 256; off <<= 1) {
        uint32_t v = 0;
        if (t < 256 && t >= off) v = sm.scan[t - off];
        __syncthreads();
        if (t < 256) sm.scan[t] += v;
        __syncthreads();
    }
    const uint32_t krem = sm.krem;
    if (t < 256) {
        const uint32_t incl = sm.scan[t], excl = (t == 0) ? 0u : sm.scan[t - 1];
        if (excl < krem && incl >= krem) { sm.digit = 255u - t; sm.krem = krem - excl; }
    }
    __syncthreads();
}

template <bool BF16>
__device__ void radix_select(TopkSmem& sm, const void* srow, int64_t n, int k, int32_t* out) {
    constexpr int kBits = BF16 ? 16 : 32;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    if (t == 0) sm.krem = (uint32_t)k;
    uint32_t prefix = 0;
    for (int p = 0; p < kBits / 8; ++p) {
        const int shift = kBits - 8 * (p + 1);
        if (t < 256) sm.hist[t] = 0;
        __syncthreads();
        for (int64_t i = t; i < n; i += kThreads) {
            const uint32_t key = load_key<BF16>(srow, i);
            if (p == 0 || (key >> (shift + 8)) == prefix) atomicAdd(&sm.hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        pick_digit(sm);
        prefix = (prefix << 8) | sm.digit;
    }
    const uint32_t thr = prefix, take_eq = sm.krem;
    // ordered compaction: warp w owns [w*seg, (w+1)*seg)
    const int64_t seg = ((n + kWarps - 1) / kWarps + 31) / 32 * 32;
    const int64_t s0 = warp * seg, s1 = (s0 + seg < n) ? s0 + seg : n;
    uint32_t cgt = 0, ceq = 0;
    for (int64_t base = s0; base < s1; base += 32) {
        const int64_t i = base + lane;
        const bool act = i < s1;
        const uint32_t key = act ? load_key<BF16>(srow, i) : 0u;
        cgt += __popc(__ballot_sync(0xffffffffu, act && key > thr));
        ceq += __popc(__ballot_sync(0xffffffffu, act && key == thr));
    }
    if (lane == 0) { sm.warp_cnt[warp] = cgt; sm.warp_off[warp] = ceq; }
    __syncthreads();
    uint32_t gt_before = 0, eq_before = 0;
    for (int w = 0; w < warp; ++w) { gt_before += sm.warp_cnt[w]; eq_before += sm.warp_off[w]; }
    uint32_t sel = gt_before + (eq_before < take_eq ? eq_before : take_eq);
    uint32_t eqr = eq_before;
    const uint32_t lt = (1u << lane) - 1u;
    for (int64_t base = s0; base < s1; base += 32) {
        const int64_t i = base + lane;
        const bool act = i < s1;
        const uint32_t key = act ? load_key<BF16>(srow, i) : 0u;
        const bool gt = act && key > thr, eq = act && key == thr;
        const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
        const bool take = gt || (eq && (eqr + __popc(eqm & lt)) < take_eq);
        const uint32_t tm = __ballot_sync(0xffffffffu, take);
        if (take) out[sel + __popc(tm & lt)] = (int32_t)i;
        sel += __popc(tm);
        eqr += __popc(eqm);
    }
}

// Exclusive prefix over the kWarps per-warp values in sm.wsum (scanned in place by
// warp 0; lanes >= kWarps carry zeros and write nothing).
static_assert(kWarps <= 32, "one warp scans the per-warp sums");
__device__ __forceinline__ void scan_warp_sums(TopkSmem& sm) {
    if (threadIdx.x < 32) {
        const uint32_t v = (threadIdx.x < kWarps) ? sm.wsum[threadIdx.x] : 0u;
        uint32_t incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
            if (threadIdx.x >= o) incl += x;
        }
        if (threadIdx.x < kWarps) sm.wsum[threadIdx.x] = incl - v;
        if (threadIdx.x == kWarps - 1) sm.total = incl;
    }
    __syncthreads();
}

// Block-wide: the bin holding the k-th largest of the histogram (bins in descending
// order of value from the top).  Sets sm.tbin and sm.above (count in higher bins).
__device__ void find_bin(TopkSmem& sm, uint32_t k) {
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    constexpr int kPer = kBins / kThreads;      // thread 0 owns the top bins
    const int hi_bin = kBins - 1 - t * kPer;
    uint32_t c[kPer];
    uint32_t local = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) { c[j] = sm.bins[hb(hi_bin - j)]; local += c[j]; }
    uint32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) sm.wsum[warp] = incl;
    __syncthreads();
    scan_warp_sums(sm);
    const uint32_t excl = sm.wsum[warp] + incl - local;
    if (excl < k && excl + local >= k) {
        uint32_t run = excl;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            if (run + c[j] >= k) { sm.tbin = hi_bin - j; sm.above = run; break; }
            run += c[j];
        }
    }
    __syncthreads();
}

// Loads the 32 consecutive keys [i0, i0+32) of lane-owned scores (clipped at n).
template <bool BF16>
__device__ __forceinline__ void load32(const char* srow, int64_t i0, int64_t n, uint32_t (&key)[32]) {
    if (i0 + 32 <= n) {
        if constexpr (BF16) {
            const uint4* p = reinterpret_cast<const uint4*>(srow + i0 * 2);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const uint4 w = __ldg(p + v);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    key[8 * v + 2 * q] = bf16_key((uint16_t)(ww[q] & 0xFFFF));
                    key[8 * v + 2 * q + 1] = bf16_key((uint16_t)(ww[q] >> 16));
                }
            }
        } else {
            const float4* p = reinterpret_cast<const float4*>(srow + i0 * 4);
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const float4 f = __ldg(p + v);
                key[4 * v] = f32_key(f.x);
                key[4 * v + 1] = f32_key(f.y);
                key[4 * v + 2] = f32_key(f.z);
                key[4 * v + 3] = f32_key(f.w);
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) key[j] = (i0 + j < n) ? load_key<BF16>(srow, i0 + j) : 0u;
    }
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads, 1) topk_kernel(const void* __restrict__ scores, int64_t N_c,
                                                           const int64_t* __restrict__ q_pos, int m, int k,
                                                           int32_t* __restrict__ idx_out) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TopkSmem& sm = *reinterpret_cast<TopkSmem*>(smem_raw);
    constexpr int kShift = (BF16 ? 16 : 32) - kBinBits;
    const int64_t row = blockIdx.x;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    int64_t n = N_c;
    if (q_pos != nullptr) {
        const int64_t a = (q_pos[row] + 1) / m;
        n = a < N_c ? (a < 0 ? 0 : a) : N_c;
    }
    int32_t* out = idx_out + row * k;
    const char* srow = static_cast<const char*>(scores) + row * N_c * (BF16 ? 2 : 4);

#if defined(__CUDA_ARCH__)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // The dependent kernel (attention) may start its prologue now: it reads this kernel's
    // output only after its own griddepcontrol.wait, which waits for this grid to finish.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif

    if (n <= k) {
        for (int i = t; i < k; i += kThreads) out[i] = (i < n) ? i : -1;
        return;
    }

    // ---- 1. lower bound from a strided sample of one key per thread
    for (int i = t; i < kBins + kBins / 32; i += kThreads) sm.bins[i] = 0;
    __syncthreads();
    uint32_t T = 0;
    if (n > kListCap / 2) {
        atomicAdd(&sm.bins[hb(load_key<BF16>(srow, (int64_t)(((uint64_t)t * (uint64_t)n) / kThreads)) >> kShift)], 1u);
        __syncthreads();
        uint32_t r = (uint32_t)((3 * (int64_t)k * kThreads) / (2 * n)) + 8;
        if (r > (uint32_t)kThreads) r = kThreads;
        find_bin(sm, r);
        T = sm.tbin << kShift;
        for (int i = t; i < kBins + kBins / 32; i += kThreads) sm.bins[i] = 0;
    }

    // ---- 2. one pass: lane-owned runs of 32 consecutive keys; keys >= T go to the warp's
    // buffer in index order (per-lane counts, warp scan for the lane's slot base)
    unsigned long long* wb = sm.wbuf + warp * kWarpCap;
    const int64_t per_warp = ((n + kWarps - 1) / kWarps + 1023) / 1024 * 1024;   // whole 32x32 batches
    const int64_t w0 = warp * per_warp, w1 = (w0 + per_warp < n) ? w0 + per_warp : n;
    uint32_t wcnt = 0;
    for (int64_t bb = w0; bb < w1; bb += 1024) {
        const int64_t i0 = bb + 32 * lane;
        uint32_t key[32];
        load32<BF16>(srow, i0, w1, key);
        uint32_t c = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) c += (i0 + j < w1 && key[j] >= T);
        uint32_t incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += x;
        }
        uint32_t slot = wcnt + incl - c;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (i0 + j < w1 && key[j] >= T) {
                if (slot < kWarpCap)
                    wb[slot] = ((unsigned long long)key[j] << 32) | (unsigned long long)(~(uint32_t)(i0 + j));
                ++slot;
            }
        wcnt += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) { sm.warp_cnt[warp] = wcnt; sm.wsum[warp] = wcnt; }
    __syncthreads();
    scan_warp_sums(sm);
    if (t == 0) {
        uint32_t fail = sm.total < (uint32_t)k;
        for (int w = 0; w < kWarps; ++w) fail |= sm.warp_cnt[w] > (uint32_t)kWarpCap;
        sm.fail = fail;
    }
    __syncthreads();
    if (sm.fail) {
        radix_select<BF16>(sm, srow, n, k, out);
        return;
    }
    const uint32_t C = sm.total;
    {
        const uint32_t o = sm.wsum[warp];
        for (uint32_t j = lane; j < wcnt; j += 32) sm.list[o + j] = wb[j];
    }
    __syncthreads();

    // ---- 3. exact selection among the candidates
    for (uint32_t j = t; j < C; j += kThreads) atomicAdd(&sm.bins[hb((uint32_t)(sm.list[j] >> 32) >> kShift)], 1u);
    __syncthreads();
    find_bin(sm, (uint32_t)k);
    const uint32_t tbin = sm.tbin, need = (uint32_t)k - sm.above;
    const uint32_t m_t = sm.bins[hb(tbin)];
    if (m_t > kCandCap) {
        radix_select<BF16>(sm, srow, n, k, out);
        return;
    }
    // The list is split into 32 contiguous slices, one per warp, walked in tiles of 32.
    const uint32_t slice = (C + kWarps - 1) / kWarps;
    const uint32_t l0 = warp * slice, l1 = (l0 + slice < C) ? l0 + slice : C;
    const uint32_t lt = (1u << lane) - 1u;
    // threshold-bin members: count per slice, then compact in list order
    uint32_t mc = 0;
    for (uint32_t bs = l0; bs < l1; bs += 32) {
        const uint32_t j = bs + lane;
        const bool mem = j < l1 && ((uint32_t)(sm.list[j] >> 32) >> kShift) == tbin;
        mc += __popc(__ballot_sync(0xffffffffu, mem));
    }
    if (lane == 0) sm.wsum[warp] = mc;
    __syncthreads();
    scan_warp_sums(sm);
    {
        uint32_t pos = sm.wsum[warp];
        for (uint32_t bs = l0; bs < l1; bs += 32) {
            const uint32_t j = bs + lane;
            const uint32_t bn = j < l1 ? ((uint32_t)(sm.list[j] >> 32) >> kShift) : 0u;
            const bool mem = j < l1 && bn == tbin;
            const uint32_t mm = __ballot_sync(0xffffffffu, mem);
            if (mem) sm.mpos[pos + __popc(mm & lt)] = (uint16_t)j;
            if (j < l1) sm.take[j] = bn > tbin;
            pos += __popc(mm);
        }
    }
    __syncthreads();
    // rank the members among themselves by counting (composite keys are distinct)
    for (uint32_t j = t; j < m_t; j += kThreads) {
        const unsigned long long c = sm.list[sm.mpos[j]];
        uint32_t r = 0;
        for (uint32_t i = 0; i < m_t; ++i) r += sm.list[sm.mpos[i]] > c;
        sm.take[sm.mpos[j]] = r < need;
    }
    __syncthreads();
    // ordered compaction over the candidate list (already in index order)
    uint32_t sc = 0;
    for (uint32_t bs = l0; bs < l1; bs += 32) {
        const uint32_t j = bs + lane;
        sc += __popc(__ballot_sync(0xffffffffu, j < l1 && sm.take[j]));
    }
    if (lane == 0) sm.wsum[warp] = sc;
    __syncthreads();
    scan_warp_sums(sm);
    uint32_t pos = sm.wsum[warp];
    for (uint32_t bs = l0; bs < l1; bs += 32) {
        const uint32_t j = bs + lane;
        const bool tk = j < l1 && sm.take[j];
        const uint32_t tm = __ballot_sync(0xffffffffu, tk);
        if (tk) out[pos + __popc(tm & lt)] = (int32_t)(~(uint32_t)(sm.list[j] & 0xFFFFFFFFull));
        pos += __popc(tm);
    }
}

}  // namespace

int64_t topk_scratch_bytes(int64_t rows, int64_t N_c) {
    (void)rows;
    (void)N_c;
    return 0;
}

cudaError_t launch_topk(const void* scores, int score_dtype, int64_t B, int64_t Q, int64_t N_c,
                        const int64_t* q_pos, int m, int k, int32_t* idx, void* scratch, int* status,
                        cudaStream_t s, bool pdl) {
    (void)scratch;
    (void)status;
    const int64_t rows = B * Q;
    if (rows == 0 || k == 0) return cudaSuccess;
    const size_t smem = sizeof(TopkSmem);
    if (score_dtype == LCS_BF16) {
        cudaError_t e = set_smem_once(reinterpret_cast<const void*>(topk_kernel<true>), smem);
        if (e != cudaSuccess) return e;
        return launch_k(topk_kernel<true>, dim3((unsigned)rows), dim3(kThreads), smem, s, pdl, scores, N_c, q_pos, m,
                        k, idx);
    }
    cudaError_t e = set_smem_once(reinterpret_cast<const void*>(topk_kernel<false>), smem);
    if (e != cudaSuccess) return e;
    return launch_k(topk_kernel<false>, dim3((unsigned)rows), dim3(kThreads), smem, s, pdl, scores, N_c, q_pos, m, k,
                    idx);
}

}  // namespace lcs
