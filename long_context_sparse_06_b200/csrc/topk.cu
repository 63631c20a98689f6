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
// One CTA of 1024 threads per query row, three coalesced passes over the row:
//  1. Histogram of the top 14 bits of every key (sign, exponent and the top
//     mantissa bits of the score) in shared memory; the bins are fine enough
//     that the 32 lanes of a warp rarely collide on one counter.  A block-wide
//     suffix scan finds the bin holding the k-th largest score: every key in a
//     higher bin is selected, and `need` more come from the threshold bin.
//  2. The threshold bin's elements are gathered in index order (each warp walks
//     its own contiguous segment; slots from __ballot_sync / __popc) and ranked
//     exactly by counting, on the composite key.
//  3. Ordered compaction: each warp re-walks its segment and writes the selected
//     indices at offsets from ballots, so the output is ascending without a sort.
// If the threshold bin is too crowded for the counting rank (massive ties) the
// row falls back to an exact MSB-first radix select (8-bit digits, shared-memory
// histograms) followed by the same kind of ordered compaction.  The result does
// not depend on the order of the shared atomics, so every step is deterministic.
#include <utility>

#include "lcs_common.cuh"
#include "lcs_internal.h"

namespace lcs {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBinBits = 14;
constexpr int kBins = 1 << kBinBits;
constexpr int kCandCap = 2048;                 // threshold-bin elements ranked by counting
constexpr int kWarpCap = 256;                  // per-warp gather buffer

struct TopkSmem {
    uint32_t bins[kBins];                       // 64 KB histogram
    unsigned long long wbuf[kWarps * kWarpCap]; // per-warp gather buffers (64 KB)
    unsigned long long cand[kCandCap];          // threshold-bin candidates in index order
    uint8_t take[kCandCap];                     // candidate selected?
    uint32_t hist[256], scan[256];              // radix fallback
    uint32_t warp_cnt[kWarps], warp_off[kWarps], warp_gt[kWarps], warp_sel[kWarps];
    uint32_t wsum[kWarps];
    uint32_t digit, krem, tbin, above, fail;
};

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

// ------------------------------------------------------------------ kernel
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
#endif

    if (n <= k) {
        for (int i = t; i < k; i += kThreads) out[i] = (i < n) ? i : -1;
        return;
    }

    // ---- 1. histogram of the top bits, then the threshold bin by a suffix scan
    for (int i = t; i < kBins; i += kThreads) sm.bins[i] = 0;
    __syncthreads();
    for (int64_t i = t; i < n; i += kThreads) atomicAdd(&sm.bins[load_key<BF16>(srow, i) >> kShift], 1u);
    __syncthreads();
    constexpr int kPer = kBins / kThreads;      // bins per thread, thread 0 owns the top ones
    const int hi_bin = kBins - 1 - t * kPer;
    uint32_t local = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) local += sm.bins[hi_bin - j];
    uint32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) sm.wsum[warp] = incl;
    __syncthreads();
    uint32_t wbase = 0;
    for (int w = 0; w < warp; ++w) wbase += sm.wsum[w];
    const uint32_t excl = wbase + incl - local;
    if (excl < (uint32_t)k && excl + local >= (uint32_t)k) {
        uint32_t run = excl;
        for (int j = 0; j < kPer; ++j) {
            const uint32_t c = sm.bins[hi_bin - j];
            if (run + c >= (uint32_t)k) { sm.tbin = hi_bin - j; sm.above = run; break; }
            run += c;
        }
    }
    __syncthreads();
    const uint32_t tbin = sm.tbin, above = sm.above, need = (uint32_t)k - above;
    const uint32_t m_t = sm.bins[tbin];          // elements in the threshold bin

    // ---- 2. gather the threshold bin in index order; count the keys above it
    const int64_t seg = ((n + kWarps - 1) / kWarps + 31) / 32 * 32;
    const int64_t s0 = warp * seg, s1 = (s0 + seg < n) ? s0 + seg : n;
    const uint32_t lt = (1u << lane) - 1u;
    unsigned long long* wb = sm.wbuf + warp * kWarpCap;
    uint32_t cnt = 0, gt = 0;
    if (m_t <= kCandCap) {
        for (int64_t base = s0; base < s1; base += 32) {
            const int64_t i = base + lane;
            const bool act = i < s1;
            const uint32_t key = act ? load_key<BF16>(srow, i) : 0u;
            const uint32_t bn = key >> kShift;
            const bool eq = act && bn == tbin;
            const uint32_t em = __ballot_sync(0xffffffffu, eq);
            const uint32_t slot = cnt + __popc(em & lt);
            if (eq && slot < kWarpCap)
                wb[slot] = ((unsigned long long)key << 32) | (unsigned long long)(~(uint32_t)i);
            cnt += __popc(em);
            gt += __popc(__ballot_sync(0xffffffffu, act && bn > tbin));
        }
    }
    if (lane == 0) { sm.warp_cnt[warp] = cnt; sm.warp_gt[warp] = gt; }
    __syncthreads();
    if (t == 0) {
        uint32_t off = 0, fail = m_t > kCandCap;
        for (int w = 0; w < kWarps; ++w) {
            sm.warp_off[w] = off;
            off += sm.warp_cnt[w];
            fail |= sm.warp_cnt[w] > (uint32_t)kWarpCap;
        }
        sm.fail = fail;
    }
    __syncthreads();
    if (sm.fail) {
        radix_select<BF16>(sm, srow, n, k, out);
        return;
    }
    for (uint32_t j = lane; j < cnt; j += 32) sm.cand[sm.warp_off[warp] + j] = wb[j];
    __syncthreads();

    // ---- rank the threshold bin by counting (composite keys are distinct)
    for (uint32_t j = t; j < m_t; j += kThreads) {
        const unsigned long long c = sm.cand[j];
        uint32_t r = 0;
        for (uint32_t i = 0; i < m_t; ++i) r += sm.cand[i] > c;
        sm.take[j] = r < need;
    }
    __syncthreads();
    {   // selected candidates per warp segment
        const uint32_t o = sm.warp_off[warp];
        uint32_t c = 0;
        for (uint32_t j = lane; j < cnt; j += 32) c += sm.take[o + j];
#pragma unroll
        for (int x = 16; x > 0; x >>= 1) c += __shfl_xor_sync(0xffffffffu, c, x);
        if (lane == 0) sm.warp_sel[warp] = c;
    }
    __syncthreads();

    // ---- 3. ordered compaction
    uint32_t pos = 0;
    for (int w = 0; w < warp; ++w) pos += sm.warp_gt[w] + sm.warp_sel[w];
    uint32_t ci = sm.warp_off[warp];
    for (int64_t base = s0; base < s1; base += 32) {
        const int64_t i = base + lane;
        const bool act = i < s1;
        const uint32_t key = act ? load_key<BF16>(srow, i) : 0u;
        const uint32_t bn = key >> kShift;
        const bool eq = act && bn == tbin;
        const uint32_t em = __ballot_sync(0xffffffffu, eq);
        const bool tk = (act && bn > tbin) || (eq && sm.take[ci + __popc(em & lt)]);
        const uint32_t tm = __ballot_sync(0xffffffffu, tk);
        if (tk) out[pos + __popc(tm & lt)] = (int32_t)i;
        pos += __popc(tm);
        ci += __popc(em);
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
        cudaError_t e = cudaFuncSetAttribute(topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        return launch_k(topk_kernel<true>, dim3((unsigned)rows), dim3(kThreads), smem, s, pdl, scores, N_c, q_pos, m,
                        k, idx);
    }
    cudaError_t e = cudaFuncSetAttribute(topk_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_k(topk_kernel<false>, dim3((unsigned)rows), dim3(kThreads), smem, s, pdl, scores, N_c, q_pos, m, k,
                    idx);
}

}  // namespace lcs
