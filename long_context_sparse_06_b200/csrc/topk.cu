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
// One CTA of 1024 threads per query row:
//  1. Sample: a fixed strided sample of the row is bitonic-sorted in shared
//     memory; its element of rank r (r chosen well below the sample's expected
//     count above the true threshold) is a lower bound T for the k-th score.
//  2. Filter: the row is read once; each warp walks its own contiguous segment
//     and appends the composites with key >= T to its private candidate buffer,
//     slots from __ballot_sync / __popc (no atomics, no contention).
//  3. The candidates (typically ~2.5 k) are compacted and bitonic-sorted; the
//     first k are the selection; their indices are bitonic-sorted ascending.
// Rows no longer than the candidate capacity skip step 1.  If the bound misses
// (fewer than k candidates, or a buffer overflows) the row falls back to an
// exact MSB-first radix select (8-bit digits, shared-memory histograms) followed
// by an ordered ballot compaction.  Every step is deterministic.
#include <utility>

#include "lcs_common.cuh"
#include "lcs_internal.h"

namespace lcs {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kCandCap = 8192;                 // total candidate capacity
constexpr int kWarpCap = kCandCap / kWarps;    // per-warp candidate buffer
constexpr int kSampleMax = 4096;

struct TopkSmem {
    unsigned long long cand[kCandCap];      // per-warp candidate buffers, then the compacted sort array
    unsigned long long sorted[kCandCap];    // compacted candidates (bitonic-sorted)
    uint32_t sample[kSampleMax];            // sample keys; later the k selected indices
    uint32_t hist[256], scan[256];
    uint32_t warp_cnt[kWarps], warp_off[kWarps];
    uint32_t digit, krem, total, fail;
};

template <bool BF16>
__device__ __forceinline__ uint32_t load_key(const void* row, int64_t i) {
    if constexpr (BF16) return bf16_key(static_cast<const uint16_t*>(row)[i]);
    else return f32_key(static_cast<const float*>(row)[i]);
}

// Bitonic sort of n (power of two) elements in shared memory, descending when
// desc, by the whole block.
template <typename T>
__device__ void bitonic_sort(T* a, int n, bool desc) {
    for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = threadIdx.x; t < (n >> 1); t += blockDim.x) {
                const int i = 2 * t - (t & (stride - 1));
                const int j = i + stride;
                const bool up = ((i & size) == 0) == desc;   // this pair's block is ordered "desc" when up
                const T x = a[i], y = a[j];
                if ((x < y) == up) { a[i] = y; a[j] = x; }
            }
            __syncthreads();
        }
    }
}

__device__ __forceinline__ int next_pow2(int x) {
    int p = 1;
    while (p < x) p <<= 1;
    return p;
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

    // ---- 1. lower bound from a sorted strided sample
    uint32_t T = 0;
    if (n > kCandCap) {
        const int S = n <= 65536 ? 2048 : kSampleMax;
        for (int i = t; i < S; i += kThreads) sm.sample[i] = load_key<BF16>(srow, (int64_t)i * n / S);
        __syncthreads();
        bitonic_sort(sm.sample, S, true);
        int r = (int)((3 * (int64_t)k * S) / (2 * n)) + 8;   // 1.5x the expected rank of the k-th score, + 8
        if (r > S - 1) r = S - 1;
        T = sm.sample[r];
    }

    // ---- 2. filter into per-warp buffers (warp w owns a contiguous segment)
    const int64_t seg = ((n + kWarps - 1) / kWarps + 31) / 32 * 32;
    const int64_t s0 = warp * seg, s1 = (s0 + seg < n) ? s0 + seg : n;
    unsigned long long* wbuf = sm.cand + warp * kWarpCap;
    uint32_t cnt = 0;
    const uint32_t lt = (1u << lane) - 1u;
    for (int64_t base = s0; base < s1; base += 32) {
        const int64_t i = base + lane;
        const bool act = i < s1;
        const uint32_t key = act ? load_key<BF16>(srow, i) : 0u;
        const bool keep = act && key >= T;
        const uint32_t mk = __ballot_sync(0xffffffffu, keep);
        const uint32_t slot = cnt + __popc(mk & lt);
        if (keep && slot < kWarpCap)
            wbuf[slot] = ((unsigned long long)key << 32) | (unsigned long long)(~(uint32_t)i);
        cnt += __popc(mk);
    }
    if (lane == 0) sm.warp_cnt[warp] = cnt;
    __syncthreads();
    if (t == 0) {
        uint32_t off = 0, fail = 0;
        for (int w = 0; w < kWarps; ++w) {
            sm.warp_off[w] = off;
            off += sm.warp_cnt[w];
            fail |= sm.warp_cnt[w] > (uint32_t)kWarpCap;
        }
        sm.total = off;
        sm.fail = fail || off < (uint32_t)k;
    }
    __syncthreads();
    if (sm.fail) {
        radix_select<BF16>(sm, srow, n, k, out);
        return;
    }

    // ---- 3. compact, sort descending, take k, sort their indices ascending
    const int C = (int)sm.total;
    const int P = next_pow2(C);
    for (int w = warp; w < kWarps; w += kWarps) {
        const uint32_t c = sm.warp_cnt[w], o = sm.warp_off[w];
        for (uint32_t j = lane; j < c; j += 32) sm.sorted[o + j] = sm.cand[w * kWarpCap + j];
    }
    for (int i = C + t; i < P; i += kThreads) sm.sorted[i] = 0ull;
    __syncthreads();
    bitonic_sort(sm.sorted, P, true);
    const int Pk = next_pow2(k);
    for (int i = t; i < Pk; i += kThreads) sm.sample[i] = (i < k) ? ~(uint32_t)(sm.sorted[i] & 0xFFFFFFFFull) : 0xFFFFFFFFu;
    __syncthreads();
    bitonic_sort(sm.sample, Pk, false);
    for (int i = t; i < k; i += kThreads) out[i] = (int32_t)sm.sample[i];
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
