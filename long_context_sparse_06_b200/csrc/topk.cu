// topk.cu -- per-query top-k selection over index scores.
//
// "DeepSeek V4 深度解析" §2, CSA step 2: each query keeps the top-k compressed
// entries (1024 for Pro, 512 for Flash); "V3 vs V4" page, "FP4 为什么能无损":
// index scores in BF16 make this selection cheaper.
//
// Selection = the k largest scores of the row (ties -> lower index), returned in
// ascending index order, padded with -1 when the row has fewer than k entries.
//
// Method: MSB-first radix select on order-preserving unsigned keys (8-bit
// digits: 4 passes for fp32 scores, 2 for bf16), then one ordered compaction.
//  * Each pass builds a 256-bin histogram in shared memory; lanes holding the
//    same digit are merged with __match_any_sync so each distinct digit costs one
//    shared atomic per warp.
//  * After the first pass the elements that still tie with the threshold prefix
//    are gathered into a shared candidate list, so later passes scan only them.
//  * The final pass walks the row in index order: 32 warps own contiguous
//    segments; within a segment each 32-element tile decides with warp ballots
//    (__ballot_sync + __popc of the lower lanes) which elements are taken and at
//    which output slot, so the output is sorted without a sort.
// The threshold key and tie count do not depend on the order of the atomics, so
// the result is deterministic.
#include <utility>

#include "lcs_common.cuh"
#include "lcs_internal.h"

namespace lcs {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kCandCap = 8192;          // candidates kept after the first pass
constexpr int kSmemKeyCap = 40960;      // rows up to this length are cached in shared memory

struct TopkSmem {
    uint32_t hist[256];
    uint32_t warp_gt[kWarps], warp_eq[kWarps];
    uint32_t ncand;
    uint32_t digit, krem;
    uint32_t cand_key[kCandCap];
};

template <bool BF16>
__device__ __forceinline__ uint32_t load_key(const void* row, int64_t i) {
    if constexpr (BF16) return bf16_key(static_cast<const uint16_t*>(row)[i]);
    else return f32_key(static_cast<const float*>(row)[i]);
}

// Histogram of digit (key >> shift) & 255 over keys whose bits above the digit
// equal `prefix`; merged per warp with match_any.
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t key, bool active, int shift, uint32_t prefix,
                                         int hi_shift) {
    const bool match = active && (hi_shift >= 32 ? true : ((key >> hi_shift) == prefix));
    const uint32_t digit = match ? ((key >> shift) & 255u) : 256u;
    const uint32_t peers = __match_any_sync(0xffffffffu, digit);
    const int lane = threadIdx.x & 31;
    if (match && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], (uint32_t)__popc(peers));
}

// Picks the digit bin holding the krem-th largest remaining key.  Called by all
// threads; thread d < 256 owns bin d.  Updates sm.digit and sm.krem.
__device__ __forceinline__ void pick_digit(TopkSmem& sm, uint32_t* scan) {
    const int t = threadIdx.x;
    // suffix sums from the top bin down: scan[d] = sum_{e >= d} hist[e]
    if (t < 256) scan[t] = sm.hist[255 - t];
    __syncthreads();
    for (int off = 1; off < 256; off <<= 1) {
        uint32_t v = 0;
        if (t < 256 && t >= off) v = scan[t - off];
        __syncthreads();
        if (t < 256) scan[t] += v;
        __syncthreads();
    }
    // scan[i] = count of keys in bins >= 255 - i (inclusive)
    const uint32_t krem = sm.krem;
    if (t < 256) {
        const uint32_t incl = scan[t];
        const uint32_t excl = (t == 0) ? 0u : scan[t - 1];
        if (excl < krem && incl >= krem) {
            sm.digit = 255u - t;
            sm.krem = krem - excl;
        }
    }
    __syncthreads();
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads, 1) topk_kernel(const void* __restrict__ scores, int64_t Q, int64_t N_c,
                                                        const int64_t* __restrict__ q_pos, int m, int k,
                                                        int32_t* __restrict__ idx_out) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TopkSmem& sm = *reinterpret_cast<TopkSmem*>(smem_raw);
    uint32_t* scan = reinterpret_cast<uint32_t*>(smem_raw + sizeof(TopkSmem));
    uint32_t* keys = scan + 256;   // cached keys when the row fits

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

    const bool cached = n <= kSmemKeyCap;
    constexpr int kBits = BF16 ? 16 : 32;
    constexpr int kPasses = kBits / 8;

    if (t < 256) sm.hist[t] = 0;
    if (t == 0) { sm.krem = (uint32_t)k; sm.ncand = 0; }
    __syncthreads();

    // ---- pass 1: top digit over every element (and cache the keys)
    const int64_t nround = (n + kThreads - 1) / kThreads * kThreads;
    for (int64_t i = t; i < nround; i += kThreads) {
        const bool act = i < n;
        const uint32_t key = act ? load_key<BF16>(srow, i) : 0u;
        if (cached && act) keys[i] = key;
        hist_add(sm.hist, key, act, kBits - 8, 0, 32);
    }
    __syncthreads();
    pick_digit(sm, scan);
    uint32_t prefix = sm.digit;

    // ---- gather the candidates that tie with the first digit
    const bool use_cand = sm.hist[sm.digit] <= (uint32_t)kCandCap;
    if (use_cand) {
        for (int64_t i = t; i < n; i += kThreads) {
            const uint32_t key = cached ? keys[i] : load_key<BF16>(srow, i);
            if ((key >> (kBits - 8)) == prefix) sm.cand_key[atomicAdd(&sm.ncand, 1u)] = key;
        }
        __syncthreads();
    }

    // ---- remaining passes
    for (int p = 1; p < kPasses; ++p) {
        const int shift = kBits - 8 * (p + 1);
        if (t < 256) sm.hist[t] = 0;
        __syncthreads();
        if (use_cand) {
            const int nc = (int)sm.ncand;
            const int ncr = (nc + kThreads - 1) / kThreads * kThreads;
            for (int i = t; i < ncr; i += kThreads) {
                const bool act = i < nc;
                hist_add(sm.hist, act ? sm.cand_key[i] : 0u, act, shift, prefix, shift + 8);
            }
        } else {
            for (int64_t i = t; i < nround; i += kThreads) {
                const bool act = i < n;
                const uint32_t key = act ? (cached ? keys[i] : load_key<BF16>(srow, i)) : 0u;
                hist_add(sm.hist, key, act, shift, prefix, shift + 8);
            }
        }
        __syncthreads();
        pick_digit(sm, scan);
        prefix = (prefix << 8) | sm.digit;
    }
    const uint32_t thr = prefix;          // the k-th largest key
    const uint32_t take_eq = sm.krem;     // how many keys equal to thr are taken (lowest indices)

    // ---- ordered compaction: warp w owns [w*seg, (w+1)*seg)
    const int64_t seg = ((n + kWarps - 1) / kWarps + 31) / 32 * 32;
    const int64_t s0 = warp * seg, s1 = (s0 + seg < n) ? s0 + seg : n;
    uint32_t cgt = 0, ceq = 0;
    for (int64_t base = s0; base < s1; base += 32) {
        const int64_t i = base + lane;
        const bool act = i < s1;
        const uint32_t key = act ? (cached ? keys[i] : load_key<BF16>(srow, i)) : 0u;
        cgt += __popc(__ballot_sync(0xffffffffu, act && key > thr));
        ceq += __popc(__ballot_sync(0xffffffffu, act && key == thr));
    }
    if (lane == 0) { sm.warp_gt[warp] = cgt; sm.warp_eq[warp] = ceq; }
    __syncthreads();
    uint32_t gt_before = 0, eq_before = 0;
    for (int w = 0; w < warp; ++w) { gt_before += sm.warp_gt[w]; eq_before += sm.warp_eq[w]; }
    uint32_t sel = gt_before + (eq_before < take_eq ? eq_before : take_eq);
    uint32_t eqr = eq_before;
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int64_t base = s0; base < s1; base += 32) {
        const int64_t i = base + lane;
        const bool act = i < s1;
        const uint32_t key = act ? (cached ? keys[i] : load_key<BF16>(srow, i)) : 0u;
        const bool gt = act && key > thr, eq = act && key == thr;
        const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
        const bool take = gt || (eq && (eqr + __popc(eqm & lt_mask)) < take_eq);
        const uint32_t tm = __ballot_sync(0xffffffffu, take);
        if (take) out[sel + __popc(tm & lt_mask)] = (int32_t)i;
        sel += __popc(tm);
        eqr += __popc(eqm);
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
    const int64_t cache = N_c <= kSmemKeyCap ? N_c : 0;
    const size_t smem = sizeof(TopkSmem) + 256 * sizeof(uint32_t) + cache * sizeof(uint32_t);
    if (score_dtype == LCS_BF16) {
        cudaError_t e = cudaFuncSetAttribute(topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        return launch_k(topk_kernel<true>, dim3((unsigned)rows), dim3(kThreads), smem, s, pdl, scores, Q, N_c, q_pos,
                        m, k, idx);
    }
    cudaError_t e = cudaFuncSetAttribute(topk_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_k(topk_kernel<false>, dim3((unsigned)rows), dim3(kThreads), smem, s, pdl, scores, Q, N_c, q_pos, m,
                    k, idx);
}

}  // namespace lcs
