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
// Few rows of at most 65536 entries (decode over 128K tokens, the tiny prefill): a cluster
// of up to 8 CTAs per row with the whole row in registers and an exact radix select
// (topk_row_kernel, below).  Longer rows: one CTA of 256 threads per query row, two CTAs
// per SM, or a cluster of 512-thread CTAs per row when there are few rows:
//  1. Lower bound: a fixed strided sample of 512 keys is histogrammed over the
//     top 13 (256 threads) or 14 (512 threads) key bits (sign, exponent, top
//     mantissa bits); the lower edge of the
//     bin holding the sample's rank-r element, r about 1.5 k x sample/row + 8,
//     bounds the k-th score from below with overwhelming probability.
//  2. One pass over the row: each lane loads 32 consecutive keys with 16-byte
//     vector loads and appends those >= the bound to its warp's buffer; slots
//     come from per-lane counts and a warp scan, so candidates stay in index
//     order.
//  3. The candidates (about 1.5 k) are histogrammed on the same bits; a
//     suffix scan finds the bin holding the k-th largest; that bin's members are
//     ranked exactly by counting on the composite key; an ordered compaction over
//     the candidate list (warp slices, __ballot_sync / __popc for the slots) writes
//     the ascending selection.
// Shared-memory atomics: ~1024 + ~1.5 k per row instead of one per entry.  If
// the bound misses (fewer than k candidates, a full buffer, a crowded bin) the
// row falls back to an exact MSB-first radix select (8-bit digits) followed by
// an ordered ballot compaction.  Nothing depends on the order of the atomics,
// so every step is deterministic.
#include <mutex>
#include <utility>

#include "lcs_common.cuh"
#include "lcs_internal.h"

namespace lcs {

namespace {

// Block shapes of topk_kernel: 512 threads when a row is split over a cluster (few long
// rows), 256 threads when each row has a CTA of its own (many rows: prefill), two CTAs per
// SM, so that one row's passes run while the other's wait at block barriers.
template <int NT>
struct TkCfg {
    static constexpr int kThreads = NT;
    static constexpr int kWarps = NT / 32;
    static constexpr int kBinBits = NT >= 512 ? 14 : 13;
    static constexpr int kBins = 1 << kBinBits;
    static constexpr int kWarpCap = 512;                   // per-warp candidate buffer
    static constexpr int kListCap = kWarps * kWarpCap;     // all candidates
    static_assert(kWarps <= 32, "one warp scans the per-warp sums");
};
constexpr int kCandCap = 2048;    // threshold-bin elements ranked by counting
constexpr int kSamples = 512;     // keys in the sampled lower bound
constexpr int kMaxP = 16;         // CTAs per row (one cluster of 512-thread CTAs)
static_assert(kMaxP <= TkCfg<512>::kWarps, "per-rank counts reuse the per-warp arrays");

template <int NT>
struct TopkSmem {
    using C = TkCfg<NT>;
    uint32_t bins[C::kBins + C::kBins / 32];    // histogram, one pad word per 32 bins
    unsigned long long wbuf[C::kListCap];       // per-warp candidate buffers
    unsigned long long list[C::kListCap];       // compacted candidates, index order
    uint8_t take[C::kListCap];                  // candidate selected?
    uint16_t mpos[kCandCap];                    // list positions of the threshold bin's members
    uint32_t hist[256], scan[256];              // radix fallback
    uint32_t warp_cnt[C::kWarps], warp_off[C::kWarps], warp_gt[C::kWarps], warp_sel[C::kWarps];
    uint32_t wsum[C::kWarps];
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
template <int NT>
__device__ void pick_digit(TopkSmem<NT>& sm) {
    static_assert(NT >= 256, "one thread per digit");
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

template <bool BF16, int NT>
__device__ void radix_select(TopkSmem<NT>& sm, const void* srow, int64_t n, int k, int32_t* out) {
    constexpr int kBits = BF16 ? 16 : 32;
    constexpr int kThreads = NT, kWarps = NT / 32;
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
template <int NT>
__device__ __forceinline__ void scan_warp_sums(TopkSmem<NT>& sm) {
    constexpr int kWarps = NT / 32;
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
template <int NT>
__device__ void find_bin(TopkSmem<NT>& sm, uint32_t k) {
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    constexpr int kBins = TkCfg<NT>::kBins;
    constexpr int kPer = kBins / NT;            // thread 0 owns the top bins
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

// One warp batch of 1024 keys starting at bb, loaded coalesced: lane l holds the kE keys
// bb + 32*kE*v + kE*l + j (v < kV, j < kE).  A whole batch of a 16-byte aligned row is
// kV 16-byte loads per lane, all issued before any is used (raw words, converted to keys
// later, so that the next batch's loads can be in flight while this one is processed);
// a partial batch or an unaligned row uses element loads, keys at or beyond n invalid.
template <bool BF16>
struct Batch {
    static constexpr int kE = BF16 ? 8 : 4, kV = 1024 / (32 * kE);
    uint4 raw[kV];
    bool whole;
};
template <bool BF16>
__device__ __forceinline__ void issue_batch(const char* srow, bool vec_ok, int64_t bb, int64_t n, int lane,
                                            Batch<BF16>& bt) {
    constexpr int kE = Batch<BF16>::kE, kV = Batch<BF16>::kV;
    bt.whole = vec_ok && bb + 1024 <= n;
    if (bt.whole) {
        const uint4* p = reinterpret_cast<const uint4*>(srow + (bb + kE * lane) * (BF16 ? 2 : 4));
#pragma unroll
        for (int v = 0; v < kV; ++v) bt.raw[v] = __ldg(p + v * 32);
    }
}
// Keys of a batch (and the valid mask per vector slot).
template <bool BF16>
__device__ __forceinline__ void batch_keys(const char* srow, int64_t bb, int64_t n, int lane, const Batch<BF16>& bt,
                                           uint32_t (&key)[Batch<BF16>::kV][Batch<BF16>::kE],
                                           uint32_t (&valid)[Batch<BF16>::kV]) {
    constexpr int kE = Batch<BF16>::kE, kV = Batch<BF16>::kV;
    if (bt.whole) {
#pragma unroll
        for (int v = 0; v < kV; ++v) {
            valid[v] = (1u << kE) - 1u;
            const uint32_t ww[4] = {bt.raw[v].x, bt.raw[v].y, bt.raw[v].z, bt.raw[v].w};
            if constexpr (BF16) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    key[v][2 * q] = bf16_key((uint16_t)(ww[q] & 0xFFFF));
                    key[v][2 * q + 1] = bf16_key((uint16_t)(ww[q] >> 16));
                }
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) key[v][q] = f32_key(__uint_as_float(ww[q]));
            }
        }
    } else {
#pragma unroll
        for (int v = 0; v < kV; ++v) {
            const int64_t i = bb + 32 * kE * v + kE * lane;
            valid[v] = 0;
#pragma unroll
            for (int j = 0; j < kE; ++j) {
                const bool ok = i + j < n;
                key[v][j] = ok ? load_key<BF16>(srow, i + j) : 0u;
                valid[v] |= (ok ? 1u : 0u) << j;
            }
        }
    }
}

// NT = 512: one CTA per SM, P CTAs per row in a cluster.  NT = 256: P = 1, two CTAs per SM.
template <bool BF16, int NT>
__global__ void __launch_bounds__(NT, 512 / NT) topk_kernel(const void* __restrict__ scores, int64_t N_c,
                                                            const int64_t* __restrict__ q_pos, int m, int k,
                                                            int32_t* __restrict__ idx_out, int P) {
    using Cfg = TkCfg<NT>;
    constexpr int kThreads = NT, kWarps = Cfg::kWarps, kBins = Cfg::kBins;
    constexpr int kWarpCap = Cfg::kWarpCap, kListCap = Cfg::kListCap;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TopkSmem<NT>& sm = *reinterpret_cast<TopkSmem<NT>*>(smem_raw);
    constexpr int kShift = (BF16 ? 16 : 32) - Cfg::kBinBits;
    const int64_t row = blockIdx.x / P;
    const int rank = (int)(blockIdx.x - row * P);   // == rank in the row's cluster
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
#pragma unroll
        for (int j = 0; j < kSamples / kThreads; ++j) {   // sample s = t + j * kThreads at s * n / kSamples
            const uint64_t s = (uint64_t)(t + j * kThreads);
            atomicAdd(&sm.bins[hb(load_key<BF16>(srow, (int64_t)((s * (uint64_t)n) / kSamples)) >> kShift)], 1u);
        }
        __syncthreads();
        uint32_t r = (uint32_t)((3 * (int64_t)k * kSamples) / (2 * n)) + 8;
        if (r > (uint32_t)kSamples) r = kSamples;
        find_bin(sm, r);
        T = sm.tbin << kShift;
        for (int i = t; i < kBins + kBins / 32; i += kThreads) sm.bins[i] = 0;
    }

    // ---- 2. one pass over the row: warp w owns [w0, w1) in whole batches of 1024 keys,
    // loaded coalesced, the next batch in flight (see issue_batch).  Keys >= T go to the warp's buffer in index order:
    // a key's slot is the warp's running count, plus the batch counts of the earlier
    // load slots v, plus the counts of the lower lanes in slot v (a warp prefix sum of
    // the per-slot counts packed in 16-bit fields), plus the earlier keys of its own vector.
    unsigned long long* wb = sm.wbuf + warp * kWarpCap;
    const int64_t part = ((n + P - 1) / P + 1023) / 1024 * 1024;   // this CTA's part of the row
    const int64_t r0 = rank * part, r1 = (r0 + part < n) ? r0 + part : n;
    const int64_t per_warp = ((r1 > r0 ? r1 - r0 : 0) + kWarps * 1024 - 1) / (kWarps * 1024) * 1024;
    const int64_t w0 = r0 + warp * per_warp, w1 = (w0 + per_warp < r1) ? w0 + per_warp : r1;
    const bool vec_ok = (reinterpret_cast<uintptr_t>(srow) & 15) == 0;
    constexpr int kE = Batch<BF16>::kE, kV = Batch<BF16>::kV;
    uint32_t wcnt = 0;
    Batch<BF16> nb;
    if (w0 < w1) issue_batch<BF16>(srow, vec_ok, w0, w1, lane, nb);
    for (int64_t bb = w0; bb < w1; bb += 1024) {
        uint32_t key[kV][kE], valid[kV];
        batch_keys<BF16>(srow, bb, w1, lane, nb, key, valid);
        if (bb + 1024 < w1) issue_batch<BF16>(srow, vec_ok, bb + 1024, w1, lane, nb);
        uint32_t pm[kV], cnt[kV];
#pragma unroll
        for (int v = 0; v < kV; ++v) {
            pm[v] = 0;
#pragma unroll
            for (int j = 0; j < kE; ++j) pm[v] |= (key[v][j] >= T ? 1u : 0u) << j;
            pm[v] &= valid[v];
            cnt[v] = __popc(pm[v]);
        }
        uint32_t incl[kV / 2], tot[kV / 2];
#pragma unroll
        for (int w = 0; w < kV / 2; ++w) {
            const uint32_t own = cnt[2 * w] | (cnt[2 * w + 1] << 16);
            uint32_t x = own;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            tot[w] = __shfl_sync(0xffffffffu, x, 31);
            incl[w] = x - own;   // exclusive
        }
        uint32_t base = wcnt;
#pragma unroll
        for (int v = 0; v < kV; ++v) {
            const uint32_t ex = (v & 1) ? (incl[v >> 1] >> 16) : (incl[v >> 1] & 0xFFFF);
            const uint32_t tv = (v & 1) ? (tot[v >> 1] >> 16) : (tot[v >> 1] & 0xFFFF);
            uint32_t slot = base + ex;
            const int64_t i = bb + 32 * kE * v + kE * lane;
#pragma unroll
            for (int j = 0; j < kE; ++j)
                if ((pm[v] >> j) & 1u) {
                    if (slot < kWarpCap)
                        wb[slot] = ((unsigned long long)key[v][j] << 32) | (unsigned long long)(~(uint32_t)(i + j));
                    ++slot;
                }
            base += tv;
        }
        wcnt = base;
    }
    if (lane == 0) { sm.warp_cnt[warp] = wcnt; sm.wsum[warp] = wcnt; }
    __syncthreads();
    scan_warp_sums(sm);
    if (t == 0) {
        uint32_t fail = (P == 1) && sm.total < (uint32_t)k;
        for (int w = 0; w < kWarps; ++w) fail |= sm.warp_cnt[w] > (uint32_t)kWarpCap;
        sm.fail = fail;
    }
    __syncthreads();
    if (P == 1 && sm.fail) {
        radix_select<BF16>(sm, srow, n, k, out);
        return;
    }
    if (!sm.fail) {
        const uint32_t o = sm.wsum[warp];
        for (uint32_t j = lane; j < wcnt; j += 32) sm.list[o + j] = wb[j];
    }
    __syncthreads();
    if constexpr (kWarps >= kMaxP) if (P > 1) {
        // ---- the row's CTAs form one cluster: CTA 0 appends the peers' candidate lists
        // (slices in rank order, so the list stays in index order) through distributed
        // shared memory, then selects; a missed bound falls back to CTA 0 alone.
        cluster_sync_all();
        if (rank == 0) {
            if (t < 32) {   // lane r reads rank r's count and flag (one remote load each, in parallel)
                const bool has = t < P;
                const uint32_t c = has ? ld_dsmem_u32(dsmem_addr(&sm.total, (uint32_t)t)) : 0u;
                const uint32_t f = has ? ld_dsmem_u32(dsmem_addr(&sm.fail, (uint32_t)t)) : 0u;
                uint32_t incl = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (t >= o) incl += y;
                }
                const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
                const bool anyf = __any_sync(0xffffffffu, f != 0);
                __syncwarp();
                if (has) {
                    sm.warp_off[t] = incl - c;
                    sm.warp_cnt[t] = c;
                }
                if (t == 0) {
                    sm.fail = anyf || tot < (uint32_t)k || tot > (uint32_t)kListCap;
                    sm.total = tot;
                }
            }
            __syncthreads();
            if (!sm.fail)
                for (int r = 1; r < P; ++r) {   // four remote loads in flight per thread
                    const uint32_t c = sm.warp_cnt[r], o = sm.warp_off[r];
                    const uint32_t src = dsmem_addr(&sm.list[0], (uint32_t)r);
                    for (uint32_t j0 = t; j0 < c; j0 += 4 * kThreads) {
                        unsigned long long v[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const uint32_t j = j0 + u * kThreads;
                            v[u] = j < c ? ld_dsmem_u64(src + j * 8) : 0ull;
                        }
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const uint32_t j = j0 + u * kThreads;
                            if (j < c) sm.list[o + j] = v[u];
                        }
                    }
                }
        }
        cluster_sync_all();   // the peers' lists have been read
        if (rank != 0) return;
        if (sm.fail) {
            radix_select<BF16>(sm, srow, n, k, out);
            return;
        }
    }
    const uint32_t C = sm.total;

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

// ------------------------------------------------------ rows held in registers
// Rows of at most kRowMaxP * kRowT * kRowKPT entries: a cluster of P CTAs per row (P the
// fewest that hold the row), CTA r of kRowT threads holding entries [r * kRowT * kRowKPT,
// ...), thread t the kRowKPT consecutive keys from t * kRowKPT of its part -- in registers,
// and mirrored in shared memory for the passes that visit only a thread's remaining
// candidates (a bit mask per thread).  Cluster order, then thread order, is index order.
// An exact MSB-first radix select finds the k-th largest key: each pass histograms the next
// digit of the keys that still share the resolved prefix, every CTA sums the cluster's
// histograms over distributed shared memory (each CTA adds its nonzero bins into every
// peer's copy with fire-and-forget remote reductions; the copies are double-buffered, so one
// cluster barrier per pass suffices), and the same block scan in every CTA picks the
// digit holding the k-th; the select stops early once the remaining count equals that
// bin's population (the whole bin is taken).  A last exchange of per-CTA counts places every
// selected key: all keys above the threshold, and the lowest-index ones equal to it, in
// ascending index order.
constexpr int kRowT = 512, kRowKPT = 16, kRowBins = 2048, kRowMaxP = 8;
constexpr int kRowPart = kRowT * kRowKPT;   // 8192 entries per CTA

struct RowSmem {
    uint32_t ks[kRowKPT * kRowT];           // key j of thread t at ks[j * kRowT + t]
    uint32_t hist[kRowBins];                // this CTA's histogram
    uint32_t ghist[2][kRowBins];            // the cluster's histogram (pass p: buffer p & 1)
    uint32_t wsum[2][32];
    uint32_t cnt[2];                        // this CTA's keys above / tied (read by the peers)
    uint32_t s_digit, s_above, s_inbin;
};

template <bool BF16>
__global__ void __launch_bounds__(kRowT, 1) topk_row_kernel(const void* __restrict__ scores, int64_t N_c,
                                                            const int64_t* __restrict__ q_pos, int m, int k,
                                                            int32_t* __restrict__ idx_out, int P) {
    extern __shared__ __align__(16) uint8_t row_smem_raw[];
    RowSmem& sm = *reinterpret_cast<RowSmem*>(row_smem_raw);
    constexpr int kBits = BF16 ? 16 : 32;
    constexpr int kWarpsR = kRowT / 32;
    const int64_t row = blockIdx.x / P;
    const int rank = (int)(blockIdx.x - row * P);   // == rank in the row's cluster
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
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif

    if (n <= k) {   // the same decision in every CTA of the cluster
        if (rank == 0)
            for (int i = t; i < k; i += kRowT) out[i] = (i < n) ? i : -1;
        return;
    }

    // ---- keys of this thread (entries at or beyond n read as key 0, below every finite score)
    const int64_t base = (int64_t)rank * kRowPart + (int64_t)t * kRowKPT;
    uint32_t key[kRowKPT];
    const bool vec = (reinterpret_cast<uintptr_t>(srow) & 15) == 0 && base + kRowKPT <= n;
    if (vec) {
        const uint4* p = reinterpret_cast<const uint4*>(srow + base * (BF16 ? 2 : 4));
        constexpr int kV = kRowKPT / (BF16 ? 8 : 4);
        uint4 raw[kV];
#pragma unroll
        for (int v = 0; v < kV; ++v) raw[v] = __ldg(p + v);
#pragma unroll
        for (int v = 0; v < kV; ++v) {
            const uint32_t ww[4] = {raw[v].x, raw[v].y, raw[v].z, raw[v].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if constexpr (BF16) {
                    key[v * 8 + 2 * q] = bf16_key((uint16_t)(ww[q] & 0xFFFF));
                    key[v * 8 + 2 * q + 1] = bf16_key((uint16_t)(ww[q] >> 16));
                } else {
                    key[v * 4 + q] = f32_key(__uint_as_float(ww[q]));
                }
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < kRowKPT; ++j) key[j] = (base + j < n) ? load_key<BF16>(srow, base + j) : 0u;
    }

    // the first pass's cluster histogram starts cleared in every CTA before any peer adds to it
    if (P > 1) {
        for (int i = t; i < kRowBins; i += kRowT) sm.ghist[0][i] = 0;
        cluster_sync_all();
    }

    // ---- radix select: digits of 11, 11, 10 bits (fp32 keys) or 11, 5 (bf16 keys)
    uint32_t prefix = 0, krem = (uint32_t)k;
    uint32_t cand = (1u << kRowKPT) - 1u;   // keys still sharing the prefix
    uint32_t above = 0;                     // keys known to lie above the threshold
    int done = 0;
    bool whole_bin = false;
#pragma unroll 1
    for (int pass = 0; pass < 3 && done < kBits; ++pass) {
        const int width = (kBits - done) < 11 ? (kBits - done) : 11;
        const int shift = kBits - done - width;
        const int nb = 1 << width;
        uint32_t* gh = sm.ghist[pass & 1];
        for (int i = t; i < nb; i += kRowT) sm.hist[i] = 0;
        // the next pass's buffer: its last readers (this CTA, two passes ago) are done, and
        // the barrier of this pass orders the clear before any peer's adds to it
        if (P > 1)
            for (int i = t; i < kRowBins; i += kRowT) sm.ghist[(pass + 1) & 1][i] = 0;
        __syncthreads();
        if (pass == 0) {
#pragma unroll
            for (int j = 0; j < kRowKPT; ++j) atomicAdd(&sm.hist[key[j] >> shift], 1u);
        } else {
            for (uint32_t mm = cand; mm != 0; mm &= mm - 1) {
                const uint32_t kk = sm.ks[(__ffs(mm) - 1) * kRowT + t];
                atomicAdd(&sm.hist[(kk >> shift) & (nb - 1)], 1u);
            }
        }
        // the cluster's histogram: every CTA adds its nonzero bins into every CTA's copy
        // (integer sums: the order of the additions does not matter)
        __syncthreads();
        if (P > 1) {
            for (int i = t; i < nb; i += kRowT) {
                const uint32_t v = sm.hist[i];
                if (v != 0)
                    for (int r = 0; r < P; ++r) red_dsmem_add_u32(dsmem_addr(&gh[i], (uint32_t)r), v);
            }
            cluster_sync_all();
        } else {
            gh = sm.hist;
        }
        // bins from the top: thread t owns bins b0, b0-1, ... (per of them; per = nb / kRowT
        // for nb = 2048, else 1)
        const int per = nb > kRowT ? nb / kRowT : 1;
        const int b0 = nb - 1 - t * per;
        uint32_t c[4] = {0u, 0u, 0u, 0u};
        uint32_t local = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (u < per && b0 - u >= 0) {
                c[u] = gh[b0 - u];
                local += c[u];
            }
        uint32_t incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) sm.wsum[0][warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const uint32_t v = lane < kWarpsR ? sm.wsum[0][lane] : 0u;
            uint32_t x = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            sm.wsum[1][lane] = x - v;
        }
        __syncthreads();
        uint32_t run = sm.wsum[1][warp] + incl - local;
        if (run < krem && run + local >= krem) {
            bool found = false;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (!found && u < per) {
                    if (run + c[u] >= krem) {
                        sm.s_digit = (uint32_t)(b0 - u);
                        sm.s_above = run;
                        sm.s_inbin = c[u];
                        found = true;
                    } else {
                        run += c[u];
                    }
                }
        }
        __syncthreads();
        const uint32_t dg = sm.s_digit;
        prefix = (prefix << width) | dg;
        done += width;
        krem -= sm.s_above;
        // split this thread's candidates: digit above the threshold digit, or equal to it
        uint32_t nc = 0;
        if (pass == 0) {
#pragma unroll
            for (int j = 0; j < kRowKPT; ++j) {
                const uint32_t d = key[j] >> shift;
                above |= (d > dg ? 1u : 0u) << j;
                nc |= (d == dg ? 1u : 0u) << j;
                if (d == dg) sm.ks[j * kRowT + t] = key[j];   // mirrored only where later passes look
            }
        } else {
            for (uint32_t mm = cand; mm != 0; mm &= mm - 1) {
                const int j = __ffs(mm) - 1;
                const uint32_t d = (sm.ks[j * kRowT + t] >> shift) & (nb - 1);
                if (d > dg) above |= 1u << j;
                else if (d == dg) nc |= 1u << j;
            }
        }
        cand = nc;
        const bool whole = sm.s_inbin == krem;
        __syncthreads();   // s_digit, s_above, s_inbin are rewritten by the next pass
        if (whole) {   // the whole threshold bin is taken
            whole_bin = true;
            break;
        }
    }

    // ---- ordered placement: keys above the threshold, then ties at it by index
    const uint32_t gt = __popc(above), eq = __popc(cand);
    uint32_t ig = gt, ie = eq;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t yg = __shfl_up_sync(0xffffffffu, ig, o);
        const uint32_t ye = __shfl_up_sync(0xffffffffu, ie, o);
        if (lane >= o) {
            ig += yg;
            ie += ye;
        }
    }
    if (lane == 31) {
        sm.wsum[0][warp] = ig;
        sm.wsum[1][warp] = ie;
    }
    __syncthreads();
    if (warp == 0) {
        const uint32_t vg = lane < kWarpsR ? sm.wsum[0][lane] : 0u;
        const uint32_t ve = lane < kWarpsR ? sm.wsum[1][lane] : 0u;
        uint32_t xg = vg, xe = ve;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t yg = __shfl_up_sync(0xffffffffu, xg, o);
            const uint32_t ye = __shfl_up_sync(0xffffffffu, xe, o);
            if (lane >= o) {
                xg += yg;
                xe += ye;
            }
        }
        __syncwarp();
        if (lane < kWarpsR) {
            sm.wsum[0][lane] = xg - vg;
            sm.wsum[1][lane] = xe - ve;
        }
        if (lane == 31) {   // this CTA's totals, for the peers of higher rank
            sm.cnt[0] = xg;
            sm.cnt[1] = xe;
        }
    }
    if (P > 1) cluster_sync_all();
    else __syncthreads();
    uint32_t cg = 0, ce = 0;   // keys above / tied in the CTAs of lower rank
    for (int r = 0; r < rank; ++r) {
        cg += ld_dsmem_u32(dsmem_addr(&sm.cnt[0], (uint32_t)r));
        ce += ld_dsmem_u32(dsmem_addr(&sm.cnt[1], (uint32_t)r));
    }
    const uint32_t gt_before = cg + sm.wsum[0][warp] + ig - gt;
    const uint32_t e0 = ce + sm.wsum[1][warp] + ie - eq;   // ties before this thread's keys
    uint32_t take = above;
    if (whole_bin) {
        take |= cand;
    } else if (e0 < krem) {   // the first krem - e0 ties of this thread
        uint32_t mm = cand;
        for (uint32_t r = e0; r < krem && mm != 0; ++r) mm &= mm - 1;
        take |= cand & ~mm;
    }
    uint32_t pos = gt_before + (whole_bin ? e0 : (e0 < krem ? e0 : krem));
    for (uint32_t mm = take; mm != 0; mm &= mm - 1) out[pos++] = (int32_t)(base + __ffs(mm) - 1);
    // no CTA leaves while a peer may still read its counts
    if (P > 1) cluster_sync_all();
}

}  // namespace

int64_t topk_scratch_bytes(int64_t rows, int64_t N_c) {
    (void)rows;
    (void)N_c;
    return 0;
}

namespace {
// CTAs per row: enough to spread the row pass over the SMs for a few rows, each CTA taking
// at least 4096 keys; one cluster per row, resident all at once.
template <bool BF16>
int choose_ranks(int64_t rows, int64_t N_c) {
    int64_t p = num_sms() / (rows > 0 ? rows : 1);
    const int64_t by_len = (N_c + 4095) / 4096;
    if (p > by_len) p = by_len;
    if (p > kMaxP) p = kMaxP;
    static std::mutex mu;
    static int cache[kMaxP + 1];
    std::lock_guard<std::mutex> lock(mu);
    const void* kern = reinterpret_cast<const void*>(topk_kernel<BF16, 512>);
    // The occupancy query sees the kernel's dynamic shared-memory limit: set it first.
    if (p > 1 && set_smem_once(kern, sizeof(TopkSmem<512>)) != cudaSuccess) p = 1;
    for (; p > 1; --p) {
        if (cache[p] == 0) {
            int n = 0;
            if (p <= 8 || cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
                cudaLaunchConfig_t cfg = {};
                cfg.gridDim = dim3((unsigned)p);
                cfg.blockDim = dim3(512);
                cfg.dynamicSmemBytes = sizeof(TopkSmem<512>);
                cudaLaunchAttribute attr[1];
                attr[0].id = cudaLaunchAttributeClusterDimension;
                attr[0].val.clusterDim.x = (unsigned)p;
                attr[0].val.clusterDim.y = 1;
                attr[0].val.clusterDim.z = 1;
                cfg.attrs = attr;
                cfg.numAttrs = 1;
                if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
            }
            cudaGetLastError();
            cache[p] = n > 0 ? n : -1;
        }
        if (cache[p] >= rows) break;
    }
    return (int)(p < 1 ? 1 : p);
}

// topk_kernel<BF16, NT> over rows x P CTAs, P CTAs per row in one cluster.
template <bool BF16, int NT>
cudaError_t launch_topk_cta(const void* scores, int64_t rows, int64_t N_c, const int64_t* q_pos, int m, int k,
                            int32_t* idx, cudaStream_t s, bool pdl, int P) {
    const void* kern = reinterpret_cast<const void*>(topk_kernel<BF16, NT>);
    cudaError_t e = set_smem_once(kern, sizeof(TopkSmem<NT>));
    if (e != cudaSuccess) return e;
    if constexpr (NT < 512) {   // two CTAs per SM need the whole carveout as shared memory
        static std::once_flag once;
        std::call_once(once, [&] { e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100); });
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rows * P));
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = sizeof(TopkSmem<NT>);
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (P > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)P;
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
    return cudaLaunchKernelEx(&cfg, topk_kernel<BF16, NT>, scores, N_c, q_pos, m, k, idx, P);
}

template <bool BF16>
cudaError_t launch_topk_t(const void* scores, int64_t rows, int64_t N_c, const int64_t* q_pos, int m, int k,
                          int32_t* idx, cudaStream_t s, bool pdl) {
    // The whole row fits a cluster's registers, and the clusters fit about two waves: few long
    // rows (decode).  Many rows (prefill) go to the kernel below, one CTA per row.
    const int P_row = (int)((N_c + kRowPart - 1) / kRowPart);
    if (N_c <= (int64_t)kRowMaxP * kRowPart && rows * P_row <= 2 * (int64_t)num_sms()) {
        const int P = P_row;
        constexpr size_t smem = sizeof(RowSmem);
        cudaError_t e = set_smem_once(reinterpret_cast<const void*>(topk_row_kernel<BF16>), smem);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(rows * P));
        cfg.blockDim = dim3(kRowT);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[2];
        int na = 0;
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)P;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
        if (pdl) {
            attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[na].val.programmaticStreamSerializationAllowed = 1;
            ++na;
        }
        cfg.attrs = attr;
        cfg.numAttrs = na;
        return cudaLaunchKernelEx(&cfg, topk_row_kernel<BF16>, scores, N_c, q_pos, m, k, idx, P);
    }
    const int P = choose_ranks<BF16>(rows, N_c);
    if (P == 1) return launch_topk_cta<BF16, 256>(scores, rows, N_c, q_pos, m, k, idx, s, pdl, 1);
    return launch_topk_cta<BF16, 512>(scores, rows, N_c, q_pos, m, k, idx, s, pdl, P);
}
}  // namespace

cudaError_t launch_topk(const void* scores, int score_dtype, int64_t B, int64_t Q, int64_t N_c,
                        const int64_t* q_pos, int m, int k, int32_t* idx, void* scratch, int* status,
                        cudaStream_t s, bool pdl) {
    (void)scratch;
    (void)status;
    const int64_t rows = B * Q;
    if (rows == 0 || k == 0) return cudaSuccess;
    return score_dtype == LCS_BF16 ? launch_topk_t<true>(scores, rows, N_c, q_pos, m, k, idx, s, pdl)
                                   : launch_topk_t<false>(scores, rows, N_c, q_pos, m, k, idx, s, pdl);
}

}  // namespace lcs
