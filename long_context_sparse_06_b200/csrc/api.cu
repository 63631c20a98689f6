// api.cu -- the extern "C" boundary of liblcs: argument validation, workspace
// layout and stream-ordered dispatch to the kernels.  Every host-detectable
// error returns before anything is enqueued.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "../../include/lcs.h"
#include "lcs_internal.h"

namespace lcs {

namespace {

int g_sms = 0;
bool g_device_ok = false;
std::once_flag g_once;

cudaEvent_t g_stage_events[8];
int g_n_stage_events = 0;

void probe_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return;
    cudaDeviceProp p;
    if (cudaGetDeviceProperties(&p, dev) != cudaSuccess) return;
    g_sms = p.multiProcessorCount;
    g_device_ok = (p.major == 10);
}

bool device_ok() {
    std::call_once(g_once, probe_device);
    return g_device_ok;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? LCS_OK : LCS_ERR_CUDA; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int* status_of(void* ws) { return static_cast<int*>(ws); }

// ---- workspace plans -------------------------------------------------------
struct IndexPlan {
    int64_t scores_off, qscratch_off, end;
};

int64_t score_bytes(int score_dtype) { return score_dtype == LCS_BF16 ? 2 : 4; }

IndexPlan plan_index(int64_t B, int64_t Q, int64_t N_c, int score_dtype, bool scores_external, bool fp4) {
    IndexPlan p;
    int64_t off = kStatusBytes;
    p.scores_off = off;
    if (!scores_external) off += align256(B * Q * N_c * score_bytes(score_dtype));
    p.qscratch_off = off;
    if (fp4) off += align256(index_fp4_scratch_bytes(B, Q, 128));
    p.end = off;
    return p;
}

void record_stage(int i, cudaStream_t s) {
    if (g_n_stage_events >= 2 && i < g_n_stage_events) cudaEventRecord(g_stage_events[i], s);
}

}  // namespace

int num_sms() {
    device_ok();
    return g_sms > 0 ? g_sms : 148;
}

namespace {
// Small cache of encoded tensor maps: decode loops call with the same buffers every
// step, and encoding costs microseconds of host time per map.
struct TmapKey {
    int dt;
    const void* base;
    uint64_t inner, outer, stride;
    uint32_t bi, bo;
    int swz;
    bool operator==(const TmapKey& o) const {
        return dt == o.dt && base == o.base && inner == o.inner && outer == o.outer && stride == o.stride &&
               bi == o.bi && bo == o.bo && swz == o.swz;
    }
};
constexpr int kTmapCache = 32;
TmapKey g_tkeys[kTmapCache];
CUtensorMap g_tmaps[kTmapCache];
int g_tnext = 0, g_tcount = 0;
std::mutex g_tmutex;
}  // namespace

namespace {
constexpr int kAttrSlots = 64;
const void* g_attr_fn[kAttrSlots];
size_t g_attr_bytes[kAttrSlots];
int g_attr_n = 0;
std::mutex g_attr_mutex;
}  // namespace

cudaError_t set_smem_once(const void* kern, size_t bytes) {
    std::lock_guard<std::mutex> lock(g_attr_mutex);
    int i = 0;
    for (; i < g_attr_n; ++i)
        if (g_attr_fn[i] == kern) break;
    if (i < g_attr_n && g_attr_bytes[i] >= bytes) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    if (i == g_attr_n && g_attr_n < kAttrSlots) g_attr_fn[g_attr_n++] = kern;
    if (i < kAttrSlots) g_attr_bytes[i] = bytes;
    return cudaSuccess;
}

bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
    const TmapKey key{(int)dt, base, inner, outer, row_stride_bytes, box_inner, box_outer, (int)swz};
    {
        std::lock_guard<std::mutex> lock(g_tmutex);
        for (int i = 0; i < g_tcount; ++i)
            if (g_tkeys[i] == key) {
                *map = g_tmaps[i];
                return true;
            }
    }
    EncodeTiledFn fn = get_encoder();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_stride_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    if (fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    std::lock_guard<std::mutex> lock(g_tmutex);
    g_tkeys[g_tnext] = key;
    g_tmaps[g_tnext] = *map;
    g_tnext = (g_tnext + 1) % kTmapCache;
    if (g_tcount < kTmapCache) ++g_tcount;
    return true;
}

// 3-D map over [outer2][outer1][inner] elements (rows of inner elements, row_stride bytes
// apart; planes plane_stride bytes apart), box {box_inner, box_rows, 1}, no swizzle.
// Out-of-range rows of a plane read as zeros.  Not cached (used by long-running calls).
bool encode_tmap_3d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer1,
                    uint64_t outer2, uint64_t row_stride_bytes, uint64_t plane_stride_bytes, uint32_t box_inner,
                    uint32_t box_rows) {
    EncodeTiledFn fn = get_encoder();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {inner, outer1, outer2};
    cuuint64_t strides[2] = {row_stride_bytes, plane_stride_bytes};
    cuuint32_t box[3] = {box_inner, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace lcs

using namespace lcs;

// ============================================================================
extern "C" {

const char* lcs_error_string(int code) {
    switch (code) {
        case LCS_OK: return "ok";
        case LCS_ERR_INVALID: return "invalid argument";
        case LCS_ERR_UNSUPPORTED: return "unsupported dtype or shape combination";
        case LCS_ERR_CUDA: return "CUDA error (no sm_100 device or launch failure)";
        case LCS_ERR_TIMEOUT: return "device-side wait timed out";
        case LCS_ERR_DEVICE: return "device-side check failed";
        case LCS_ERR_WORKSPACE: return "workspace missing or too small";
        case LCS_ERR_TOO_LARGE: return "problem needs more scratch than the allocation-free entry point holds";
        default: return "unknown status";
    }
}

int lcs_set_stage_events(cudaEvent_t const* events, int n) {
    if (n < 0 || n > 8 || (n > 0 && events == nullptr)) return LCS_ERR_INVALID;
    for (int i = 0; i < n; ++i) g_stage_events[i] = events[i];
    g_n_stage_events = n;
    return LCS_OK;
}

int lcs_clear_status(void* ws, cudaStream_t stream) {
    if (ws == nullptr) return LCS_ERR_INVALID;
    if (!device_ok()) return LCS_ERR_CUDA;
    return from_cuda(cudaMemsetAsync(ws, 0, kStatusBytes, stream));
}

int lcs_selftest_wait(int budget_us, void* ws, size_t ws_bytes, long long* out, cudaStream_t stream) {
    if (ws == nullptr || out == nullptr || ws_bytes < (size_t)kStatusBytes) return LCS_ERR_INVALID;
    if (budget_us < 1 || budget_us > 1000000) return LCS_ERR_INVALID;
    if (!device_ok()) return LCS_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, kStatusBytes, stream) != cudaSuccess) return LCS_ERR_CUDA;
    return from_cuda(launch_selftest_wait((uint64_t)budget_us * 1000ull, static_cast<int*>(ws), out, stream));
}

int lcs_status(void* ws, cudaStream_t stream) {
    if (ws == nullptr) return LCS_ERR_INVALID;
    if (!device_ok()) return LCS_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return LCS_ERR_CUDA;
    int st[2] = {0, 0};
    if (cudaMemcpy(st, ws, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return LCS_ERR_CUDA;
    if (st[0] != 0 && cudaMemset(ws, 0, kStatusBytes) != cudaSuccess) return LCS_ERR_CUDA;
    return st[0];
}

// ---------------------------------------------------------------- compressor
static int compress_common(const void* x, int x_dtype, int64_t B, int64_t T, int d, const void* x_tail,
                           const float* z_tail, const float* z, const float* bias, int m, int overlap, int d_rope,
                           float theta, int64_t pos0, void* out, int out_dtype, cudaStream_t stream) {
    if (x == nullptr || z == nullptr || bias == nullptr || out == nullptr) return LCS_ERR_INVALID;
    if (B < 0 || T < 0 || m < 1 || m > 1024 || overlap < 0 || overlap > 1024 || T % m) return LCS_ERR_INVALID;
    if (d <= 0 || d > 4096 || d % 8 || d_rope < 0 || d_rope > d || (d_rope & 1)) return LCS_ERR_INVALID;
    if ((x_tail == nullptr) != (z_tail == nullptr)) return LCS_ERR_INVALID;
    if (overlap == 0 && x_tail != nullptr) return LCS_ERR_INVALID;
    if ((x_dtype != LCS_F32 && x_dtype != LCS_BF16) || (out_dtype != LCS_F32 && out_dtype != LCS_BF16))
        return LCS_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(out) || (x_tail && !aligned16(x_tail))) return LCS_ERR_INVALID;
    if (!(theta > 0.f)) return LCS_ERR_INVALID;
    if (!device_ok()) return LCS_ERR_CUDA;
    return from_cuda(launch_compress(x, x_dtype, B, T, d, x_tail, z_tail, z, bias, m, overlap, d_rope, theta, pos0,
                                     out, out_dtype, stream));
}

int csa_compress(const void* x, int x_dtype, int64_t B, int64_t T, int d, const void* x_tail, const float* z_tail,
                 const float* z, const float* bias, int m, int overlap, int d_rope, float rope_theta, int64_t pos0,
                 void* out, int out_dtype, cudaStream_t stream) {
    return compress_common(x, x_dtype, B, T, d, x_tail, z_tail, z, bias, m, overlap, d_rope, rope_theta, pos0, out,
                           out_dtype, stream);
}

int hca_compress(const void* x, int x_dtype, int64_t B, int64_t T, int d, const float* z, const float* bias, int m,
                 int d_rope, float rope_theta, int64_t pos0, void* out, int out_dtype, cudaStream_t stream) {
    return compress_common(x, x_dtype, B, T, d, nullptr, nullptr, z, bias, m, 0, d_rope, rope_theta, pos0, out,
                           out_dtype, stream);
}

int lcs_compress_proj(const void* h, int h_dtype, int64_t B, int64_t T, int hidden, const void* h_tail,
                      const void* Wx, int d, const float* wz, const float* bias, int m, int overlap, int d_rope,
                      float rope_theta, int64_t pos0, void* out, int out_dtype, cudaStream_t stream) {
    if (h == nullptr || Wx == nullptr || wz == nullptr || bias == nullptr || out == nullptr) return LCS_ERR_INVALID;
    if (B < 0 || T < 0 || m < 1 || m > 1024 || overlap < 0 || overlap > 1024 || T % m) return LCS_ERR_INVALID;
    if (hidden <= 0 || d <= 0 || d > 4096 || d_rope < 0 || d_rope > d || (d_rope & 1)) return LCS_ERR_INVALID;
    if (overlap == 0 && h_tail != nullptr) return LCS_ERR_INVALID;
    if (!(rope_theta > 0.f)) return LCS_ERR_INVALID;
    if ((h_dtype != LCS_F32 && h_dtype != LCS_BF16) || (out_dtype != LCS_F32 && out_dtype != LCS_BF16))
        return LCS_ERR_UNSUPPORTED;
    if (compress_proj_tile(hidden, d, m, overlap) == 0) return LCS_ERR_UNSUPPORTED;
    if (!device_ok()) return LCS_ERR_CUDA;
    return from_cuda(launch_compress_proj(h, h_dtype, B, T, hidden, h_tail, Wx, d, wz, bias, m, overlap, d_rope,
                                          rope_theta, pos0, out, out_dtype, stream));
}

// ------------------------------------------------------------------ indexer
static int validate_index(const void* qI, int qI_dtype, const float* w, const void* kI, int kI_dtype, int64_t B,
                          int64_t Q, int64_t N_c, int H_I, int d_I, const int64_t* q_pos, int m, int k,
                          int score_dtype) {
    if (qI == nullptr || w == nullptr || kI == nullptr) return LCS_ERR_INVALID;
    if (B < 0 || Q < 0 || N_c < 0 || H_I <= 0 || d_I <= 0 || d_I % 32 || k < 0 || k > 4096) return LCS_ERR_INVALID;
    if (q_pos == nullptr && Q != 1) return LCS_ERR_INVALID;
    if (q_pos != nullptr && m < 1) return LCS_ERR_INVALID;
    if (N_c >= (int64_t(1) << 31) || B * N_c >= (int64_t(1) << 31)) return LCS_ERR_INVALID;
    if (qI_dtype == LCS_F32 && kI_dtype == LCS_F32) {
        if (score_dtype != LCS_F32 || H_I > 128 || d_I > 256) return LCS_ERR_UNSUPPORTED;
        return LCS_OK;
    }
    if (qI_dtype == LCS_BF16 && kI_dtype == LCS_BF16) {
        if (score_dtype != LCS_F32 || H_I != 64 || d_I != 128) return LCS_ERR_UNSUPPORTED;
        if (!aligned16(qI) || !aligned16(kI)) return LCS_ERR_INVALID;
        return LCS_OK;
    }
    if (qI_dtype == LCS_BF16 && kI_dtype == LCS_FP4) {
        if (score_dtype != LCS_BF16 || H_I != 64 || d_I != 128) return LCS_ERR_UNSUPPORTED;
        // the packed key plane is read by TMA as bytes (16-byte aligned base)
        if (!aligned16(qI) || !aligned16(kI)) return LCS_ERR_INVALID;
        return LCS_OK;
    }
    return LCS_ERR_UNSUPPORTED;
}

static int run_index(const void* qI, int qI_dtype, const float* w, const void* kI, int kI_dtype, int64_t B, int64_t Q,
                     int64_t N_c, int H_I, int d_I, const int64_t* q_pos, int m, void* scores, uint8_t* qscratch,
                     int* status, cudaStream_t stream, bool pdl) {
    if (kI_dtype == LCS_F32)
        return from_cuda(launch_index_f32(static_cast<const float*>(qI), w, static_cast<const float*>(kI), B, Q, N_c,
                                          H_I, d_I, q_pos, m, static_cast<float*>(scores), stream));
    if (kI_dtype == LCS_BF16)
        return from_cuda(launch_index_bf16_tc(qI, w, kI, B, Q, N_c, d_I, q_pos, m, static_cast<float*>(scores),
                                              status, stream, pdl));
    return from_cuda(launch_index_fp4_tc(qI, w, kI, B, Q, N_c, d_I, q_pos, m, static_cast<uint16_t*>(scores),
                                         qscratch, status, stream, pdl));
}

int csa_index_topk(const void* qI, int qI_dtype, const float* w, const void* kI, int kI_dtype, int64_t B, int64_t Q,
                   int64_t N_c, int H_I, int d_I, const int64_t* q_pos, int m, int k, int score_dtype, int32_t* idx,
                   void* scores, void* ws, size_t ws_bytes, cudaStream_t stream) {
    int v = validate_index(qI, qI_dtype, w, kI, kI_dtype, B, Q, N_c, H_I, d_I, q_pos, m, k, score_dtype);
    if (v != LCS_OK) return v;
    if (idx == nullptr) return LCS_ERR_INVALID;
    const bool fp4 = kI_dtype == LCS_FP4;
    const IndexPlan p = plan_index(B, Q, N_c, score_dtype, scores != nullptr, fp4);
    if (ws == nullptr || (int64_t)ws_bytes < p.end || (reinterpret_cast<uintptr_t>(ws) & 255)) return LCS_ERR_WORKSPACE;
    if (!device_ok()) return LCS_ERR_CUDA;
    uint8_t* base = static_cast<uint8_t*>(ws);
    void* sc = scores ? scores : base + p.scores_off;
    record_stage(0, stream);
    int r = run_index(qI, qI_dtype, w, kI, kI_dtype, B, Q, N_c, H_I, d_I, q_pos, m, sc, base + p.qscratch_off,
                      status_of(ws), stream, false);
    if (r != LCS_OK) return r;
    record_stage(1, stream);
    r = from_cuda(launch_topk(sc, score_dtype, B, Q, N_c, q_pos, m, k, idx, nullptr, status_of(ws), stream,
                              g_n_stage_events == 0));
    record_stage(2, stream);
    return r;
}

int csa_index_topk_proj(const float* h, int hidden, const float* W_qI, const float* W_w, const float* kI, int64_t B,
                        int64_t Q, int64_t N_c, int H_I, int d_I, const int64_t* q_pos, int m, int k, int32_t* idx,
                        float* scores, void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (h == nullptr || W_qI == nullptr || W_w == nullptr || kI == nullptr || idx == nullptr) return LCS_ERR_INVALID;
    if (B < 0 || Q < 0 || N_c < 0 || H_I <= 0 || H_I > 128 || d_I <= 0 || d_I > 256 || k < 0 || k > 4096)
        return LCS_ERR_INVALID;
    if (hidden <= 0 || hidden > 8192 || (int64_t)hidden + (int64_t)H_I * d_I + H_I > 12288) return LCS_ERR_UNSUPPORTED;
    if (q_pos == nullptr && Q != 1) return LCS_ERR_INVALID;
    if (q_pos != nullptr && m < 1) return LCS_ERR_INVALID;
    if (N_c >= (int64_t(1) << 31) || B * N_c >= (int64_t(1) << 31)) return LCS_ERR_INVALID;
    const IndexPlan p = plan_index(B, Q, N_c, LCS_F32, scores != nullptr, false);
    if (ws == nullptr || (int64_t)ws_bytes < p.end || (reinterpret_cast<uintptr_t>(ws) & 255)) return LCS_ERR_WORKSPACE;
    if (!device_ok()) return LCS_ERR_CUDA;
    float* sc = scores ? scores : reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + p.scores_off);
    int r = from_cuda(launch_index_proj_f32(h, hidden, W_qI, W_w, kI, B, Q, N_c, H_I, d_I, q_pos, m, sc, stream));
    if (r != LCS_OK) return r;
    return from_cuda(launch_topk(sc, LCS_F32, B, Q, N_c, q_pos, m, k, idx, nullptr, status_of(ws), stream, false));
}

int lcs_topk(const void* scores, int score_dtype, int64_t B, int64_t Q, int64_t N_c, const int64_t* q_pos, int m,
             int k, int32_t* idx, void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (scores == nullptr || idx == nullptr) return LCS_ERR_INVALID;
    if (B < 0 || Q < 0 || N_c < 0 || k < 0 || k > 4096) return LCS_ERR_INVALID;
    if (q_pos != nullptr && m < 1) return LCS_ERR_INVALID;
    if (score_dtype != LCS_F32 && score_dtype != LCS_BF16) return LCS_ERR_UNSUPPORTED;
    if (ws == nullptr || ws_bytes < (size_t)kStatusBytes) return LCS_ERR_WORKSPACE;
    if (!device_ok()) return LCS_ERR_CUDA;
    return from_cuda(launch_topk(scores, score_dtype, B, Q, N_c, q_pos, m, k, idx, nullptr, status_of(ws), stream, false));
}

// ---------------------------------------------------------------- attention
static int validate_attend(const AttendArgs& a, int q_dtype, int out_dtype) {
    if (a.q == nullptr || a.out == nullptr || a.comp == nullptr) return LCS_ERR_INVALID;
    if (a.B < 0 || a.Q < 0 || a.N_c < 0 || a.Tw < 0 || a.W < 1 || a.H <= 0 || a.D <= 0 || a.d_v <= 0 || a.d_v > a.D)
        return LCS_ERR_INVALID;
    if (a.Tw > 0 && a.win == nullptr) return LCS_ERR_INVALID;
    if ((a.q_pos == nullptr) != (a.win_pos0 == nullptr)) return LCS_ERR_INVALID;
    if (a.q_pos == nullptr && a.Q != 1) return LCS_ERR_INVALID;
    if (a.idx == nullptr && a.q_pos != nullptr && a.m < 1) return LCS_ERR_INVALID;
    if (!(a.scale > 0.f)) return LCS_ERR_INVALID;
    if (a.kv_dtype == LCS_F32) {
        if (q_dtype != LCS_F32 || out_dtype != LCS_F32) return LCS_ERR_UNSUPPORTED;
        if (a.H > 64 || a.D > 128 || a.d_v > 128 || a.k > 4096) return LCS_ERR_UNSUPPORTED;
        return LCS_OK;
    }
    if (a.kv_dtype == LCS_BF16 || a.kv_dtype == LCS_KV_FP8) {
        if (q_dtype != LCS_BF16 || (out_dtype != LCS_BF16 && out_dtype != LCS_F32)) return LCS_ERR_UNSUPPORTED;
        if (a.H != 64 || a.D != 576 || a.d_v != 512 || a.k > 2048) return LCS_ERR_UNSUPPORTED;
        // runs of consecutive rows are loaded by TMA, whose row coordinates are int32
        if (a.B * a.N_c >= (int64_t(1) << 31) || a.B * a.Tw >= (int64_t(1) << 31)) return LCS_ERR_UNSUPPORTED;
        if (!aligned16(a.q) || !aligned16(a.comp) || (a.win && !aligned16(a.win)) || !aligned16(a.out))
            return LCS_ERR_INVALID;
        return LCS_OK;
    }
    return LCS_ERR_UNSUPPORTED;
}

static int run_attend(const AttendArgs& a, int q_dtype, int out_dtype, void* ws, size_t ws_bytes, int64_t scratch_off,
                      cudaStream_t stream, bool pdl) {
    int v = validate_attend(a, q_dtype, out_dtype);
    if (v != LCS_OK) return v;
    const int64_t need = scratch_off + align256(attend_scratch_bytes(a));
    if (ws == nullptr || (int64_t)ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255)) return LCS_ERR_WORKSPACE;
    if (!device_ok()) return LCS_ERR_CUDA;
    return from_cuda(launch_attend(a, static_cast<uint8_t*>(ws) + scratch_off, status_of(ws), stream, pdl));
}

int csa_attend(const void* q, int q_dtype, const void* comp, const void* win, int kv_dtype, int64_t B, int64_t Q,
               int64_t N_c, int64_t Tw, const int32_t* idx, int k, const int64_t* q_pos, const int64_t* win_pos0,
               int W, int H, int D, int d_v, float scale, void* out, int out_dtype, float* lse, void* ws,
               size_t ws_bytes, cudaStream_t stream) {
    if (idx == nullptr || k < 0) return LCS_ERR_INVALID;
    AttendArgs a{q, comp, win, kv_dtype, B, Q, N_c, Tw, idx, k, q_pos, win_pos0, 1, W, H, D, d_v, scale, out, lse,
                 out_dtype};
    return run_attend(a, q_dtype, out_dtype, ws, ws_bytes, kStatusBytes, stream, false);
}

int hca_attend(const void* q, int q_dtype, const void* comp, const void* win, int kv_dtype, int64_t B, int64_t Q,
               int64_t N_c, int64_t Tw, const int64_t* q_pos, const int64_t* win_pos0, int m, int W, int H, int D,
               int d_v, float scale, void* out, int out_dtype, float* lse, void* ws, size_t ws_bytes,
               cudaStream_t stream) {
    AttendArgs a{q, comp, win, kv_dtype, B, Q, N_c, Tw, nullptr, 0, q_pos, win_pos0, m, W, H, D, d_v, scale, out, lse,
                 out_dtype};
    return run_attend(a, q_dtype, out_dtype, ws, ws_bytes, kStatusBytes, stream, false);
}

// Allocation-free csa_attend: the same validation and kernels, with the scratch in
// the library's fixed per-device array (noalloc.cu) instead of a caller workspace.
int csa_attend_noalloc(const void* q, int q_dtype, const void* comp, const void* win, int kv_dtype, int64_t B,
                       int64_t Q, int64_t N_c, int64_t Tw, const int32_t* idx, int k, const int64_t* q_pos,
                       const int64_t* win_pos0, int W, int H, int D, int d_v, float scale, void* out, int out_dtype,
                       float* lse, int* status_out, cudaStream_t stream) {
    if (idx == nullptr || k < 0) return LCS_ERR_INVALID;
    AttendArgs a{q, comp, win, kv_dtype, B, Q, N_c, Tw, idx, k, q_pos, win_pos0, 1, W, H, D, d_v, scale, out, lse,
                 out_dtype};
    int v = validate_attend(a, q_dtype, out_dtype);
    if (v != LCS_OK) return v;
    if (kStatusBytes + align256(attend_scratch_bytes(a)) > (int64_t)LCS_NOALLOC_SCRATCH_BYTES)
        return LCS_ERR_TOO_LARGE;
    if (!device_ok()) return LCS_ERR_CUDA;
    void* ws = nullptr;
    v = noalloc_scratch(&ws);
    if (v != LCS_OK) return v;
    // The status word must start at zero; the partials are written before they are read.
    if (cudaMemsetAsync(ws, 0, kStatusBytes, stream) != cudaSuccess) return LCS_ERR_CUDA;
    if (launch_attend(a, static_cast<uint8_t*>(ws) + kStatusBytes, status_of(ws), stream, false) != cudaSuccess)
        return LCS_ERR_CUDA;
    if (status_out != nullptr &&
        cudaMemcpyAsync(status_out, ws, sizeof(int), cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
        return LCS_ERR_CUDA;
    return LCS_OK;
}

// ------------------------------------------------------------- fused decode
static int64_t decode_layout(int mode, int64_t B, int64_t N_c, int64_t Tw, int k, int score_dtype, bool fp4,
                             int64_t* scores_off, int64_t* idx_off, int64_t* attend_off, const AttendArgs& a) {
    int64_t off = kStatusBytes;
    *scores_off = off;
    *idx_off = off;
    if (mode == LCS_MODE_CSA) {
        IndexPlan p = plan_index(B, 1, N_c, score_dtype, false, fp4);
        off = p.end;
        *idx_off = off;
        off += align256(B * k * 4);
    }
    *attend_off = off;
    off += align256(attend_scratch_bytes(a));
    (void)Tw;
    return off;
}

int decode_fused(int mode, int64_t B, const void* q, int q_dtype, const void* comp, const void* win, int kv_dtype,
                 int64_t N_c, int64_t Tw, int H, int D, int d_v, float scale, const void* qI, int qI_dtype,
                 const float* w, const void* kI, int kI_dtype, int H_I, int d_I, int k, int score_dtype, void* out,
                 int out_dtype, float* lse, int32_t* idx_out, void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (mode != LCS_MODE_CSA && mode != LCS_MODE_HCA) return LCS_ERR_INVALID;
    const bool csa = mode == LCS_MODE_CSA;
    if (csa) {
        int v = validate_index(qI, qI_dtype, w, kI, kI_dtype, B, 1, N_c, H_I, d_I, nullptr, 4, k, score_dtype);
        if (v != LCS_OK) return v;
    }
    AttendArgs a{q, comp, win, kv_dtype, B, 1, N_c, Tw, nullptr, csa ? k : 0, nullptr, nullptr, 1, 128, H, D, d_v,
                 scale, out, lse, out_dtype};
    if (csa) a.idx = reinterpret_cast<const int32_t*>(1);   // placeholder for validation and the split plan
    int v = validate_attend(a, q_dtype, out_dtype);
    if (v != LCS_OK) return v;
    const bool fp4 = csa && kI_dtype == LCS_FP4;
    int64_t scores_off, idx_off, attend_off;
    const int64_t need = decode_layout(mode, B, N_c, Tw, k, score_dtype, fp4, &scores_off, &idx_off, &attend_off, a);
    if (ws == nullptr || (int64_t)ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255)) return LCS_ERR_WORKSPACE;
    if (!device_ok()) return LCS_ERR_CUDA;
    uint8_t* base = static_cast<uint8_t*>(ws);
    int* status = status_of(ws);
    record_stage(0, stream);
    if (csa) {
        int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(base + idx_off);
        int r = run_index(qI, qI_dtype, w, kI, kI_dtype, B, 1, N_c, H_I, d_I, nullptr, 4, base + scores_off,
                          base + plan_index(B, 1, N_c, score_dtype, false, fp4).qscratch_off, status, stream, true);
        if (r != LCS_OK) return r;
        record_stage(1, stream);
        if (launch_topk(base + scores_off, score_dtype, B, 1, N_c, nullptr, 4, k, idx, nullptr, status, stream,
                        g_n_stage_events == 0) != cudaSuccess)
            return LCS_ERR_CUDA;
        record_stage(2, stream);
        a.idx = idx;
    }
    if (launch_attend(a, base + attend_off, status, stream, csa && g_n_stage_events == 0) != cudaSuccess)
        return LCS_ERR_CUDA;
    record_stage(csa ? 3 : 1, stream);
    return LCS_OK;
}

// ------------------------------------------------------- decode cache update
int lcs_cache_append(int64_t B, const int64_t* pos, const void* x, const void* kx, int x_dtype, const float* z,
                     const float* zI, const float* zh, const float* bias, const float* biasI, const float* biash,
                     int D, int d_rope, int d_I, float rope_theta, void* raw, float* logits, void* win, int win_dtype,
                     void* comp, void* kI, void* hca, int64_t N_c, int64_t N_h, int kv_dtype, int kI_dtype, void* ws,
                     size_t ws_bytes, cudaStream_t stream) {
    if (pos == nullptr || x == nullptr || kx == nullptr || z == nullptr || zI == nullptr || zh == nullptr ||
        bias == nullptr || biasI == nullptr || biash == nullptr || raw == nullptr || logits == nullptr ||
        win == nullptr || comp == nullptr || kI == nullptr || hca == nullptr)
        return LCS_ERR_INVALID;
    if (B < 0 || N_c < 0 || N_h < 0 || D <= 0 || D > 4096 || D % 8 || d_I <= 0 || d_I > 1024 || d_I % 32 ||
        d_rope < 0 || d_rope > D || (d_rope & 1) || !(rope_theta > 0.f))
        return LCS_ERR_INVALID;
    if (x_dtype != LCS_F32 && x_dtype != LCS_BF16) return LCS_ERR_UNSUPPORTED;
    const bool kv_ok = kv_dtype == LCS_F32 || kv_dtype == LCS_BF16 || (kv_dtype == LCS_KV_FP8 && (D - d_rope) % 128 == 0);
    const bool win_ok = win_dtype == LCS_F32 || win_dtype == LCS_BF16 || (win_dtype == LCS_KV_FP8 && (D - d_rope) % 128 == 0);
    if (!kv_ok || !win_ok || (kI_dtype != LCS_F32 && kI_dtype != LCS_BF16 && kI_dtype != LCS_FP4))
        return LCS_ERR_UNSUPPORTED;
    if ((kv_dtype == LCS_KV_FP8 || win_dtype == LCS_KV_FP8) && (!aligned16(comp) || !aligned16(win) || !aligned16(hca)))
        return LCS_ERR_INVALID;
    if (ws == nullptr || ws_bytes < (size_t)kStatusBytes || (reinterpret_cast<uintptr_t>(ws) & 255))
        return LCS_ERR_WORKSPACE;
    if (!device_ok()) return LCS_ERR_CUDA;
    return from_cuda(launch_cache_append(pos, x, kx, x_dtype, z, zI, zh, bias, biasI, biash, D, d_rope, d_I,
                                         rope_theta, raw, logits, win, win_dtype, comp, kI, hca, B, N_c, N_h, kv_dtype,
                                         kI_dtype, status_of(ws), stream));
}

// ------------------------------------------------- context parallelism (one long request)
int lcs_cp_candidates(const void* scores, int score_dtype, int64_t B, int64_t S, const int32_t* idx_local, int k,
                      int64_t offset, float* cand_score, int32_t* cand_idx, cudaStream_t stream) {
    if (scores == nullptr || idx_local == nullptr || cand_score == nullptr || cand_idx == nullptr) return LCS_ERR_INVALID;
    if (B < 0 || S < 0 || k < 0 || k > 4096 || offset < 0 || offset + S >= (int64_t(1) << 31)) return LCS_ERR_INVALID;
    if (score_dtype != LCS_F32 && score_dtype != LCS_BF16) return LCS_ERR_UNSUPPORTED;
    if (!device_ok()) return LCS_ERR_CUDA;
    return from_cuda(launch_cp_candidates(scores, score_dtype, B, S, idx_local, k, offset, cand_score, cand_idx, stream));
}

int lcs_cp_select(const float* cand_score, const int32_t* cand_idx, int G, int64_t B, int k, int64_t offset, int64_t S,
                  int32_t* idx_global, int32_t* idx_local, void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (cand_score == nullptr || cand_idx == nullptr || idx_global == nullptr || idx_local == nullptr)
        return LCS_ERR_INVALID;
    if (G < 1 || G > 64 || B < 0 || k < 0 || k > 4096 || offset < 0 || S < 0) return LCS_ERR_INVALID;
    const int64_t need = kStatusBytes + align256(cp_select_scratch_bytes(G, B, k));
    if (ws == nullptr || (int64_t)ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255)) return LCS_ERR_WORKSPACE;
    if (!device_ok()) return LCS_ERR_CUDA;
    return from_cuda(launch_cp_select(cand_score, cand_idx, G, B, k, offset, S, idx_global, idx_local,
                                      static_cast<uint8_t*>(ws) + kStatusBytes, status_of(ws), stream));
}

int lcs_attn_merge(const float* o, const float* lse, int G, int64_t rows, int d_v, void* out, int out_dtype,
                   float* lse_out, cudaStream_t stream) {
    if (o == nullptr || lse == nullptr || out == nullptr) return LCS_ERR_INVALID;
    if (G < 1 || G > 1024 || rows < 0 || d_v <= 0 || d_v > 4096) return LCS_ERR_INVALID;
    if (out_dtype != LCS_F32 && out_dtype != LCS_BF16) return LCS_ERR_UNSUPPORTED;
    if (!device_ok()) return LCS_ERR_CUDA;
    return from_cuda(launch_attn_merge(o, lse, G, rows, d_v, out, out_dtype, lse_out, stream));
}

// ------------------------------------------------------------------- misc
int group_oproj(const float* o, int64_t T, int H, int d_v, const float* Wg, int G, int d_g, const float* Wo,
                int hidden, float* y, cudaStream_t stream) {
    if (o == nullptr || Wg == nullptr || Wo == nullptr || y == nullptr) return LCS_ERR_INVALID;
    if (T < 0 || H <= 0 || d_v <= 0 || G <= 0 || H % G || d_g <= 0 || hidden <= 0) return LCS_ERR_INVALID;
    if ((H / G) * d_v > 4096 || G * d_g > 1024 || H * d_v > 8192) return LCS_ERR_UNSUPPORTED;
    if (!device_ok()) return LCS_ERR_CUDA;
    return from_cuda(launch_group_oproj(o, T, H, d_v, Wg, G, d_g, Wo, hidden, y, stream));
}

int lcs_rope(void* rows, int dtype, int64_t n, int d, int d_rope, float rope_theta, const int64_t* pos,
             cudaStream_t stream) {
    if (rows == nullptr || (n > 0 && pos == nullptr)) return LCS_ERR_INVALID;
    if (n < 0 || d <= 0 || d_rope < 0 || d_rope > d || (d_rope & 1) || !(rope_theta > 0.f)) return LCS_ERR_INVALID;
    if (dtype != LCS_F32 && dtype != LCS_BF16) return LCS_ERR_UNSUPPORTED;
    if (!device_ok()) return LCS_ERR_CUDA;
    return from_cuda(launch_rope(rows, dtype, n, d, d_rope, rope_theta, pos, stream));
}

int lcs_quant_kv_fp8(const float* x, int64_t n, int d_c, int d_r, void* out, cudaStream_t stream) {
    if (x == nullptr || out == nullptr) return LCS_ERR_INVALID;
    if (n < 0 || d_c <= 0 || d_c % 128 || d_r < 0 || !aligned16(x)) return LCS_ERR_INVALID;
    if (!device_ok()) return LCS_ERR_CUDA;
    return from_cuda(launch_quant_kv_fp8(x, n, d_c, d_r, out, stream));
}

int lcs_quant_fp4(const float* x, int64_t n, int d, void* out, cudaStream_t stream) {
    if (x == nullptr || out == nullptr) return LCS_ERR_INVALID;
    if (n < 0 || d <= 0 || d % 32) return LCS_ERR_INVALID;
    if (!device_ok()) return LCS_ERR_CUDA;
    return from_cuda(launch_quant_fp4(x, n, d, out, stream));
}

int64_t lcs_workspace_size(int op, int64_t B, int64_t Q, int64_t N_c, int64_t Tw, int k, int H, int d_v,
                           int score_dtype) {
    if (B < 0 || Q < 0 || N_c < 0 || Tw < 0 || k < 0) return -1;
    switch (op) {
        case LCS_OP_TOPK: return kStatusBytes;
        case LCS_OP_CP_SELECT:   // Q carries the number of ranks G
            if (Q < 1 || Q > 64) return -1;
            return kStatusBytes + align256(cp_select_scratch_bytes((int)Q, B, k));
        case LCS_OP_INDEX_TOPK:
            return plan_index(B, Q, N_c, score_dtype, false, score_dtype == LCS_BF16).end;
        case LCS_OP_ATTEND: {
            // Upper bound over CSA (k rows) and HCA (N_c rows); the window counted as Tw rows.
            AttendArgs a{nullptr, nullptr, nullptr, LCS_BF16, B, Q, N_c, Tw, nullptr, k, nullptr, nullptr, 1, 128,
                         H, 576, d_v, 1.f, nullptr, nullptr, LCS_BF16};
            AttendArgs c = a;
            c.idx = reinterpret_cast<const int32_t*>(1);
            int64_t s1 = attend_scratch_bytes(a), s2 = attend_scratch_bytes(c);
            return kStatusBytes + align256(s1 > s2 ? s1 : s2);
        }
        case LCS_OP_DECODE: {
            AttendArgs a{nullptr, nullptr, nullptr, LCS_BF16, B, 1, N_c, Tw, nullptr, k, nullptr, nullptr, 1, 128,
                         H, 576, d_v, 1.f, nullptr, nullptr, LCS_BF16};
            AttendArgs c = a;
            c.idx = reinterpret_cast<const int32_t*>(1);
            int64_t so, io, ao;
            int64_t hca = decode_layout(LCS_MODE_HCA, B, N_c, Tw, k, score_dtype, false, &so, &io, &ao, a);
            int64_t csa = decode_layout(LCS_MODE_CSA, B, N_c, Tw, k, score_dtype, score_dtype == LCS_BF16, &so, &io,
                                        &ao, c);
            return hca > csa ? hca : csa;
        }
        default: return -1;
    }
}

}  // extern "C"
