// lcs_internal.h -- host-side launchers shared between the kernel files and the
// C-ABI layer.  Launchers assume validated arguments and return a cudaError_t.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <utility>

namespace lcs {

// Workspace layout: [0, 256) status word; then the op's scratch regions, each
// 256-byte aligned.
constexpr int64_t kStatusBytes = 256;
inline int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }

int num_sms();

// compress.cu
cudaError_t launch_compress(const void* x, int x_dtype, int64_t B, int64_t T, int d, const void* x_tail,
                            const float* z_tail, const float* z, const float* bias, int m, int overlap, int d_rope,
                            float theta, int64_t pos0, void* out, int out_dtype, cudaStream_t s);

// misc.cu
cudaError_t launch_rope(void* rows, int dtype, int64_t n, int d, int d_rope, float theta, const int64_t* pos,
                        cudaStream_t s);
cudaError_t launch_quant_kv_fp8(const float* x, int64_t n, int d_c, int d_r, void* out, cudaStream_t s);
cudaError_t launch_quant_fp4(const float* x, int64_t n, int d, void* out, cudaStream_t s);
cudaError_t launch_group_oproj(const float* o, int64_t T, int H, int d_v, const float* Wg, int G, int d_g,
                               const float* Wo, int hidden, float* y, cudaStream_t s);

// indexer.cu -- scores [B, Q, N_c] (fp32 or bf16)
cudaError_t launch_index_f32(const float* qI, const float* w, const float* kI, int64_t B, int64_t Q, int64_t N_c,
                             int H_I, int d_I, const int64_t* q_pos, int m, float* scores, cudaStream_t s);
cudaError_t launch_index_bf16_tc(const void* qI, const float* w, const void* kI, int64_t B, int64_t Q,
                                 int64_t N_c, int d_I, const int64_t* q_pos, int m, float* scores, int* status,
                                 cudaStream_t s, bool pdl);
cudaError_t launch_index_fp4_tc(const void* qI, const float* w, const void* kI, int64_t B, int64_t Q,
                                int64_t N_c, int d_I, const int64_t* q_pos, int m, uint16_t* scores,
                                uint8_t* q_scratch, int* status, cudaStream_t s, bool pdl);
int64_t index_fp4_scratch_bytes(int64_t B, int64_t Q, int d_I);

// topk.cu
int64_t topk_scratch_bytes(int64_t rows, int64_t N_c);
cudaError_t launch_topk(const void* scores, int score_dtype, int64_t B, int64_t Q, int64_t N_c,
                        const int64_t* q_pos, int m, int k, int32_t* idx, void* scratch, int* status,
                        cudaStream_t s, bool pdl);

// attend.cu
struct AttendArgs {
    const void* q;
    const void* comp;
    const void* win;
    int kv_dtype;
    int64_t B, Q, N_c, Tw;
    const int32_t* idx;   // CSA selection or nullptr (HCA)
    int k;
    const int64_t* q_pos;
    const int64_t* win_pos0;
    int m;   // HCA availability stride
    int W, H, D, d_v;
    float scale;
    void* out;
    float* lse;
    int out_dtype;   // LCS_F32 or LCS_BF16
};
int64_t attend_scratch_bytes(const AttendArgs& a);
cudaError_t launch_attend(const AttendArgs& a, void* scratch, int* status, cudaStream_t s, bool pdl);

// cache.cu -- decode-time cache update (one token per request)
cudaError_t launch_cache_append(const int64_t* pos, const void* x, const void* kx, int x_dtype, const float* z,
                                const float* zI, const float* zh, const float* bias, const float* biasI,
                                const float* biash, int D, int d_rope, int d_I, float theta, void* raw,
                                float* logits, void* win, int win_dtype, void* comp, void* kI, void* hca, int64_t B,
                                int64_t N_c, int64_t N_h, int kv_dtype, int kI_dtype, int* status, cudaStream_t s);

// cp.cu -- context parallelism for one long request (entries split over ranks)
cudaError_t launch_cp_candidates(const void* scores, int score_dtype, int64_t B, int64_t S, const int32_t* idx_local,
                                 int k, int64_t offset, float* cand_score, int32_t* cand_idx, cudaStream_t s);
int64_t cp_select_scratch_bytes(int G, int64_t B, int k);
cudaError_t launch_cp_select(const float* cand_score, const int32_t* cand_idx, int G, int64_t B, int k, int64_t offset,
                             int64_t S, int32_t* idx_global, int32_t* idx_local, void* scratch, int* status,
                             cudaStream_t s);
cudaError_t launch_attn_merge(const float* o, const float* lse, int G, int64_t rows, int d_v, void* out, int out_dtype,
                              float* lse_out, cudaStream_t s);

// proj.cu -- compressor and fp32 indexer with their input projections fused in
int compress_proj_tile(int hidden, int d, int m, int overlap);
cudaError_t launch_compress_proj(const void* h, int h_dtype, int64_t B, int64_t T, int hidden, const void* h_tail,
                                 const void* Wx, int d, const float* wz, const float* bias, int m, int overlap,
                                 int d_rope, float theta, int64_t pos0, void* out, int out_dtype, cudaStream_t s);
cudaError_t launch_index_proj_f32(const float* h, int hidden, const float* WqI, const float* Ww, const float* kI,
                                  int64_t B, int64_t Q, int64_t N_c, int H_I, int d_I, const int64_t* q_pos, int m,
                                  float* scores, cudaStream_t s);

// noalloc.cu -- device address of the fixed scratch array behind csa_attend_noalloc
// for the current device (looked up once per device).  LCS_OK or LCS_ERR_CUDA.
int noalloc_scratch(void** ptr);

// Raises a kernel's dynamic shared-memory limit once per process and kernel (the
// attribute call costs host time on every launch otherwise).
cudaError_t set_smem_once(const void* kern, size_t bytes);

// Launch helper with optional programmatic dependent launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                     Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz);
bool encode_tmap_3d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer1,
                    uint64_t outer2, uint64_t row_stride_bytes, uint64_t plane_stride_bytes, uint32_t box_inner,
                    uint32_t box_rows);

// Bounded-wait self-test (selftest.cu): one CTA waits on an mbarrier nothing completes.
cudaError_t launch_selftest_wait(uint64_t budget_ns, int* status, long long* out, cudaStream_t stream);

}  // namespace lcs
