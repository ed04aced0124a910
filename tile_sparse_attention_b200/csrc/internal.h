// internal.h -- shared host-side declarations of the library (not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "../../include/veda.h"

namespace veda {

constexpr int kMaxHeads = 256;
constexpr int kMaxShapes = 4;
constexpr int64_t kMaxTiles = 16384;

// Validated view of a veda_problem.
struct Problem {
    int B, H, d, T, Hs, Ws, N, Bt, nT, k;
    float scale;
    int nshapes;                  // distinct tile shapes
    int shape[kMaxShapes][3];     // (p_t, p_h, p_w) per distinct shape
    int head_shape[kMaxHeads];    // head -> distinct-shape slot
};

// Records a message for veda_last_error() and returns `code`.
veda_status fail(veda_status code, const std::string& msg);

// Validates `p` (k is checked only when need_k).
veda_status make_problem(const veda_problem* p, bool need_k, Problem* out);

veda_status check_ptr(const void* ptr, const char* name, bool nullable = false);

veda_status cuda_check(cudaError_t err, const char* what);
// SMs of the current device (1 if the query fails).
int sm_count();
// VEDA_DEBUG_CHECKS set (and not "0"): index lists passed to veda_sparse_attn
// are validated on the device first (index_check.cu).
bool debug_checks_enabled();
// Reports any row of idx [rows, k] with an entry outside [0, nT) or a repeated
// entry as VEDA_ERR_BAD_INDEX in *status (index_check.cu).
veda_status launch_check_index(const int32_t* idx, long long rows, int k, int nT, int* status,
                               cudaStream_t s);

// Launchers (defined next to their kernels).  Each returns VEDA_OK or an
// error after checking the launch.
veda_status launch_tripool(const Problem& pr, const uint16_t* Q, const uint16_t* K, float* statsQ,
                           float* statsK, cudaStream_t s);
// Both projections in one launch on the tensor cores (proj_tc.cu): statsQ . Wq
// into qt and statsK . Wk into kt, in the TF32-split score operand layout
// [B*H*nT][9d] (query side [hi|hi|lo], key side [hi|lo|hi] per statistic);
// status: device status word.
veda_status launch_project_pair(const Problem& pr, const float* statsQ, const float* statsK,
                                const float* Wq, const float* Wk, float* qt, float* kt,
                                int* status, cudaStream_t s);
// S = q^ k^^T on the tensor cores (score_tc.cu); status: device status word.
veda_status launch_score(const Problem& pr, const float* qext, const float* kext, float* S,
                         int* status, cudaStream_t s);
// Bytes of one projected-statistics operand: B*H*nT*9d fp32.
inline size_t projected_bytes(const Problem& pr) {
    return (size_t)pr.B * pr.H * pr.nT * 9 * pr.d * sizeof(float);
}
// fp8 (E4M3) weights, one scale per head: W [H][n] fp32 <-> codes [H][n], scale [H].
veda_status launch_quantize_e4m3(const float* W, int H, long long n, uint8_t* codes, float* scale,
                                 cudaStream_t s);
veda_status launch_dequantize_e4m3(const uint8_t* codes, const float* scale, int H, long long n,
                                   float* W, cudaStream_t s);
// Fused score + Top-k (S stays on chip); needs k <= 128 and nT <= 6144.
bool fused_mask_supported(const Problem& pr);
veda_status launch_score_topk(const Problem& pr, const float* qext, const float* kext,
                              uint8_t* mask, int32_t* idx, int* status, cudaStream_t s);
veda_status launch_topk(const Problem& pr, const float* S, uint8_t* mask, int32_t* idx,
                        cudaStream_t s);
veda_status launch_sparse_attn(const Problem& pr, const uint16_t* Q, const uint16_t* K,
                               const uint16_t* V, const int32_t* idx, int k, uint16_t* O,
                               float* lse, int* status, cudaStream_t s);
// The persistent-CTA kernel for short key lists (launch_sparse_attn uses it
// for k <= kPersistentMaxK).
constexpr int kPersistentMaxK = 64;
veda_status launch_sparse_attn_persistent(const Problem& pr, const uint16_t* Q,
                                          const uint16_t* K, const uint16_t* V,
                                          const int32_t* idx, int k, uint16_t* O, float* lse,
                                          int* status, cudaStream_t s);

// One query tile per CTA, two softmax groups on alternate 64-key chunks
// (sparse_attn_dual.cu): d = 128 and 128-token tiles, k >= kDualMinK.
constexpr int kDualMinK = 8;
bool dual_attn_supported(const Problem& pr);
veda_status launch_sparse_attn_dual(const Problem& pr, const uint16_t* Q, const uint16_t* K,
                                    const uint16_t* V, const int32_t* idx, int k, uint16_t* O,
                                    float* lse, int* status, cudaStream_t s);

// TMA descriptors (tensor_maps.cu): the 5-D tile view (d, Ws, Hs, T, B*H) of a
// [B,H,N,d] bf16 tensor with a (64, p_w, p_h, p_t, 1) box, and a 2-D row view
// of an fp32 [rows][cols] matrix with a (32, 128) box; both 128-byte swizzled.
veda_status encode_tile_map(CUtensorMap* map, const void* base, const Problem& pr,
                            const int* shape);
// The same tile view for d = 128 with both 64-channel chunks in one box:
// dims (64, Ws, Hs, T*B*H, 2), box (64, p_w, p_h, p_t, 2) -> two 128-row planes.
veda_status encode_tile_map_2c(CUtensorMap* map, const void* base, const Problem& pr,
                               const int* shape);
veda_status encode_rows_map(CUtensorMap* map, const float* base, long long rows, int cols,
                            int box_rows = 128);
// Time limit of a device wait (VEDA_WAIT_LIMIT_MS, default 10 s).
unsigned long long wait_limit_ns();

// Batched fp32 SIMT GEMM (sgemm.cu): C[z] (+)= op(A[z']) . op(B[z''])
// with z' = z % a_batch_mod, z'' = z % b_batch_mod (when > 0); a_t: A stored
// K x M; b_t: B stored N x K.  K must be a multiple of 8.
veda_status launch_sgemm(const float* A, const float* B, float* C, int M, int N, int K, int lda,
                         int ldb, int ldc, long long strideA, long long strideB, long long strideC,
                         int batches, int a_batch_mod, int b_batch_mod, bool a_t, bool b_t,
                         bool accumulate, cudaStream_t s);

// Max-pooled teacher (teacher.cu): T [B,H,nT,nT] from Q, K and the dense lse.
veda_status launch_teacher(const Problem& pr, const uint16_t* Q, const uint16_t* K,
                           const float* lse, float* teacher, int* status, cudaStream_t s);
// Tile recall of idx_pred against idx_ref (both [B,H,nT,k], ascending rows);
// scratch8: 8 bytes of device scratch for the hit counter.
veda_status launch_recall(const Problem& pr, const int32_t* idx_pred, const int32_t* idx_ref,
                          float* per_row, double* mean, void* scratch8, cudaStream_t s);

// KL structure distillation (distill.cu).
struct DistillLayout {
    size_t qt, kt, dq, dk, G, row_kl, total;
};
DistillLayout distill_layout(const Problem& pr);
veda_status launch_distill(const Problem& pr, const float* statsQ, const float* statsK,
                           const float* Wq, const float* Wk, const float* S, const float* teacher,
                           float tau, double* loss, float* dWq, float* dWk, void* ws,
                           cudaStream_t s);

// Head-aware tile search helpers (tile_search.cu).
veda_status launch_sq_err(const uint16_t* a, const uint16_t* b, int heads, long long per_head,
                          double* err, cudaStream_t s);
veda_status launch_argmin(const double* err, int ncand, int B, int H, int32_t* best,
                          cudaStream_t s);
// The whole layer on a validated problem (veda_api.cu).
veda_status forward_impl(const Problem& pr, const uint16_t* Q, const uint16_t* K,
                         const uint16_t* V, const float* Wq, const float* Wk, uint16_t* O,
                         float* lse, int32_t* idx_out, uint8_t* mask_out, void* ws,
                         cudaStream_t s);

// veda_forward on host buffers, pipelined over chunks of head_chunk heads.
veda_status forward_host_impl(const veda_problem* p, const Problem& pr, const uint16_t* hQ,
                              const uint16_t* hK, const uint16_t* hV, const float* hWq,
                              const float* hWk, uint16_t* hO, float* hlse, uint16_t* dQ,
                              uint16_t* dK, uint16_t* dV, float* dWq, float* dWk, uint16_t* dO,
                              float* dlse, void* ws, int head_chunk, cudaStream_t s);

// Workspace layout of veda_forward (byte offsets, 256-aligned).
struct WorkspaceLayout {
    size_t status, statsQ, statsK, qt, kt, S, idx, total;
};
WorkspaceLayout workspace_layout(const Problem& pr);

}  // namespace veda
