/*
 * veda.h -- C ABI of the B200 (sm_100a) tile-sparse attention library.
 *
 * The library implements the inference hot path of Veda, "Veda: Scalable Video
 * Diffusion via Distilled Sparse Attention" (project page), per head:
 *   1. TripPool tile statistics (avg, max, min of Q and K over each tile);
 *   2. tile scores through head-specific Q/K projections;
 *   3. per query-tile Top-k into a tile mask / index list;
 *   4. tile-skipping attention that reads only the selected K/V tiles.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every pointer is a caller-owned DEVICE pointer, except
 *   `veda_problem::tile_shapes` and the pointers a call names HOST (the host
 *   buffers of veda_forward_host, the candidates of veda_tile_search).  The
 *   library never allocates, frees or keeps a pointer after the call returns.
 *   All work is enqueued asynchronously on `stream`; results are ready when the
 *   stream reaches that point.
 * - Tensors are dense and row-major.  Q, K, V, O are bf16 (passed as uint16_t
 *   bit patterns) of shape [B, H, N, d] with N = T*Hs*Ws tokens in raster
 *   (t, y, x) order: token n = (t*Hs + y)*Ws + x.
 * - Head h uses the tile shape tile_shapes[h] = (p_t, p_h, p_w): tile j is the
 *   p_t x p_h x p_w box of the token grid at tile-grid position
 *   (a, b, c) with j = (a*(Hs/p_h) + b)*(Ws/p_w) + c.  Every head has the same
 *   tile size Bt = p_t*p_h*p_w, so every head has nT = N/Bt tiles.
 * - Supported: d in {64, 128}; Bt in {64, 128}; 1 <= k <= nT; H <= 256; at most
 *   4 distinct tile shapes per call; nT <= 16384.  Other sizes return
 *   VEDA_ERR_UNSUPPORTED before anything is launched.
 * - Device pointers must be 16-byte aligned (VEDA_ERR_ALIGN otherwise).
 * - A call that returns anything but VEDA_OK has launched nothing.
 *   `veda_last_error()` then describes the failure (thread-local string).
 * - Calls that take `ws` use its first VEDA_STATUS_BYTES bytes as a device
 *   status word: they clear it, and a kernel that detects an error (a bounded
 *   wait that gave up, an index-list entry out of range) writes its code there.
 *   `veda_get_status` reads it back.
 */
#ifndef VEDA_H
#define VEDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The CUDA stream type (identical to cudaStream_t / CUstream). */
typedef struct CUstream_st* veda_stream_t;

typedef enum veda_status {
    VEDA_OK = 0,
    VEDA_ERR_INVALID_ARG = 1,  /* null pointer, k out of range, bad scale */
    VEDA_ERR_SHAPE = 2,        /* grid not divisible by a tile shape, tile sizes differ */
    VEDA_ERR_UNSUPPORTED = 3,  /* d, Bt, H, nT or number of distinct shapes out of range */
    VEDA_ERR_ALIGN = 4,        /* a device pointer is not 16-byte aligned */
    VEDA_ERR_CUDA = 5,         /* a CUDA runtime / driver call failed */
    VEDA_ERR_TIMEOUT = 6,      /* device: a bounded wait gave up (read via veda_get_status) */
    VEDA_ERR_BAD_INDEX = 7     /* device: an index-list entry was outside [0, nT) */
} veda_status;

/* Bytes at the start of every workspace that hold the device status word. */
#define VEDA_STATUS_BYTES 256

typedef struct veda_problem {
    int64_t B;                  /* batch */
    int64_t H;                  /* heads */
    int64_t d;                  /* head dimension: 64 or 128 */
    int64_t T, Hs, Ws;          /* latent grid (frames, height, width) */
    const int32_t* tile_shapes; /* HOST pointer, [H][3] = (p_t, p_h, p_w) per head */
    int64_t k;                  /* key tiles kept per query-tile row */
    float scale;                /* softmax scale on q.k; 0 means 1/sqrt(d) */
} veda_problem;

/* Library version, major*10000 + minor*100 + patch. */
int veda_version(void);

/* Message of the last failed call on this host thread ("" if none). */
const char* veda_last_error(void);

/*
 * Workspace bytes needed by veda_forward (a superset of what veda_tile_score
 * and veda_sparse_attn need): status word, TripPool statistics, projected
 * statistics, the score matrix and an index list.
 */
veda_status veda_workspace_size(const veda_problem* p, size_t* bytes);

/*
 * TripPool (project page, "Attention Structure Distillation", Estimator;
 * "Theoretical Rationale" 2, Tile Statistics): per head, tile and channel, the
 * average, maximum and minimum of Q (and of K) over the tile's Bt tokens.
 *   Q, K          : bf16 [B, H, N, d]
 *   statsQ, statsK: fp32 [B, H, nT, 3, d], statistic order (avg, max, min);
 *                   avg is the fp32 sum divided by Bt; max and min are exact.
 */
veda_status veda_tripool(const veda_problem* p, const uint16_t* Q, const uint16_t* K,
                         float* statsQ, float* statsK, veda_stream_t stream);

/*
 * Tile score (project page, "Attention Structure Distillation", Estimator:
 * head-specific Q/K projections of the statistics; "Theoretical Rationale" 4:
 * the estimator's scores over key tiles before Top-k):
 *   q~_{i,s} = statsQ[i,s,:] . Wq[h],  k~_{j,s} = statsK[j,s,:] . Wk[h],
 *   S[i, j]  = sum over s in {avg, max, min} of <q~_{i,s}, k~_{j,s}>.
 *   Wq, Wk: fp32 [H, d, d] (row = input channel, column = output channel)
 *   S     : fp32 [B, H, nT, nT]
 *   ws    : device workspace of at least
 *           VEDA_STATUS_BYTES + 2 * B*H*nT*9*d*4 bytes (projected statistics,
 *           stored as TF32 hi/lo splits).
 * The projection and the score are each a tensor-core product of three TF32
 * terms (hi.hi + hi.lo + lo.hi, fp32 accumulation), within about 3 * 2^-21 of
 * the fp32 product per term.
 */
veda_status veda_tile_score(const veda_problem* p, const float* statsQ, const float* statsK,
                            const float* Wq, const float* Wk, float* S, void* ws,
                            veda_stream_t stream);

/*
 * Head-aware Top-k (project page, "Attention Structure Distillation",
 * Execution): for every query-tile row of S keep the k largest scores; ties go
 * to the lower tile index, -0.0 ties with +0.0 (scores must be finite).
 *   S   : fp32 [B, H, nT, nT]
 *   mask: uint8 [B, H, nT, nT] of 0/1, may be NULL
 *   idx : int32 [B, H, nT, k], the kept tile indices in ascending order
 */
veda_status veda_topk_mask(const veda_problem* p, const float* S, uint8_t* mask, int32_t* idx,
                           veda_stream_t stream);

/*
 * fp8 estimator weights (news page "Veda from ByteDance, HKU and USTC: an open
 * method that speeds up video generation fivefold", "Why this matters for
 * users": the predictor is distributed in fp8).  Encoding: OCP FP8 E4M3, one
 * scale per head:
 *   scale[h] = max |W[h]| / 448 (fp32; 1 for an all-zero head),
 *   W8[h]    = E4M3(W[h] / scale[h]), round to nearest even, saturating at +-448.
 *   W    : fp32 [H, d, d] (device)      W8: uint8 [H, d, d]      scale: fp32 [H]
 * veda_dequantize_fp8 writes the fp32 weights fp32(E4M3(W8) * scale[h]), which
 * veda_tile_score / veda_mask_fused / veda_forward take as Wq, Wk.
 * Errors: VEDA_ERR_INVALID_ARG (H outside 1..2^20, d outside 1..4096, or a NULL
 * pointer), VEDA_ERR_ALIGN (a pointer not 16-byte aligned).
 */
veda_status veda_quantize_fp8(const float* W, int64_t H, int64_t d, uint8_t* W8, float* scale,
                              veda_stream_t stream);
veda_status veda_dequantize_fp8(const uint8_t* W8, const float* scale, int64_t H, int64_t d,
                                float* W, veda_stream_t stream);

/*
 * Fused tile score + head-aware Top-k (project page, "Attention Structure
 * Distillation", Estimator and Execution): the same projection, score and
 * selection as veda_tile_score followed by veda_topk_mask, with the score
 * matrix S held on chip (never written to memory).  Results are identical to
 * the two-call path (the scores are computed by the same products in the same
 * order).
 *   statsQ, statsK, Wq, Wk: as for veda_tile_score
 *   mask: uint8 [B, H, nT, nT] of 0/1, may be NULL
 *   idx : int32 [B, H, nT, k], the kept tile indices in ascending order
 *   ws  : device workspace of at least VEDA_STATUS_BYTES + 2 * B*H*nT*9*d*4
 *         bytes (the projected statistics); veda_workspace_size() is enough.
 * Limits: k <= 128 and nT <= 6144, else VEDA_ERR_UNSUPPORTED (use the two-call
 * path).  A device-side wait that gives up is reported through
 * veda_get_status(ws) as VEDA_ERR_TIMEOUT.
 */
veda_status veda_mask_fused(const veda_problem* p, const float* statsQ, const float* statsK,
                            const float* Wq, const float* Wk, uint8_t* mask, int32_t* idx,
                            void* ws, veda_stream_t stream);

/*
 * Tile-skipping attention (project page, "Attention Structure Distillation",
 * Execution and "Principle 03 Tile-Sparse Kernel"; "Theoretical Rationale" 1:
 * the kept keys are renormalised among themselves).  For every query token of
 * tile i of head h:
 *   O   = softmax(scale * q.k over every key of the tiles idx[b,h,i,:]) . V
 *   lse = ln sum exp(scale * q.k) over the same keys
 *   idx: int32 [B, H, nT, k] tile indices in [0, nT) (each row's entries should
 *        be distinct; order does not matter), or NULL for the dense schedule
 *        (every tile, k taken as nT).
 *   O  : bf16 [B, H, N, d];  lse: fp32 [B, H, N] or NULL
 *   ws : device workspace of at least VEDA_STATUS_BYTES bytes
 * bf16 tensor-core products with fp32 accumulation and an fp32 softmax; P is
 * rounded to bf16 before the P.V product.  An out-of-range index is replaced
 * by tile 0 and reported as VEDA_ERR_BAD_INDEX in the status word.  With the
 * environment variable VEDA_DEBUG_CHECKS set (not "0"), every row is checked
 * on the device first and a row with an out-of-range or repeated entry is
 * also reported as VEDA_ERR_BAD_INDEX (a repeated tile would otherwise be
 * counted twice).
 */
veda_status veda_sparse_attn(const veda_problem* p, const uint16_t* Q, const uint16_t* K,
                             const uint16_t* V, const int32_t* idx, uint16_t* O, float* lse,
                             void* ws, veda_stream_t stream);

/*
 * The whole layer: TripPool -> projection and score -> Top-k -> tile-skipping
 * attention, all on `stream`.
 *   idx_out : int32 [B, H, nT, k] or NULL (then held in ws)
 *   mask_out: uint8 [B, H, nT, nT] or NULL
 *   lse     : fp32 [B, H, N] or NULL
 *   ws      : at least veda_workspace_size() bytes
 */
veda_status veda_forward(const veda_problem* p, const uint16_t* Q, const uint16_t* K,
                         const uint16_t* V, const float* Wq, const float* Wk, uint16_t* O,
                         float* lse, int32_t* idx_out, uint8_t* mask_out, void* ws,
                         veda_stream_t stream);

/*
 * The whole layer from HOST memory, pipelined over chunks of heads (every step
 * of the layer is independent per batch entry and head): chunk g+1 is copied
 * in on an internal copy stream while chunk g runs veda_forward's kernels on
 * `stream`, and chunk g-1's O is copied out on a second copy stream.  Results
 * equal one veda_forward call on the whole problem.
 *   hQ, hK, hV: host bf16 [B, H, N, d]      hWq, hWk: host fp32 [H, d, d]
 *   hO        : host bf16 [B, H, N, d]      hlse: host fp32 [B, H, N] or NULL
 *   dQ, dK, dV, dO: device bf16 [B, H, N, d] staging (owned by the caller)
 *   dWq, dWk  : device fp32 [H, d, d] staging
 *   dlse      : device fp32 [B, H, N] staging, needed when hlse is not NULL
 *   ws        : at least veda_workspace_size() bytes
 *   head_chunk: heads per chunk, 1..H (0 picks 1)
 * Host buffers should be page-locked (cudaHostAlloc / pinned) for the copies
 * to overlap the kernels; with pageable memory the copies are synchronous.
 * When `stream` completes, hO (and hlse) hold the results.  The status word in
 * ws covers every chunk (veda_get_status).
 * Exception to the rule that a failed call has launched nothing: an error met
 * after the first chunk's copies were queued (a CUDA call failing mid-way) is
 * returned after `stream` has been made to wait for every copy already queued
 * (or, if that fails too, after those copies finished), so once `stream`
 * completes no copy of this call reads or writes the host buffers; the earlier
 * chunks' kernels and copies may have run.
 */
veda_status veda_forward_host(const veda_problem* p, const uint16_t* hQ, const uint16_t* hK,
                              const uint16_t* hV, const float* hWq, const float* hWk,
                              uint16_t* hO, float* hlse, uint16_t* dQ, uint16_t* dK, uint16_t* dV,
                              float* dWq, float* dWk, uint16_t* dO, float* dlse, void* ws,
                              int32_t head_chunk, veda_stream_t stream);

/*
 * Head-aware tile search (project page, "Head-Aware Tile Search"; "Principle
 * 02 Head-Conditioned Tile Geometry"): for each head, the candidate tiling pi
 * (p_t, p_h, p_w with the same product) that minimises
 * ||O_full - O_sparse(pi)||_F^2 over the calibration batch.
 *   p->tile_shapes is ignored; candidates: HOST int32 [ncand][3], 1 <= ncand <= 16,
 *   each valid for the grid, all with the same p_t*p_h*p_w.
 *   O_dense: bf16 [B, H, N, d], the full attention (dense schedule)
 *   O_cand : bf16 [B, H, N, d] scratch (the layer output of the last candidate)
 *   err    : fp64 [ncand, B, H], sum over tokens and channels of (O_dense - O_cand)^2
 *   best   : int32 [H], argmin over candidates of the sum over B of err (ties: lower index)
 *   ws     : at least veda_workspace_size() bytes (of `p` with any candidate)
 * Each candidate runs the whole layer (veda_forward) on every head.
 */
veda_status veda_tile_search(const veda_problem* p, const int32_t* candidates, int32_t ncand,
                             const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                             const float* Wq, const float* Wk, uint16_t* O_dense,
                             uint16_t* O_cand, double* err, int32_t* best, void* ws,
                             veda_stream_t stream);

/*
 * Max-pooled full-attention teacher (project page, "Attention Structure
 * Distillation", Teacher; "Empirical Study" 02, Controlled Mask Intervention):
 *   teacher[b,h,i,j] = max over query tokens q of tile i and key tokens of
 *                      tile j of P[q, key],  P = softmax(scale * q.k) over all N keys.
 * Runs the dense attention schedule (every key tile) first, which also yields
 *   O_dense  : bf16 [B, H, N, d], dense attention output
 *   lse_dense: fp32 [B, H, N], ln of each row's softmax normaliser
 * and then one Q K^T pass per tile pair that max-pools exp(scale*s - lse).
 *   teacher: fp32 [B, H, nT, nT] (k is not used)
 *   ws     : at least VEDA_STATUS_BYTES bytes
 * The oracle mask of the page is veda_topk_mask applied to `teacher`.
 */
veda_status veda_teacher(const veda_problem* p, const uint16_t* Q, const uint16_t* K,
                         const uint16_t* V, uint16_t* O_dense, float* lse_dense, float* teacher,
                         void* ws, veda_stream_t stream);

/*
 * Tile recall (project page, "Empirical Study" 02): the fraction of the
 * reference mask's tiles that a predicted mask also selects.
 *   idx_pred, idx_ref: int32 [B, H, nT, k], each row ascending and duplicate-free
 *   recall_rows: fp32 [B, H, nT] per-row recall, or NULL
 *   recall_mean: one fp64 on the device, hits / (B*H*nT*k)
 *   ws         : at least VEDA_STATUS_BYTES bytes (holds the hit counter)
 * Integer counting: exact and deterministic.
 */
veda_status veda_tile_recall(const veda_problem* p, const int32_t* idx_pred,
                             const int32_t* idx_ref, float* recall_rows, double* recall_mean,
                             void* ws, veda_stream_t stream);

/*
 * KL structure distillation of the estimator (project page, "Principle 01
 * Full-Attention Structure Distillation"; "Theoretical Rationale" 4,
 * Distillation Objective: row-wise KL between the max-pooled teacher's tile
 * distribution and the estimator's soft distribution over key tiles, before
 * Top-k).  With R = B*H*nT rows:
 *   A_tgt[i,:]  = teacher[i,:] / sum_j teacher[i,j]
 *   A_pred[i,:] = softmax(S[i,:] / tau)
 *   loss        = (1/R) sum_i KL(A_tgt[i] || A_pred[i])            (fp64, device)
 *   dWq, dWk    = d loss / d Wq, d loss / d Wk  (fp32 [H, d, d]) through
 *                 S = sum_s (statsQ_s Wq) . (statsK_s Wk)
 *   S must be the score of (statsQ, statsK, Wq, Wk) (veda_tile_score);
 *   teacher: fp32 [B, H, nT, nT], rows with a positive sum (veda_teacher).
 *   tau > 0; nT must be a multiple of 8.
 *   ws: at least veda_distill_workspace_size() bytes.
 * fp32 arithmetic with fp64 row sums; the loss is reduced in a fixed order.
 */
veda_status veda_distill_workspace_size(const veda_problem* p, size_t* bytes);
veda_status veda_distill_kl(const veda_problem* p, const float* statsQ, const float* statsK,
                            const float* Wq, const float* Wk, const float* S, const float* teacher,
                            float tau, double* loss, float* dWq, float* dWk, void* ws,
                            veda_stream_t stream);

/*
 * Waits for `stream`, then copies the device status word of `ws` into
 * *device_status (VEDA_OK or a device-detected veda_status code).
 */
veda_status veda_get_status(const void* ws, veda_stream_t stream, int32_t* device_status);

/*
 * The paper has no counterpart for the calls below; they exist for
 * callers that cannot allocate device memory (an application that only
 * receives device pointers for its inputs and outputs from another runtime, a
 * plugin whose host forbids allocations after start-up, a real-time loop that
 * must not call cudaMalloc because it can synchronise the device).
 *
 * veda_tile_score_noalloc computes exactly what veda_tile_score computes, but
 * keeps its scratch (status word and projected statistics) in a fixed device
 * array inside the library instead of a caller workspace:
 *   - the array holds veda_noalloc_scratch_bytes() bytes (64 MiB); every GPU
 *     that loads the library keeps it until the process exits;
 *   - a problem needing more than VEDA_STATUS_BYTES + 2*B*H*nT*9*d*4 bytes of
 *     it returns VEDA_ERR_UNSUPPORTED and launches nothing;
 *   - the first call on a device looks up the array's address on that device
 *     (the device must be current); make that first call before any stream
 *     capture;
 *   - all calls share the array: calls whose work overlaps on the GPU race;
 *     each call clears the status word it uses;
 *   - it allocates nothing (no cudaMalloc, no cudaFree).
 */
size_t veda_noalloc_scratch_bytes(void);
veda_status veda_tile_score_noalloc(const veda_problem* p, const float* statsQ,
                                    const float* statsK, const float* Wq, const float* Wk,
                                    float* S, veda_stream_t stream);

/*
 * No counterpart in the paper either.  Waits for `stream`, then copies the
 * status word that the last veda_tile_score_noalloc call on the current device
 * left in the fixed array into *device_status: VEDA_OK, or VEDA_ERR_TIMEOUT if
 * a bounded wait of the score kernel gave up (that call's S is then
 * incomplete).  The same race as above applies: a later or overlapping call
 * clears and reuses the word.  VEDA_ERR_INVALID_ARG if device_status is NULL.
 */
veda_status veda_noalloc_get_status(veda_stream_t stream, int32_t* device_status);

#ifdef __cplusplus
}
#endif

#endif /* VEDA_H */
