// veda_api.cu -- the C ABI (include/veda.h): argument validation, workspace
// layout and the composition of the four kernels into the layer call.
//
// "Veda: Scalable Video Diffusion via Distilled Sparse Attention" (project
// page), "Attention Structure Distillation": TripPool and the head-specific
// projections (Estimator) feed a head-aware Top-k whose tile mask drives the
// tile-skipping kernel (Execution).
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <string>

#include "internal.h"

namespace veda {

namespace {
thread_local std::string g_last_error;
}

veda_status fail(veda_status code, const std::string& msg) {
    g_last_error = msg;
    return code;
}

veda_status cuda_check(cudaError_t err, const char* what) {
    if (err == cudaSuccess) return VEDA_OK;
    return fail(VEDA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(err));
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
        return 1;
    return n;
}

veda_status check_ptr(const void* ptr, const char* name, bool nullable) {
    if (ptr == nullptr) {
        if (nullable) return VEDA_OK;
        return fail(VEDA_ERR_INVALID_ARG, std::string(name) + " is NULL");
    }
    if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0)
        return fail(VEDA_ERR_ALIGN, std::string(name) + " is not 16-byte aligned");
    return VEDA_OK;
}

veda_status make_problem(const veda_problem* p, bool need_k, Problem* out) {
    if (p == nullptr) return fail(VEDA_ERR_INVALID_ARG, "problem is NULL");
    if (p->tile_shapes == nullptr) return fail(VEDA_ERR_INVALID_ARG, "tile_shapes is NULL");
    if (p->B < 1 || p->H < 1 || p->T < 1 || p->Hs < 1 || p->Ws < 1)
        return fail(VEDA_ERR_INVALID_ARG, "B, H, T, Hs and Ws must be >= 1");
    if (p->d != 64 && p->d != 128) return fail(VEDA_ERR_UNSUPPORTED, "d must be 64 or 128");
    if (p->H > kMaxHeads) return fail(VEDA_ERR_UNSUPPORTED, "at most 256 heads");
    const int64_t N = p->T * p->Hs * p->Ws;
    if (N > (1ll << 30) || p->B * p->H > 65535)
        return fail(VEDA_ERR_UNSUPPORTED, "token count or B*H too large");
    Problem& pr = *out;
    memset(&pr, 0, sizeof(pr));
    pr.B = (int)p->B;
    pr.H = (int)p->H;
    pr.d = (int)p->d;
    pr.T = (int)p->T;
    pr.Hs = (int)p->Hs;
    pr.Ws = (int)p->Ws;
    pr.N = (int)N;
    pr.nshapes = 0;
    int Bt = -1;
    for (int h = 0; h < pr.H; ++h) {
        const int32_t* s = p->tile_shapes + 3 * h;
        if (s[0] < 1 || s[1] < 1 || s[2] < 1)
            return fail(VEDA_ERR_SHAPE, "tile shape entries must be >= 1");
        if (p->T % s[0] || p->Hs % s[1] || p->Ws % s[2])
            return fail(VEDA_ERR_SHAPE, "grid not divisible by the tile shape of head " +
                                            std::to_string(h));
        const int bt = s[0] * s[1] * s[2];
        if (Bt < 0) Bt = bt;
        if (bt != Bt) return fail(VEDA_ERR_SHAPE, "tile sizes p_t*p_h*p_w differ between heads");
        int slot = -1;
        for (int q = 0; q < pr.nshapes; ++q)
            if (pr.shape[q][0] == s[0] && pr.shape[q][1] == s[1] && pr.shape[q][2] == s[2]) slot = q;
        if (slot < 0) {
            if (pr.nshapes == kMaxShapes)
                return fail(VEDA_ERR_UNSUPPORTED, "more than 4 distinct tile shapes");
            slot = pr.nshapes++;
            pr.shape[slot][0] = s[0];
            pr.shape[slot][1] = s[1];
            pr.shape[slot][2] = s[2];
        }
        pr.head_shape[h] = slot;
    }
    if (Bt != 64 && Bt != 128) return fail(VEDA_ERR_UNSUPPORTED, "tile size must be 64 or 128");
    pr.Bt = Bt;
    pr.nT = pr.N / Bt;
    if (pr.nT > kMaxTiles) return fail(VEDA_ERR_UNSUPPORTED, "more than 16384 tiles per head");
    if (need_k && (p->k < 1 || p->k > pr.nT))
        return fail(VEDA_ERR_INVALID_ARG, "k must be in [1, nT]");
    pr.k = (int)p->k;
    float scale = p->scale;
    if (scale == 0.f) scale = 1.0f / sqrtf((float)pr.d);
    if (!(scale > 0.f) || !isfinite(scale))
        return fail(VEDA_ERR_INVALID_ARG, "scale must be positive and finite (0 = 1/sqrt(d))");
    pr.scale = scale;
    return VEDA_OK;
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

WorkspaceLayout workspace_layout(const Problem& pr) {
    WorkspaceLayout w{};
    const size_t stats = (size_t)pr.B * pr.H * pr.nT * 3 * pr.d * sizeof(float);
    const size_t proj = projected_bytes(pr);
    size_t off = 0;
    w.status = off;
    off += VEDA_STATUS_BYTES;
    w.qt = off;  // tile_score's own workspace follows the status word
    off = align256(off + proj);
    w.kt = off;
    off = align256(off + proj);
    w.statsQ = off;
    off = align256(off + stats);
    w.statsK = off;
    off = align256(off + stats);
    w.S = off;
    off = align256(off + (size_t)pr.B * pr.H * pr.nT * pr.nT * sizeof(float));
    w.idx = off;
    off = align256(off + (size_t)pr.B * pr.H * pr.nT * pr.k * sizeof(int32_t));
    w.total = off;
    return w;
}

// The layer on an already validated problem; the status word in ws is not cleared.
veda_status forward_impl(const Problem& pr, const uint16_t* Q, const uint16_t* K,
                         const uint16_t* V, const float* Wq, const float* Wk, uint16_t* O,
                         float* lse, int32_t* idx_out, uint8_t* mask_out, void* ws,
                         cudaStream_t s) {
    const WorkspaceLayout w = workspace_layout(pr);
    char* base = static_cast<char*>(ws);
    int* status = reinterpret_cast<int*>(base + w.status);
    float* statsQ = reinterpret_cast<float*>(base + w.statsQ);
    float* statsK = reinterpret_cast<float*>(base + w.statsK);
    float* qt = reinterpret_cast<float*>(base + w.qt);
    float* kt = reinterpret_cast<float*>(base + w.kt);
    float* S = reinterpret_cast<float*>(base + w.S);
    int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(base + w.idx);
    veda_status st;
    if ((st = launch_tripool(pr, Q, K, statsQ, statsK, s))) return st;
    if ((st = launch_project_pair(pr, statsQ, statsK, Wq, Wk, qt, kt, status, s))) return st;
    if ((st = launch_score(pr, qt, kt, S, status, s))) return st;
    if ((st = launch_topk(pr, S, mask_out, idx, s))) return st;
    return launch_sparse_attn(pr, Q, K, V, idx, pr.k, O, lse, status, s);
}

}  // namespace veda

using namespace veda;

extern "C" {

int veda_version(void) { return 10000; }

const char* veda_last_error(void) { return g_last_error.c_str(); }

veda_status veda_workspace_size(const veda_problem* p, size_t* bytes) {
    Problem pr;
    veda_status st = make_problem(p, true, &pr);
    if (st != VEDA_OK) return st;
    if (bytes == nullptr) return fail(VEDA_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = workspace_layout(pr).total;
    return VEDA_OK;
}

veda_status veda_tripool(const veda_problem* p, const uint16_t* Q, const uint16_t* K,
                         float* statsQ, float* statsK, veda_stream_t stream) {
    Problem pr;
    veda_status st;
    if ((st = make_problem(p, false, &pr)) != VEDA_OK) return st;
    if ((st = check_ptr(Q, "Q")) || (st = check_ptr(K, "K")) || (st = check_ptr(statsQ, "statsQ")) ||
        (st = check_ptr(statsK, "statsK")))
        return st;
    return launch_tripool(pr, Q, K, statsQ, statsK, (cudaStream_t)stream);
}

veda_status veda_tile_score(const veda_problem* p, const float* statsQ, const float* statsK,
                            const float* Wq, const float* Wk, float* S, void* ws,
                            veda_stream_t stream) {
    Problem pr;
    veda_status st;
    if ((st = make_problem(p, false, &pr)) != VEDA_OK) return st;
    if ((st = check_ptr(statsQ, "statsQ")) || (st = check_ptr(statsK, "statsK")) ||
        (st = check_ptr(Wq, "Wq")) || (st = check_ptr(Wk, "Wk")) || (st = check_ptr(S, "S")) ||
        (st = check_ptr(ws, "ws")))
        return st;
    cudaStream_t s = (cudaStream_t)stream;
    const WorkspaceLayout w = workspace_layout(pr);
    char* base = static_cast<char*>(ws);
    float* qt = reinterpret_cast<float*>(base + w.qt);
    float* kt = reinterpret_cast<float*>(base + w.kt);
    if ((st = cuda_check(cudaMemsetAsync(base + w.status, 0, sizeof(int), s), "status reset")))
        return st;
    int* status = reinterpret_cast<int*>(base + w.status);
    if ((st = launch_project_pair(pr, statsQ, statsK, Wq, Wk, qt, kt, status, s))) return st;
    return launch_score(pr, qt, kt, S, status, s);
}

veda_status veda_topk_mask(const veda_problem* p, const float* S, uint8_t* mask, int32_t* idx,
                           veda_stream_t stream) {
    Problem pr;
    veda_status st;
    if ((st = make_problem(p, true, &pr)) != VEDA_OK) return st;
    if ((st = check_ptr(S, "S")) || (st = check_ptr(idx, "idx")) ||
        (st = check_ptr(mask, "mask", true)))
        return st;
    return launch_topk(pr, S, mask, idx, (cudaStream_t)stream);
}

veda_status veda_quantize_fp8(const float* W, int64_t H, int64_t d, uint8_t* W8, float* scale,
                              veda_stream_t stream) {
    if (H < 1 || d < 1 || H > (1 << 20) || d > 4096)
        return fail(VEDA_ERR_INVALID_ARG, "fp8 weights: 1 <= H <= 2^20, 1 <= d <= 4096");
    veda_status st;
    if ((st = check_ptr(W, "W")) || (st = check_ptr(W8, "W8")) || (st = check_ptr(scale, "scale")))
        return st;
    return launch_quantize_e4m3(W, (int)H, (long long)d * d, W8, scale, (cudaStream_t)stream);
}

veda_status veda_dequantize_fp8(const uint8_t* W8, const float* scale, int64_t H, int64_t d,
                                float* W, veda_stream_t stream) {
    if (H < 1 || d < 1 || H > (1 << 20) || d > 4096)
        return fail(VEDA_ERR_INVALID_ARG, "fp8 weights: 1 <= H <= 2^20, 1 <= d <= 4096");
    veda_status st;
    if ((st = check_ptr(W8, "W8")) || (st = check_ptr(scale, "scale")) || (st = check_ptr(W, "W")))
        return st;
    return launch_dequantize_e4m3(W8, scale, (int)H, (long long)d * d, W, (cudaStream_t)stream);
}

veda_status veda_mask_fused(const veda_problem* p, const float* statsQ, const float* statsK,
                            const float* Wq, const float* Wk, uint8_t* mask, int32_t* idx,
                            void* ws, veda_stream_t stream) {
    Problem pr;
    veda_status st;
    if ((st = make_problem(p, true, &pr)) != VEDA_OK) return st;
    if ((st = check_ptr(statsQ, "statsQ")) || (st = check_ptr(statsK, "statsK")) ||
        (st = check_ptr(Wq, "Wq")) || (st = check_ptr(Wk, "Wk")) || (st = check_ptr(idx, "idx")) ||
        (st = check_ptr(mask, "mask", true)) || (st = check_ptr(ws, "ws")))
        return st;
    if (!fused_mask_supported(pr))
        return fail(VEDA_ERR_UNSUPPORTED, "fused mask: needs k <= 128 and nT <= 6144");
    cudaStream_t s = (cudaStream_t)stream;
    const WorkspaceLayout w = workspace_layout(pr);
    char* base = static_cast<char*>(ws);
    float* qt = reinterpret_cast<float*>(base + w.qt);
    float* kt = reinterpret_cast<float*>(base + w.kt);
    int* status = reinterpret_cast<int*>(base + w.status);
    if ((st = cuda_check(cudaMemsetAsync(status, 0, sizeof(int), s), "status reset"))) return st;
    if ((st = launch_project_pair(pr, statsQ, statsK, Wq, Wk, qt, kt, status, s))) return st;
    return launch_score_topk(pr, qt, kt, mask, idx, status, s);
}

veda_status veda_sparse_attn(const veda_problem* p, const uint16_t* Q, const uint16_t* K,
                             const uint16_t* V, const int32_t* idx, uint16_t* O, float* lse,
                             void* ws, veda_stream_t stream) {
    Problem pr;
    veda_status st;
    if ((st = make_problem(p, idx != nullptr, &pr)) != VEDA_OK) return st;
    if ((st = check_ptr(Q, "Q")) || (st = check_ptr(K, "K")) || (st = check_ptr(V, "V")) ||
        (st = check_ptr(O, "O")) || (st = check_ptr(idx, "idx", true)) ||
        (st = check_ptr(lse, "lse", true)) || (st = check_ptr(ws, "ws")))
        return st;
    cudaStream_t s = (cudaStream_t)stream;
    int* status = static_cast<int*>(ws);
    if ((st = cuda_check(cudaMemsetAsync(status, 0, sizeof(int), s), "status reset"))) return st;
    const int k = idx ? pr.k : pr.nT;
    if (idx != nullptr && debug_checks_enabled() &&
        (st = launch_check_index(idx, (long long)pr.B * pr.H * pr.nT, k, pr.nT, status, s)))
        return st;
    return launch_sparse_attn(pr, Q, K, V, idx, k, O, lse, status, s);
}

veda_status veda_forward(const veda_problem* p, const uint16_t* Q, const uint16_t* K,
                         const uint16_t* V, const float* Wq, const float* Wk, uint16_t* O,
                         float* lse, int32_t* idx_out, uint8_t* mask_out, void* ws,
                         veda_stream_t stream) {
    Problem pr;
    veda_status st;
    if ((st = make_problem(p, true, &pr)) != VEDA_OK) return st;
    if ((st = check_ptr(Q, "Q")) || (st = check_ptr(K, "K")) || (st = check_ptr(V, "V")) ||
        (st = check_ptr(Wq, "Wq")) || (st = check_ptr(Wk, "Wk")) || (st = check_ptr(O, "O")) ||
        (st = check_ptr(lse, "lse", true)) || (st = check_ptr(idx_out, "idx_out", true)) ||
        (st = check_ptr(mask_out, "mask_out", true)) || (st = check_ptr(ws, "ws")))
        return st;
    cudaStream_t s = (cudaStream_t)stream;
    if ((st = cuda_check(cudaMemsetAsync(ws, 0, sizeof(int), s), "status reset"))) return st;
    return forward_impl(pr, Q, K, V, Wq, Wk, O, lse, idx_out, mask_out, ws, s);
}

veda_status veda_forward_host(const veda_problem* p, const uint16_t* hQ, const uint16_t* hK,
                              const uint16_t* hV, const float* hWq, const float* hWk,
                              uint16_t* hO, float* hlse, uint16_t* dQ, uint16_t* dK, uint16_t* dV,
                              float* dWq, float* dWk, uint16_t* dO, float* dlse, void* ws,
                              int32_t head_chunk, veda_stream_t stream) {
    Problem pr;
    veda_status st;
    if ((st = make_problem(p, true, &pr)) != VEDA_OK) return st;
    if (hQ == nullptr || hK == nullptr || hV == nullptr || hWq == nullptr || hWk == nullptr ||
        hO == nullptr)
        return fail(VEDA_ERR_INVALID_ARG, "host buffers must be non-NULL");
    if ((st = check_ptr(dQ, "dQ")) || (st = check_ptr(dK, "dK")) || (st = check_ptr(dV, "dV")) ||
        (st = check_ptr(dWq, "dWq")) || (st = check_ptr(dWk, "dWk")) || (st = check_ptr(dO, "dO")) ||
        (st = check_ptr(dlse, "dlse", hlse == nullptr)) || (st = check_ptr(ws, "ws")))
        return st;
    if (head_chunk < 0 || head_chunk > pr.H)
        return fail(VEDA_ERR_INVALID_ARG, "head_chunk must be in 0..H");
    // default: one head per chunk (the copies bound the layer, and the smallest
    // chunk shortens the fill and drain of the pipeline the most)
    if (head_chunk == 0) head_chunk = 1;
    return forward_host_impl(p, pr, hQ, hK, hV, hWq, hWk, hO, hlse, dQ, dK, dV, dWq, dWk, dO,
                             hlse ? dlse : nullptr, ws, head_chunk, (cudaStream_t)stream);
}

veda_status veda_tile_search(const veda_problem* p, const int32_t* candidates, int32_t ncand,
                             const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                             const float* Wq, const float* Wk, uint16_t* O_dense,
                             uint16_t* O_cand, double* err, int32_t* best, void* ws,
                             veda_stream_t stream) {
    if (p == nullptr || candidates == nullptr)
        return fail(VEDA_ERR_INVALID_ARG, "problem and candidates must be non-NULL");
    if (ncand < 1 || ncand > 16) return fail(VEDA_ERR_INVALID_ARG, "1 to 16 candidate tilings");
    if (p->H < 1 || p->H > kMaxHeads) return fail(VEDA_ERR_UNSUPPORTED, "at most 256 heads");
    veda_status st;
    if ((st = check_ptr(Q, "Q")) || (st = check_ptr(K, "K")) || (st = check_ptr(V, "V")) ||
        (st = check_ptr(Wq, "Wq")) || (st = check_ptr(Wk, "Wk")) ||
        (st = check_ptr(O_dense, "O_dense")) || (st = check_ptr(O_cand, "O_cand")) ||
        (st = check_ptr(err, "err")) || (st = check_ptr(best, "best")) || (st = check_ptr(ws, "ws")))
        return st;
    // every candidate tiling, applied to every head, must make a valid problem
    // with the same tile count
    static thread_local int32_t shapes[16][kMaxHeads * 3];
    Problem prs[16];
    for (int c = 0; c < ncand; ++c) {
        for (int h = 0; h < p->H; ++h)
            for (int q = 0; q < 3; ++q) shapes[c][3 * h + q] = candidates[3 * c + q];
        veda_problem pc = *p;
        pc.tile_shapes = shapes[c];
        if ((st = make_problem(&pc, true, &prs[c])) != VEDA_OK) return st;
        if (prs[c].nT != prs[0].nT)
            return fail(VEDA_ERR_SHAPE, "candidate tilings must have the same tile size");
    }
    cudaStream_t s = (cudaStream_t)stream;
    int* status = static_cast<int*>(ws);
    if ((st = cuda_check(cudaMemsetAsync(status, 0, sizeof(int), s), "status reset"))) return st;
    const Problem& p0 = prs[0];
    // full attention (the dense schedule does not depend on the tiling)
    if ((st = launch_sparse_attn(p0, Q, K, V, nullptr, p0.nT, O_dense, nullptr, status, s)))
        return st;
    const long long per_head = (long long)p0.N * p0.d;
    for (int c = 0; c < ncand; ++c) {
        if ((st = forward_impl(prs[c], Q, K, V, Wq, Wk, O_cand, nullptr, nullptr, nullptr, ws, s)))
            return st;
        if ((st = launch_sq_err(O_dense, O_cand, p0.B * p0.H, per_head,
                                err + (size_t)c * p0.B * p0.H, s)))
            return st;
    }
    return launch_argmin(err, ncand, p0.B, p0.H, best, s);
}

veda_status veda_teacher(const veda_problem* p, const uint16_t* Q, const uint16_t* K,
                         const uint16_t* V, uint16_t* O_dense, float* lse_dense, float* teacher,
                         void* ws, veda_stream_t stream) {
    Problem pr;
    veda_status st;
    if ((st = make_problem(p, false, &pr)) != VEDA_OK) return st;
    if ((st = check_ptr(Q, "Q")) || (st = check_ptr(K, "K")) || (st = check_ptr(V, "V")) ||
        (st = check_ptr(O_dense, "O_dense")) || (st = check_ptr(lse_dense, "lse_dense")) ||
        (st = check_ptr(teacher, "teacher")) || (st = check_ptr(ws, "ws")))
        return st;
    cudaStream_t s = (cudaStream_t)stream;
    int* status = static_cast<int*>(ws);
    if ((st = cuda_check(cudaMemsetAsync(status, 0, sizeof(int), s), "status reset"))) return st;
    // dense schedule: every key tile, for the softmax normaliser of every row
    if ((st = launch_sparse_attn(pr, Q, K, V, nullptr, pr.nT, O_dense, lse_dense, status, s)))
        return st;
    return launch_teacher(pr, Q, K, lse_dense, teacher, status, s);
}

veda_status veda_tile_recall(const veda_problem* p, const int32_t* idx_pred,
                             const int32_t* idx_ref, float* recall_rows, double* recall_mean,
                             void* ws, veda_stream_t stream) {
    Problem pr;
    veda_status st;
    if ((st = make_problem(p, true, &pr)) != VEDA_OK) return st;
    if ((st = check_ptr(idx_pred, "idx_pred")) || (st = check_ptr(idx_ref, "idx_ref")) ||
        (st = check_ptr(recall_rows, "recall_rows", true)) ||
        (st = check_ptr(recall_mean, "recall_mean")) || (st = check_ptr(ws, "ws")))
        return st;
    // the hit counter lives in the status area of the workspace, past the status word
    return launch_recall(pr, idx_pred, idx_ref, recall_rows, recall_mean,
                         static_cast<char*>(ws) + 128, (cudaStream_t)stream);
}

veda_status veda_distill_workspace_size(const veda_problem* p, size_t* bytes) {
    Problem pr;
    veda_status st = make_problem(p, false, &pr);
    if (st != VEDA_OK) return st;
    if (bytes == nullptr) return fail(VEDA_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = distill_layout(pr).total;
    return VEDA_OK;
}

veda_status veda_distill_kl(const veda_problem* p, const float* statsQ, const float* statsK,
                            const float* Wq, const float* Wk, const float* S, const float* teacher,
                            float tau, double* loss, float* dWq, float* dWk, void* ws,
                            veda_stream_t stream) {
    Problem pr;
    veda_status st;
    if ((st = make_problem(p, false, &pr)) != VEDA_OK) return st;
    if ((st = check_ptr(statsQ, "statsQ")) || (st = check_ptr(statsK, "statsK")) ||
        (st = check_ptr(Wq, "Wq")) || (st = check_ptr(Wk, "Wk")) || (st = check_ptr(S, "S")) ||
        (st = check_ptr(teacher, "teacher")) || (st = check_ptr(loss, "loss", false)) ||
        (st = check_ptr(dWq, "dWq")) || (st = check_ptr(dWk, "dWk")) || (st = check_ptr(ws, "ws")))
        return st;
    if (!(tau > 0.f) || !isfinite(tau))
        return fail(VEDA_ERR_INVALID_ARG, "tau must be positive and finite");
    cudaStream_t s = (cudaStream_t)stream;
    if ((st = cuda_check(cudaMemsetAsync(ws, 0, sizeof(int), s), "status reset"))) return st;
    return launch_distill(pr, statsQ, statsK, Wq, Wk, S, teacher, tau, loss, dWq, dWk, ws, s);
}

veda_status veda_get_status(const void* ws, veda_stream_t stream, int32_t* device_status) {
    if (ws == nullptr || device_status == nullptr)
        return fail(VEDA_ERR_INVALID_ARG, "ws and device_status must be non-NULL");
    veda_status st;
    cudaStream_t s = (cudaStream_t)stream;
    if ((st = cuda_check(cudaStreamSynchronize(s), "stream synchronize"))) return st;
    return cuda_check(cudaMemcpy(device_status, ws, sizeof(int32_t), cudaMemcpyDeviceToHost),
                      "status read");
}

}  // extern "C"
