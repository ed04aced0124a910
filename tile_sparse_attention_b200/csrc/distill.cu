// distill.cu -- KL structure distillation of the tile-score estimator.
//
// "Veda: Scalable Video Diffusion via Distilled Sparse Attention" (project
// page), "Principle 01 Full-Attention Structure Distillation" and
// "Theoretical Rationale" 4 (Distillation Objective): the max-pooled teacher
// defines a target distribution over key tiles, the estimator produces a soft
// distribution over key tiles, and the row-wise KL divergence between them is
// minimised before Top-k.
//
//   A_tgt[i, :]  = T[i, :] / sum_j T[i, j]
//   A_pred[i, :] = softmax(S[i, :] / tau)
//   L            = (1 / R) sum_i KL(A_tgt[i] || A_pred[i])      (R rows)
//   dL/dS        = G = (A_pred - A_tgt) / (tau R)
//   dq~ = G k~,  dk~ = G^T q~,  dW_q[h] = sum_b statsQ^T dq~,  dW_k likewise
//
// One warp per row computes the row's log-softmax, its KL term and its row of
// G (fp32 values, fp64 row sums); the loss is the mean of the row terms in a
// fixed summation order (deterministic).  The backward products run on the
// batched fp32 GEMM.
#include "internal.h"

namespace veda {

namespace {

__global__ void kl_rows_kernel(const float* __restrict__ S, const float* __restrict__ T,
                               float* __restrict__ G, double* __restrict__ row_kl, long long rows,
                               int nT, float inv_tau, float g_scale) {
    const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float* s = S + row * nT;
    const float* t = T + row * nT;
    float* g = G + row * nT;
    float mx = -INFINITY;
    double tsum = 0.0;
    for (int j = lane; j < nT; j += 32) {
        mx = fmaxf(mx, s[j]);
        tsum += (double)t[j];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        tsum += __shfl_xor_sync(0xffffffffu, tsum, off);
    }
    const float m = mx * inv_tau;
    double se = 0.0;
    for (int j = lane; j < nT; j += 32) se += (double)expf(fmaf(s[j], inv_tau, -m));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) se += __shfl_xor_sync(0xffffffffu, se, off);
    const float lse = m + (float)log(se);
    const float inv_tsum = (float)(1.0 / tsum);
    double kl = 0.0;
    for (int j = lane; j < nT; j += 32) {
        const float logp = fmaf(s[j], inv_tau, -lse);
        const float pr = expf(logp);
        const float tg = t[j] * inv_tsum;
        if (tg > 0.f) kl += (double)tg * ((double)logf(tg) - (double)logp);
        g[j] = (pr - tg) * g_scale;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kl += __shfl_xor_sync(0xffffffffu, kl, off);
    if (lane == 0) row_kl[row] = kl;
}

// Mean of v[0..n) in a fixed order: thread t sums t, t+1024, ..., then a tree.
__global__ void __launch_bounds__(1024) mean_kernel(const double* __restrict__ v, long long n,
                                                    double* out) {
    __shared__ double part[1024];
    double acc = 0.0;
    for (long long i = threadIdx.x; i < n; i += 1024) acc += v[i];
    part[threadIdx.x] = acc;
    __syncthreads();
    for (int w = 512; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) *out = part[0] / (double)n;
}

}  // namespace

DistillLayout distill_layout(const Problem& pr) {
    auto align = [](size_t x) { return (x + 255) & ~(size_t)255; };
    DistillLayout w{};
    const size_t proj = (size_t)pr.B * pr.H * pr.nT * 3 * pr.d * sizeof(float);
    const size_t rows = (size_t)pr.B * pr.H * pr.nT;
    size_t off = VEDA_STATUS_BYTES;
    w.qt = off;
    off = align(off + proj);
    w.kt = off;
    off = align(off + proj);
    w.dq = off;
    off = align(off + proj);
    w.dk = off;
    off = align(off + proj);
    w.G = off;
    off = align(off + rows * pr.nT * sizeof(float));
    w.row_kl = off;
    off = align(off + rows * sizeof(double));
    w.total = off;
    return w;
}

veda_status launch_distill(const Problem& pr, const float* statsQ, const float* statsK,
                           const float* Wq, const float* Wk, const float* S, const float* teacher,
                           float tau, double* loss, float* dWq, float* dWk, void* ws,
                           cudaStream_t s) {
    if (pr.nT % 8 != 0) return fail(VEDA_ERR_UNSUPPORTED, "distillation needs nT divisible by 8");
    const DistillLayout w = distill_layout(pr);
    char* base = static_cast<char*>(ws);
    float* qt = reinterpret_cast<float*>(base + w.qt);
    float* kt = reinterpret_cast<float*>(base + w.kt);
    float* dq = reinterpret_cast<float*>(base + w.dq);
    float* dk = reinterpret_cast<float*>(base + w.dk);
    float* G = reinterpret_cast<float*>(base + w.G);
    double* row_kl = reinterpret_cast<double*>(base + w.row_kl);
    const int BH = pr.B * pr.H, nT = pr.nT, d = pr.d;
    const long long st3 = (long long)3 * nT * d;  // per (b, h) block of stats / q~ / dq~
    const long long rows = (long long)BH * nT;
    veda_status st;
    // q~ = stats . W  ([3 nT] x d per (b, h)), plain fp32 layout [nT][3][d]
    if ((st = launch_sgemm(statsQ, Wq, qt, 3 * nT, d, d, d, d, d, st3, (long long)d * d, st3, BH,
                           0, pr.H, false, false, false, s)))
        return st;
    if ((st = launch_sgemm(statsK, Wk, kt, 3 * nT, d, d, d, d, d, st3, (long long)d * d, st3, BH,
                           0, pr.H, false, false, false, s)))
        return st;
    const float inv_tau = 1.0f / tau;
    const float g_scale = (float)(1.0 / ((double)tau * (double)rows));
    const unsigned blocks = (unsigned)((rows * 32 + 255) / 256);
    kl_rows_kernel<<<blocks, 256, 0, s>>>(S, teacher, G, row_kl, rows, nT, inv_tau, g_scale);
    if ((st = cuda_check(cudaGetLastError(), "kl rows launch"))) return st;
    mean_kernel<<<1, 1024, 0, s>>>(row_kl, rows, loss);
    if ((st = cuda_check(cudaGetLastError(), "loss launch"))) return st;
    const long long gst = (long long)nT * nT;
    // dq~ = G k~ : [nT x nT] . [nT x 3d]
    if ((st = launch_sgemm(G, kt, dq, nT, 3 * d, nT, nT, 3 * d, 3 * d, gst, st3, st3, BH, 0, 0,
                           false, false, false, s)))
        return st;
    // dk~ = G^T q~ : A = G stored [i][j] = [K][M]
    if ((st = launch_sgemm(G, qt, dk, nT, 3 * d, nT, nT, 3 * d, 3 * d, gst, st3, st3, BH, 0, 0,
                           true, false, false, s)))
        return st;
    // dW[h] = sum over b of stats[b,h]^T dq~[b,h] : [d x 3nT] . [3nT x d]
    for (int b = 0; b < pr.B; ++b) {
        const long long off = (long long)b * pr.H * st3;
        if ((st = launch_sgemm(statsQ + off, dq + off, dWq, d, d, 3 * nT, d, d, d, st3, st3,
                               (long long)d * d, pr.H, 0, 0, true, false, b > 0, s)))
            return st;
        if ((st = launch_sgemm(statsK + off, dk + off, dWk, d, d, 3 * nT, d, d, d, st3, st3,
                               (long long)d * d, pr.H, 0, 0, true, false, b > 0, s)))
            return st;
    }
    return VEDA_OK;
}

}  // namespace veda
