// sgemm.cu -- batched register-blocked fp32 SIMT GEMM for the distillation
// products ("Principle 01 Full-Attention Structure Distillation" and
// "Theoretical Rationale" 4 of the Veda project page: the loss gradients
// dL/dW_q and dL/dW_k are fp32 matrix products of the statistics and the
// score gradient).  128 x 128 block tile, 8 x 8 outputs per thread,
// double-buffered shared memory; transposed-A, transposed-B and accumulate
// modes.  (The estimator's forward projection runs on the tensor cores in
// proj_tc.cu.)
#include "internal.h"

namespace veda {

namespace {

constexpr int BM = 128, BN = 128, BK = 8, PAD = 4;

struct GemmParams {
    const float* A;
    const float* B;
    float* C;
    int M, N, K;
    int lda, ldb, ldc;
    long long strideA, strideB, strideC;  // per batch entry
    int b_batch_mod;                      // >0: B index = batch % b_batch_mod
    int accumulate;                       // C += A . B
    int a_batch_mod;                      // >0: A index = batch % a_batch_mod
};

// C[z] = A[z] . B[z]  (B_T = false: B is K x N row-major)
// C[z] = A[z] . B[z]^T (B_T = true: B is N x K row-major)
// A_T = true: A is stored K x M row-major (C = A^T . B).  K is a multiple of 8.
template <bool B_T, bool A_T = false>
__global__ void __launch_bounds__(256) sgemm_kernel(const __grid_constant__ GemmParams p) {
    __shared__ __align__(16) float As[2][BK][BM + PAD];
    __shared__ __align__(16) float Bs[2][BK][BN + PAD];

    const int z = blockIdx.z;
    const int az = p.a_batch_mod > 0 ? z % p.a_batch_mod : z;
    const float* A = p.A + (long long)az * p.strideA;
    const int bz = p.b_batch_mod > 0 ? z % p.b_batch_mod : z;
    const float* Bm = p.B + (long long)bz * p.strideB;
    float* C = p.C + (long long)z * p.strideC;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;

    // global -> register staging
    const int a_row = tid >> 1, a_k = (tid & 1) * 4;
    const int bn_k = tid >> 5, bn_n = (tid & 31) * 4;  // B not transposed
    float4 ra, rb;

    auto load_a = [&](int k0) {
        if (A_T) {
            const int m = m0 + bn_n;
            ra = (m < p.M)
                     ? *reinterpret_cast<const float4*>(A + (long long)(k0 + bn_k) * p.lda + m)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
            const int m = m0 + a_row;
            ra = (m < p.M) ? *reinterpret_cast<const float4*>(A + (long long)m * p.lda + k0 + a_k)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    auto load_b = [&](int k0) {
        if (B_T) {
            const int n = n0 + a_row;
            rb = (n < p.N) ? *reinterpret_cast<const float4*>(Bm + (long long)n * p.ldb + k0 + a_k)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
            const int n = n0 + bn_n;
            rb = (n < p.N)
                     ? *reinterpret_cast<const float4*>(Bm + (long long)(k0 + bn_k) * p.ldb + n)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    auto store_tiles = [&](int buf) {
        if (A_T) {
            *reinterpret_cast<float4*>(&As[buf][bn_k][bn_n]) = ra;
        } else {
            As[buf][a_k + 0][a_row] = ra.x;
            As[buf][a_k + 1][a_row] = ra.y;
            As[buf][a_k + 2][a_row] = ra.z;
            As[buf][a_k + 3][a_row] = ra.w;
        }
        if (B_T) {
            Bs[buf][a_k + 0][a_row] = rb.x;
            Bs[buf][a_k + 1][a_row] = rb.y;
            Bs[buf][a_k + 2][a_row] = rb.z;
            Bs[buf][a_k + 3][a_row] = rb.w;
        } else {
            *reinterpret_cast<float4*>(&Bs[buf][bn_k][bn_n]) = rb;
        }
    };

    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

    load_a(0);
    load_b(0);
    store_tiles(0);
    __syncthreads();
    const int nk = p.K / BK;
    for (int kt = 0; kt < nk; ++kt) {
        const int buf = kt & 1;
        if (kt + 1 < nk) {
            load_a((kt + 1) * BK);
            load_b((kt + 1) * BK);
        }
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        if (kt + 1 < nk) {
            store_tiles(buf ^ 1);
            __syncthreads();
        }
    }

    const bool vec = (p.ldc % 4) == 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
        if (m >= p.M) continue;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int n = n0 + half * 64 + tx * 4;
            const float* v = &acc[i][half * 4];
            float* dst = C + (long long)m * p.ldc + n;
            if (vec && n + 3 < p.N) {
                float4 o = make_float4(v[0], v[1], v[2], v[3]);
                if (p.accumulate) {
                    const float4 c = *reinterpret_cast<const float4*>(dst);
                    o.x += c.x; o.y += c.y; o.z += c.z; o.w += c.w;
                }
                *reinterpret_cast<float4*>(dst) = o;
            } else {
                for (int e = 0; e < 4; ++e)
                    if (n + e < p.N) dst[e] = p.accumulate ? dst[e] + v[e] : v[e];
            }
        }
    }
}

}  // namespace

veda_status launch_sgemm(const float* A, const float* B, float* C, int M, int N, int K, int lda,
                         int ldb, int ldc, long long strideA, long long strideB, long long strideC,
                         int batches, int a_batch_mod, int b_batch_mod, bool a_t, bool b_t,
                         bool accumulate, cudaStream_t s) {
    if (K % 8 != 0 || lda % 4 != 0 || ldb % 4 != 0)
        return fail(VEDA_ERR_UNSUPPORTED, "fp32 GEMM needs K and leading dimensions divisible by 8/4");
    GemmParams g{};
    g.A = A;
    g.B = B;
    g.C = C;
    g.M = M;
    g.N = N;
    g.K = K;
    g.lda = lda;
    g.ldb = ldb;
    g.ldc = ldc;
    g.strideA = strideA;
    g.strideB = strideB;
    g.strideC = strideC;
    g.a_batch_mod = a_batch_mod;
    g.b_batch_mod = b_batch_mod;
    g.accumulate = accumulate ? 1 : 0;
    dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM, batches);
    if (a_t && !b_t) sgemm_kernel<false, true><<<grid, 256, 0, s>>>(g);
    else if (!a_t && b_t) sgemm_kernel<true, false><<<grid, 256, 0, s>>>(g);
    else if (!a_t && !b_t) sgemm_kernel<false, false><<<grid, 256, 0, s>>>(g);
    else return fail(VEDA_ERR_UNSUPPORTED, "fp32 GEMM: A and B both transposed");
    return cuda_check(cudaGetLastError(), "fp32 GEMM launch");
}

}  // namespace veda
