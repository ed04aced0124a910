// tile_search.cu -- head-aware tile search.
//
// "Veda: Scalable Video Diffusion via Distilled Sparse Attention" (project
// page), "Head-Aware Tile Search": among factorisations p_t * p_h * p_w = Bt
// of the hardware tile, each head takes the tiling pi that minimises
// ||O_full - O_sparse(pi)||_F^2 on calibration samples ("Principle 02
// Head-Conditioned Tile Geometry"; "Theoretical Rationale" 3).
//
// For every candidate the whole layer runs with that tiling on every head
// (TripPool, score, Top-k, tile-skipping attention); the dense schedule gives
// O_full once.  Per (candidate, batch entry, head) the squared error is summed
// in fp64 in a fixed order (one CTA per head and batch entry), and per head
// the candidate with the smallest error summed over the batch (the calibration
// samples) wins, ties to the lower candidate index.
#include "internal.h"

namespace veda {

namespace {

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// err[bh] = sum over the N*d entries of head bh of (a - b)^2, fixed order.
__global__ void __launch_bounds__(1024) sq_err_kernel(const uint16_t* __restrict__ a,
                                                      const uint16_t* __restrict__ b,
                                                      long long per_head, double* err) {
    __shared__ double part[1024];
    const long long base = (long long)blockIdx.x * per_head;
    double acc = 0.0;
    for (long long e = threadIdx.x; e < per_head; e += 1024) {
        const double d = (double)bf16_to_f32(a[base + e]) - (double)bf16_to_f32(b[base + e]);
        acc += d * d;
    }
    part[threadIdx.x] = acc;
    __syncthreads();
    for (int w = 512; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) err[blockIdx.x] = part[0];
}

// best[h] = argmin over candidates c of sum over b of err[c][b][h].
__global__ void argmin_kernel(const double* err, int ncand, int B, int H, int32_t* best) {
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= H) return;
    int arg = 0;
    double lo = 0.0;
    for (int c = 0; c < ncand; ++c) {
        double s = 0.0;
        for (int b = 0; b < B; ++b) s += err[((size_t)c * B + b) * H + h];
        if (c == 0 || s < lo) {
            lo = s;
            arg = c;
        }
    }
    best[h] = arg;
}

}  // namespace

veda_status launch_sq_err(const uint16_t* a, const uint16_t* b, int heads, long long per_head,
                          double* err, cudaStream_t s) {
    sq_err_kernel<<<heads, 1024, 0, s>>>(a, b, per_head, err);
    return cuda_check(cudaGetLastError(), "squared error launch");
}

veda_status launch_argmin(const double* err, int ncand, int B, int H, int32_t* best,
                          cudaStream_t s) {
    argmin_kernel<<<(H + 127) / 128, 128, 0, s>>>(err, ncand, B, H, best);
    return cuda_check(cudaGetLastError(), "argmin launch");
}

}  // namespace veda
