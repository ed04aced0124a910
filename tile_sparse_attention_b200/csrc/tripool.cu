// tripool.cu -- TripPool tile statistics.
//
// "Veda: Scalable Video Diffusion via Distilled Sparse Attention" (project
// page), "Attention Structure Distillation", Estimator, and "Theoretical
// Rationale" 2 (Tile Statistics): per head, tile and channel, the average, the
// maximum and the minimum of Q (and K) over the tile's tokens.
//
// HBM-bound: every byte of Q and K is read exactly once with 16-byte vector
// loads.  One CTA of 128 threads pools one tile of one tensor: the tile is
// p_t*p_h runs of p_w contiguous tokens (a token row is d bf16 = 128 or 256
// bytes).  Thread t owns channel group (t % G) (8 channels = 16 bytes) and
// token lane (t / G); it walks its tokens with all loads issued up front, then
// the token lanes are reduced by warp shuffles and across the four warps through
// shared memory.  Output rows (avg, max, min) are written as coalesced fp32.
#include <cuda_bf16.h>

#include "internal.h"

namespace veda {

namespace {

struct TripoolParams {
    const uint16_t* X[2];  // Q, K
    float* out[2];         // statsQ, statsK
    int H, T, Hs, Ws, N, nT;
    int shape[kMaxShapes][3];
    unsigned char head_shape[kMaxHeads];
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// D = head dim, BT = tile tokens.  128 threads.
template <int D, int BT>
__global__ void __launch_bounds__(128) tripool_kernel(const __grid_constant__ TripoolParams p) {
    constexpr int G = D / 8;            // 16-byte channel groups per token row
    constexpr int LANES = 128 / G;      // token lanes
    constexpr int PER = BT / LANES;     // tokens per thread
    __shared__ float red[3][4][8][G];  // [statistic][warp][channel in group][group]

    const int j = blockIdx.x;           // tile
    const int bh = blockIdx.y;          // b*H + h
    const int which = blockIdx.z;       // 0 = Q, 1 = K
    const int h = bh % p.H;
    const int* shp = p.shape[p.head_shape[h]];
    const int pt = shp[0], ph = shp[1], pw = shp[2];
    const int nh = p.Hs / ph, nw = p.Ws / pw;
    const int a = j / (nh * nw), b = (j / nw) % nh, c = j % nw;

    const int g = threadIdx.x % G;
    const int lane_tok = threadIdx.x / G;
    const uint16_t* base = p.X[which] + (size_t)bh * p.N * D;

    // Row r = lane_tok + i*LANES of the tile is token (lt, lh, lw) of the box
    // in raster order; the position is computed once and then advanced by
    // LANES rows with carries (no division per load).
    int lw = lane_tok % pw, lh = (lane_tok / pw) % ph, lt = lane_tok / (ph * pw);
    const int step_w = LANES % pw, step_h = (LANES / pw) % ph, step_t = LANES / (ph * pw);
    uint4 v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int n = ((a * pt + lt) * p.Hs + (b * ph + lh)) * p.Ws + (c * pw + lw);
        v[i] = __ldg(reinterpret_cast<const uint4*>(base + (size_t)n * D) + g);
        lw += step_w;
        lh += step_h;
        lt += step_t;
        if (lw >= pw) {
            lw -= pw;
            ++lh;
        }
        if (lh >= ph) {
            lh -= ph;
            ++lt;
        }
    }
    float sum[8], mx[8], mn[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        sum[e] = 0.f;
        mx[e] = -INFINITY;
        mn[e] = INFINITY;
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        float f[8];
        bf16x8_to_f32(v[i], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            sum[e] += f[e];
            mx[e] = fmaxf(mx[e], f[e]);
            mn[e] = fminf(mn[e], f[e]);
        }
    }
    // token lanes that sit in the same warp hold the same channels: combine them
    // with shuffles, then the four warps through shared memory ([e][g] order, so
    // the 16-byte channel groups of a warp land in distinct banks)
#pragma unroll
    for (int off = G; off < 32; off <<= 1)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            sum[e] += __shfl_xor_sync(0xffffffffu, sum[e], off);
            mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], off));
            mn[e] = fminf(mn[e], __shfl_xor_sync(0xffffffffu, mn[e], off));
        }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane < G) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            red[0][warp][e][g] = sum[e];
            red[1][warp][e][g] = mx[e];
            red[2][warp][e][g] = mn[e];
        }
    }
    __syncthreads();
    float* out = p.out[which] + ((size_t)bh * p.nT + j) * 3 * D;
    for (int ch = threadIdx.x; ch < D; ch += 128) {
        const int cg = ch >> 3, ce = ch & 7;
        float s = 0.f, M = -INFINITY, m = INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            s += red[0][w][ce][cg];
            M = fmaxf(M, red[1][w][ce][cg]);
            m = fminf(m, red[2][w][ce][cg]);
        }
        out[ch] = s * (1.0f / BT);
        out[D + ch] = M;
        out[2 * D + ch] = m;
    }
}

template <int D, int BT>
void launch(const TripoolParams& prm, dim3 grid, cudaStream_t s) {
    tripool_kernel<D, BT><<<grid, 128, 0, s>>>(prm);
}

}  // namespace

veda_status launch_tripool(const Problem& pr, const uint16_t* Q, const uint16_t* K, float* statsQ,
                           float* statsK, cudaStream_t s) {
    TripoolParams prm{};
    prm.X[0] = Q;
    prm.X[1] = K;
    prm.out[0] = statsQ;
    prm.out[1] = statsK;
    prm.H = pr.H;
    prm.T = pr.T;
    prm.Hs = pr.Hs;
    prm.Ws = pr.Ws;
    prm.N = pr.N;
    prm.nT = pr.nT;
    for (int i = 0; i < kMaxShapes; ++i)
        for (int q = 0; q < 3; ++q) prm.shape[i][q] = pr.shape[i][q];
    for (int h = 0; h < pr.H; ++h) prm.head_shape[h] = (unsigned char)pr.head_shape[h];
    dim3 grid(pr.nT, pr.B * pr.H, 2);
    if (pr.d == 128 && pr.Bt == 128) launch<128, 128>(prm, grid, s);
    else if (pr.d == 128 && pr.Bt == 64) launch<128, 64>(prm, grid, s);
    else if (pr.d == 64 && pr.Bt == 128) launch<64, 128>(prm, grid, s);
    else launch<64, 64>(prm, grid, s);
    return cuda_check(cudaGetLastError(), "tripool launch");
}

}  // namespace veda
