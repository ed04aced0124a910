// topk.cu -- head-aware Top-k of the tile scores into a 0/1 tile mask and an
// ascending index list.
//
// "Veda: Scalable Video Diffusion via Distilled Sparse Attention" (project
// page), "Attention Structure Distillation", Execution: Top-k selection per
// query tile produces the tile mask handed to the tile-skipping kernel.  Ties
// go to the lower tile index; -0.0 and +0.0 tie.
//
// One warp per row.  Scores become order-preserving 32-bit keys (larger score
// -> larger key), held in shared memory.  An exact radix select (8 bits per
// pass, most significant first, over the bits in which the row's keys differ)
// finds the k-th largest key K* and how many keys equal to K* are kept (the
// lowest-index ones).  A final pass in
// ascending index order emits the mask and, through warp ballots and prefix
// pop-counts, the index list already sorted.  The selection is an integer
// computation on the fp32 scores, so it is exactly reproducible.
#include "internal.h"
#include "kernel_common.cuh"

namespace veda {

namespace {

struct TopkParams {
    const float* S;
    uint8_t* mask;
    int32_t* idx;
    long long rows;
    int nT, k;
};

template <int WARPS>
__global__ void __launch_bounds__(WARPS * 32) topk_kernel(const __grid_constant__ TopkParams p) {
    extern __shared__ __align__(16) uint32_t smem_u[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * WARPS + warp;
    if (row >= p.rows) return;
    const int nT = p.nT;
    const int nT4 = (nT + 3) & ~3;
    uint32_t* keys = smem_u + (size_t)warp * (nT4 + 256);
    uint32_t* hist = keys + nT4;
    const float* srow = p.S + row * nT;

    for (int j = lane; j < nT; j += 32) keys[j] = order_key(__ldg(srow + j));

    // Bits above the highest bit in which the row's keys differ are common to
    // all keys: the radix passes start below them, so the first histogram is
    // spread out instead of piling every key into one bin.
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int j = lane; j < nT; j += 32) {
        kmin = min(kmin, keys[j]);
        kmax = max(kmax, keys[j]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, off));
    }
    const int top = 32 - __clz(kmin ^ kmax);  // number of bits that vary (0..32)
    uint32_t prefix = kmin & (top == 32 ? 0u : ~((1u << top) - 1u));
    uint32_t pmask = top == 32 ? 0u : ~((1u << top) - 1u);
    int kr = p.k;  // rank of the wanted key among the candidates, from the top
#pragma unroll 1
    for (int hi = top; hi > 0; hi -= 8) {
        const int shift = hi >= 8 ? hi - 8 : 0;
        const uint32_t dmask = (hi >= 8 ? 255u : (1u << hi) - 1u);
        for (int b = lane; b < 256; b += 32) hist[b] = 0;
        __syncwarp();
        for (int j = lane; j < nT; j += 32) {
            const uint32_t key = keys[j];
            if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
        }
        __syncwarp();
        // lane l owns bins 255-8l ... 248-8l (descending digit order)
        uint32_t cnt[8];
        uint32_t local = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            cnt[e] = hist[255 - 8 * lane - e];
            local += cnt[e];
        }
        uint32_t incl = local;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        const uint32_t hit = __ballot_sync(0xffffffffu, incl >= (uint32_t)kr);
        const int src = __ffs(hit) - 1;  // kr <= candidates, so some lane hits
        uint32_t digit = 0, above = 0;
        if (lane == src) {
            uint32_t run = incl - local;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (run + cnt[e] >= (uint32_t)kr) {
                    digit = 255 - 8 * lane - e;
                    above = run;
                    break;
                }
                run += cnt[e];
            }
        }
        digit = __shfl_sync(0xffffffffu, digit, src);
        above = __shfl_sync(0xffffffffu, above, src);
        kr -= (int)above;
        prefix |= digit << shift;
        pmask |= dmask << shift;
        __syncwarp();
    }
    const uint32_t thr = prefix;  // k-th largest key; keep kr of the keys equal to it

    const unsigned lt_mask = (1u << lane) - 1u;
    int eq_seen = 0, sel_seen = 0;
    int32_t* irow = p.idx + row * p.k;
    uint8_t* mrow = p.mask ? p.mask + row * nT : nullptr;
    for (int j0 = 0; j0 < nT; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t key = j < nT ? keys[j] : 0u;
        const bool eq = (j < nT) && key == thr;
        const unsigned eq_b = __ballot_sync(0xffffffffu, eq);
        const int eq_rank = eq_seen + __popc(eq_b & lt_mask);
        const bool sel = (j < nT) && (key > thr || (eq && eq_rank < kr));
        const unsigned sel_b = __ballot_sync(0xffffffffu, sel);
        if (sel) irow[sel_seen + __popc(sel_b & lt_mask)] = j;
        if (mrow && j < nT) mrow[j] = sel ? 1 : 0;
        eq_seen += __popc(eq_b);
        sel_seen += __popc(sel_b);
    }
}

}  // namespace

veda_status launch_topk(const Problem& pr, const float* S, uint8_t* mask, int32_t* idx,
                        cudaStream_t s) {
    TopkParams prm{};
    prm.S = S;
    prm.mask = mask;
    prm.idx = idx;
    prm.rows = (long long)pr.B * pr.H * pr.nT;
    prm.nT = pr.nT;
    prm.k = pr.k;
    const size_t per_warp = ((size_t)((pr.nT + 3) & ~3) + 256) * sizeof(uint32_t);
    cudaError_t err;
    if (pr.nT <= 4096) {
        constexpr int W = 4;
        const size_t smem = per_warp * W;
        err = cudaFuncSetAttribute(topk_kernel<W>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)smem);
        if (err != cudaSuccess) return cuda_check(err, "topk smem attribute");
        const unsigned blocks = (unsigned)((prm.rows + W - 1) / W);
        topk_kernel<W><<<blocks, W * 32, smem, s>>>(prm);
    } else {
        constexpr int W = 1;
        const size_t smem = per_warp * W;
        err = cudaFuncSetAttribute(topk_kernel<W>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)smem);
        if (err != cudaSuccess) return cuda_check(err, "topk smem attribute");
        topk_kernel<W><<<(unsigned)prm.rows, 32, smem, s>>>(prm);
    }
    return cuda_check(cudaGetLastError(), "topk launch");
}

}  // namespace veda
