// teacher.cu -- max-pooled full-attention teacher and tile recall.
//
// "Veda: Scalable Video Diffusion via Distilled Sparse Attention" (project
// page), "Attention Structure Distillation", Teacher: max-pooling the full
// attention map gives tile-level supervision; "Empirical Study" 02
// (Controlled Mask Intervention): the oracle mask keeps, for each query tile,
// the key tiles with the highest max-pooled response, and tile recall is the
// fraction of oracle-selected tiles a predicted mask recovers.
//
// Teacher:  T[i, j] = max over query tokens q of tile i and key tokens of tile
// j of P[q, key],  P = softmax(scale * Q K^T) over all N keys.
// exp is monotonic and lse_q (the log of the row's softmax normaliser) does
// not depend on the key, so
//   T[i, j] = max over q in tile i of exp(scale * max_{key in j} s[q, key] - lse_q).
// The dense lse comes from the dense attention schedule; this kernel is one
// Q K^T pass per (query tile, key tile) with a row max, one exp per row and a
// tile max folded into T by an atomic maximum on the (non-negative) fp32 bits.
//
// Kernel layout (one CTA per query tile, 256 threads): warp 0 streams Q once
// and every K tile through an NS-deep TMA ring; warp 1 allocates tensor
// memory and one elected lane issues S_j = Q K_j^T (A = Q from tensor memory) into
// two TMEM S buffers; warps 4..7 (thread = query row) read S_j, take the row
// max and fold the tile maximum into T.  All waits are bounded.
#include "internal.h"
#include "kernel_common.cuh"
#include "ptx.cuh"

namespace veda {

namespace {

constexpr int kTThreads = 256;
constexpr int kTSoftmaxWarp0 = 4;

struct __align__(64) TeacherParams {
    CUtensorMap tmQ[kMaxShapes];
    CUtensorMap tmK[kMaxShapes];
    int shape[kMaxShapes][3];
    unsigned char head_shape[kMaxHeads];
    const float* lse;              // dense lse [B,H,N] (natural log)
    unsigned int* teacher_bits;    // [B,H,nT,nT], fp32 bit patterns, zeroed by the host
    int* status;
    int H, T, Hs, Ws, N, nT;
    float scale_log2;
    unsigned long long wait_limit_ns;
};

template <int D, int BT, int NS>
struct TCfg {
    static constexpr int kChunks = D / 64;
    static constexpr int kQChunk = 128 * 128;
    static constexpr int kQBytes = kChunks * kQChunk;
    static constexpr int kKBytes = BT * D * 2;
    static constexpr int kKChunk = BT * 128;
    static constexpr int kOffK = kQBytes;
    static constexpr int kOffBar = kOffK + NS * kKBytes;
    // barriers: q, q_tmem, k_full[NS], k_empty[NS], s_full[2], s_free[2], drain
    static constexpr int kNumBars = 2 + 2 * NS + 4 + 1;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
    static constexpr int kTmemQ = 2 * BT;            // S buffers at [0, BT) and [BT, 2 BT)
    static constexpr int kTmemCols = (2 * BT + 64) <= 256 ? 256 : 512;
    static constexpr uint32_t kIdescQK = idesc_bf16_f32(128, BT, false);
};

// Barrier phases: k_full/k_empty[st] fill n of stage st (tile j = st + n*NS):
// parity n & 1; s_full/s_free[b] use m of buffer b (tile j = b + 2m): parity
// m & 1.  Every next completion needs its waiter to have passed the current
// wait, so parities are unambiguous.
template <int D, int BT, int NS>
__global__ void __launch_bounds__(kTThreads, 1)
    teacher_kernel(const __grid_constant__ TeacherParams p) {
    using C = TCfg<D, BT, NS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sQ = smem;
    uint8_t* sK = smem + C::kOffK;
    uint64_t* bar_q = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* bar_q_tmem = bar_q + 1;
    uint64_t* k_full = bar_q + 2;
    uint64_t* k_empty = k_full + NS;
    uint64_t* s_full = k_empty + NS;
    uint64_t* s_free = s_full + 2;
    uint64_t* bar_drain = s_free + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i_tile = blockIdx.x, bh = blockIdx.y;
    const int h = bh % p.H;
    const int slot = p.head_shape[h];
    const int pt = p.shape[slot][0], ph = p.shape[slot][1], pw = p.shape[slot][2];
    const int nT = p.nT;

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        mbar_init(bar_q_tmem, 4);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_free[b], 4);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (BT < 128) {
        for (int c = 0; c < C::kChunks; ++c) {
            uint4* q = reinterpret_cast<uint4*>(sQ + c * C::kQChunk + BT * 128);
            for (int e = threadIdx.x; e < (128 - BT) * 8; e += kTThreads) q[e] = make_uint4(0, 0, 0, 0);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == 0) {
        // ============================================================ producer
        if (lane == 0) {
            int t0, y0, x0;
            tile_origin(i_tile, pt, ph, pw, p.Hs, p.Ws, t0, y0, x0);
            tma_prefetch_desc(&p.tmQ[slot]);
            tma_prefetch_desc(&p.tmK[slot]);
            mbar_arrive_expect_tx(bar_q, BT * D * 2);
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c)
                tma_load_5d(sQ + c * C::kQChunk, &p.tmQ[slot], bar_q, c * 64, x0, y0, t0, bh);
            int fills = 0;
            for (int j = 0; j < nT; ++j) {
                const int st = j % NS, n = j / NS;
                if (n > 0 && !wait_bar(&k_empty[st], (n - 1) & 1, p, abort_flag)) break;
                tile_origin(j, pt, ph, pw, p.Hs, p.Ws, t0, y0, x0);
                mbar_arrive_expect_tx(&k_full[st], C::kKBytes);
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c)
                    tma_load_5d(sK + st * C::kKBytes + c * C::kKChunk, &p.tmK[slot], &k_full[st],
                                c * 64, x0, y0, t0, bh);
                fills = j + 1;
            }
            drain_bar(bar_q, 0, p);
            for (int st = 0; st < NS; ++st)
                if (st < fills) drain_bar(&k_full[st], ((fills - 1 - st) / NS) & 1, p);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ============================================================ MMA issuer
        if (elect_one()) {
            const uint32_t k_addr = smem_addr(sK);
            const uint32_t tQ = tbase + C::kTmemQ;
            bool ok = wait_bar(bar_q_tmem, 0, p, abort_flag);
            for (int j = 0; j < nT && ok; ++j) {
                const int st = j % NS, b = j & 1;
                if (!wait_bar(&k_full[st], (j / NS) & 1, p, abort_flag)) break;
                if (j >= 2 && !wait_bar(&s_free[b], ((j - 2) >> 1) & 1, p, abort_flag)) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const int c = ks >> 2, w = ks & 3;
                    const uint64_t bd = smem_desc_sw128(
                        k_addr + st * C::kKBytes + c * C::kKChunk + w * 32, 16, 1024);
                    mma_bf16_ts(tbase + b * BT, tQ + ks * 8, bd, C::kIdescQK, ks > 0 ? 1u : 0u);
                }
                mma_commit(&s_full[b]);
                mma_commit(&k_empty[st]);
            }
            mma_commit(bar_drain);
            drain_bar(bar_drain, 0, p);
        }
        __syncwarp();
    } else if (warp >= kTSoftmaxWarp0) {
        // ============================================================ row maxima
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tS = tbase + lane_off;
        const uint32_t tQ = tbase + lane_off + C::kTmemQ;
        float lse2 = 0.f;
        if (r < BT) {
            int t0, y0, x0;
            tile_origin(i_tile, pt, ph, pw, p.Hs, p.Ws, t0, y0, x0);
            const int lt = r / (ph * pw), lh = (r / pw) % ph, lw = r % pw;
            const int n = ((t0 + lt) * p.Hs + (y0 + lh)) * p.Ws + (x0 + lw);
            lse2 = p.lse[(size_t)bh * p.N + n] * 1.4426950408889634f;
        }
        bool ok = warp_wait_bar(bar_q, 0, p, abort_flag);
        if (ok) ok = __all_sync(0xffffffffu, mbar_try_wait(bar_q, 0));
        if (ok) {
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c) {
                uint32_t v[32];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint4 x = *reinterpret_cast<const uint4*>(sQ + c * C::kQChunk + r * 128 +
                                                                    ((u ^ (r & 7)) << 4));
                    v[4 * u] = x.x;
                    v[4 * u + 1] = x.y;
                    v[4 * u + 2] = x.z;
                    v[4 * u + 3] = x.w;
                }
                tmem_st_32x32b_x32(tQ + c * 32, v);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_q_tmem);
        }
        unsigned int* trow = p.teacher_bits + ((size_t)bh * nT + i_tile) * nT;
        for (int j = 0; j < nT && ok; ++j) {
            const int b = j & 1;
            if (!warp_wait_bar(&s_full[b], (j >> 1) & 1, p, abort_flag)) break;
            tc_fence_after();
            uint32_t s[BT];
#pragma unroll
            for (int cc = 0; cc < BT / 32; ++cc)
                tmem_ld_32x32b_x32(tS + b * BT + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&s[cc * 32]));
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[b]);
            float m8[8];
#pragma unroll
            for (int a = 0; a < 8; ++a)
                m8[a] = fmaxf(__uint_as_float(s[a]), __uint_as_float(s[a + 8]));
#pragma unroll
            for (int e = 16; e < BT; e += 16)
#pragma unroll
                for (int a = 0; a < 8; ++a)
                    m8[a] = fmax3(m8[a], __uint_as_float(s[e + a]), __uint_as_float(s[e + 8 + a]));
            const float mx = fmaxf(fmax3(m8[0], m8[1], m8[2]),
                                   fmax3(fmax3(m8[3], m8[4], m8[5]), m8[6], m8[7]));
            // max over the row's keys of P[q, key]; rows beyond the tile are padding
            float pm = (r < BT) ? exp2f(fmaf(mx, p.scale_log2, -lse2)) : 0.f;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, off));
            if (lane == 0 && wq * 32 < BT) atomicMax(trow + j, __float_as_uint(pm));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, C::kTmemCols);
    }
}

template <int D, int BT, int NS>
veda_status launch_teacher_cfg(const TeacherParams& prm, const Problem& pr, cudaStream_t s) {
    using C = TCfg<D, BT, NS>;
    static_assert(C::kSmemBytes <= 227 * 1024, "shared memory budget");
    cudaError_t err = cudaFuncSetAttribute(teacher_kernel<D, BT, NS>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           C::kSmemBytes);
    if (err != cudaSuccess) return cuda_check(err, "teacher smem attribute");
    dim3 grid(pr.nT, pr.B * pr.H);
    teacher_kernel<D, BT, NS><<<grid, kTThreads, C::kSmemBytes, s>>>(prm);
    return cuda_check(cudaGetLastError(), "teacher launch");
}

// Tile recall: one thread per row; both index lists are ascending.
__global__ void recall_count_kernel(const int32_t* a, const int32_t* b, long long rows, int k,
                                    float* per_row, unsigned long long* hits) {
    const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    unsigned int c = 0;
    if (row < rows) {
        const int32_t* x = a + row * k;
        const int32_t* y = b + row * k;
        int u = 0, v = 0;
        while (u < k && v < k) {
            const int32_t xu = x[u], yv = y[v];
            c += (xu == yv) ? 1u : 0u;
            u += (xu <= yv) ? 1 : 0;
            v += (yv <= xu) ? 1 : 0;
        }
        if (per_row) per_row[row] = (float)c / (float)k;
    }
    // block sum of the hit counts, one atomic per block (exact integer sum)
    __shared__ unsigned int part[8];
    unsigned int w = c;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) w += __shfl_xor_sync(0xffffffffu, w, off);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = w;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long t = 0;
        for (int q = 0; q < (int)(blockDim.x >> 5); ++q) t += part[q];
        atomicAdd(hits, t);
    }
}

__global__ void recall_finalize_kernel(const unsigned long long* hits, long long total,
                                       double* mean) {
    *mean = (double)*hits / (double)total;
}

}  // namespace

veda_status launch_teacher(const Problem& pr, const uint16_t* Q, const uint16_t* K,
                           const float* lse, float* teacher, int* status, cudaStream_t s) {
    TeacherParams prm;
    memset(&prm, 0, sizeof(prm));
    for (int sh = 0; sh < pr.nshapes; ++sh) {
        veda_status st;
        if ((st = encode_tile_map(&prm.tmQ[sh], Q, pr, pr.shape[sh])) != VEDA_OK) return st;
        if ((st = encode_tile_map(&prm.tmK[sh], K, pr, pr.shape[sh])) != VEDA_OK) return st;
        for (int q = 0; q < 3; ++q) prm.shape[sh][q] = pr.shape[sh][q];
    }
    for (int h = 0; h < pr.H; ++h) prm.head_shape[h] = (unsigned char)pr.head_shape[h];
    prm.lse = lse;
    prm.teacher_bits = reinterpret_cast<unsigned int*>(teacher);
    prm.status = status;
    prm.H = pr.H;
    prm.T = pr.T;
    prm.Hs = pr.Hs;
    prm.Ws = pr.Ws;
    prm.N = pr.N;
    prm.nT = pr.nT;
    prm.scale_log2 = pr.scale * 1.4426950408889634f;
    prm.wait_limit_ns = wait_limit_ns();
    veda_status st = cuda_check(
        cudaMemsetAsync(teacher, 0, (size_t)pr.B * pr.H * pr.nT * pr.nT * sizeof(float), s),
        "teacher reset");
    if (st != VEDA_OK) return st;
    if (pr.d == 128 && pr.Bt == 128) return launch_teacher_cfg<128, 128, 4>(prm, pr, s);
    if (pr.d == 128 && pr.Bt == 64) return launch_teacher_cfg<128, 64, 6>(prm, pr, s);
    if (pr.d == 64 && pr.Bt == 128) return launch_teacher_cfg<64, 128, 6>(prm, pr, s);
    return launch_teacher_cfg<64, 64, 8>(prm, pr, s);
}

veda_status launch_recall(const Problem& pr, const int32_t* idx_pred, const int32_t* idx_ref,
                          float* per_row, double* mean, void* scratch8, cudaStream_t s) {
    const long long rows = (long long)pr.B * pr.H * pr.nT;
    unsigned long long* hits = static_cast<unsigned long long*>(scratch8);
    veda_status st = cuda_check(cudaMemsetAsync(hits, 0, sizeof(unsigned long long), s),
                                "recall reset");
    if (st != VEDA_OK) return st;
    const unsigned blocks = (unsigned)((rows + 255) / 256);
    recall_count_kernel<<<blocks, 256, 0, s>>>(idx_pred, idx_ref, rows, pr.k, per_row, hits);
    if ((st = cuda_check(cudaGetLastError(), "recall launch"))) return st;
    recall_finalize_kernel<<<1, 1, 0, s>>>(hits, rows * pr.k, mean);
    return cuda_check(cudaGetLastError(), "recall finalize launch");
}

}  // namespace veda
