// proj_tc.cu -- head-specific projection of the TripPool statistics on the
// tensor cores.
//
// "Veda: Scalable Video Diffusion via Distilled Sparse Attention" (project
// page), "Attention Structure Distillation", Estimator: head-specific Q/K
// projections of the average, maximum and minimum statistics,
//   q~[b,h] (3nT x d) = statsQ[b,h] (3nT x d) . Wq[h] (d x d),  k~ likewise with Wk.
//
// fp32 products at fp32 quality through a three-term TF32 split: with
// x = hi + lo, hi = x rounded to TF32, a.b is taken as a_hi b_hi + a_hi b_lo +
// a_lo b_hi, each term a kind::tf32 tcgen05.mma accumulating in fp32 tensor
// memory.  The kernel computes the transpose, q~^T = Wq^T . stats^T, so that
// tensor-memory lane n is output channel n and an epilogue warp writes 32
// consecutive floats per store:
//   * A = W^T (d rows, zero rows up to 128 when d = 64; K = d), built by the
//     CTA's threads from W in global memory, already split into hi and lo, in
//     the K-major 128-byte-swizzled layout that a TMA copy of W^T would give;
//     rebuilt only when the CTA's blocks move to another head or side;
//   * B = 128 statistics rows per block (N = 128), brought by TMA 64 columns
//     (one "half" of K = 128) at a time into one of two raw buffers, then split
//     in place (hi) and into a lo buffer; the next half's copy goes out as soon
//     as this half's products are issued, so it lands while they run;
//   * warps 0..3 split, build W^T and, through one elected lane, issue the
//     3 x 8 MMAs (M = N = 128, K = 8) of a half into the accumulator of the
//     block's parity (two 128-column accumulators in tensor memory);
//   * warps 4..7, the epilogue, drain the other accumulator meanwhile: thread
//     n reads its 128 columns (statistics rows m = 3j + s of the block) and
//     writes x as hi = TF32(x) and lo = x - hi into the operand layout of the
//     score GEMM (score_tc.cu), per tile j and statistic s: query side
//     [hi | hi | lo], key side [hi | lo | hi], each segment 3d long.
// One launch covers both sides.  Each CTA takes a contiguous range of the
// (side, b*h, 128-row block) blocks, so it changes head rarely.  The
// accumulators pass between the groups as in the score GEMM: acc_full /
// acc_empty of accumulator a complete once per block of parity a.  Waits are
// bounded; warps 0..3 take each decision after an AND of their wait results
// at a named barrier, so they stop together (VEDA_ERR_TIMEOUT in the status
// word, a bounded drain of the copy and products in flight, tensor memory
// freed), and the epilogue warps stop at their next bounded wait.
#include "internal.h"
#include "kernel_common.cuh"
#include "ptx.cuh"

namespace veda {

namespace {

constexpr int kProjThreads = 256;  // warps 0..3: split, W^T, products; warps 4..7: epilogue
constexpr int kBarMain = 1;         // named barrier of warps 0..3
constexpr int kChunk = 128 * 128;              // 128 rows x 32 fp32 (128 B per row)
constexpr int kHalfBytes = 2 * kChunk;         // 128 rows x 64 fp32
constexpr int kOffWhi = 0;                     // W^T hi: up to 4 chunks (K = 128)
constexpr int kOffWlo = 4 * kChunk;            // W^T lo
constexpr int kOffRaw = 8 * kChunk;            // two raw statistics halves (hi after the split)
constexpr int kOffLo = kOffRaw + 2 * kHalfBytes;  // lo of the half being multiplied
constexpr int kOffBar = kOffLo + kHalfBytes;
constexpr int kProjSmem = kOffBar + 128 + 1024;  // + alignment slack
// kind::tf32, fp32 accumulate, both operands K-major, M = N = 128
constexpr uint32_t kIdescProj = (1u << 4) | (2u << 7) | (2u << 10) | ((128u >> 3) << 17) |
                                ((128u >> 4) << 24);

struct __align__(64) ProjParams {
    CUtensorMap mapQ;  // statsQ as B*H*3nT rows of d fp32
    CUtensorMap mapK;  // statsK
    const float* Wq;   // [H][d][d]
    const float* Wk;
    float* qt;         // [B*H*nT][9d]
    float* kt;
    int* status;
    int H, nT;
    int rows_bh;       // statistics rows per (b, h): 3 nT
    int mtiles;        // 128-row blocks per (b, h)
    int bh;            // B * H
    long long blocks;  // 2 * bh * mtiles
    unsigned long long wait_limit_ns;
};

// x rounded to the nearest TF32 value (10 explicit mantissa bits); x - hi is
// exact in fp32.
__device__ __forceinline__ float tf32_hi(float x) {
    return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}

__device__ __forceinline__ float4 tf32_hi4(const float4& x) {
    return make_float4(tf32_hi(x.x), tf32_hi(x.y), tf32_hi(x.z), tf32_hi(x.w));
}

struct Block {
    int side, bhi, h, mt;
};

__device__ __forceinline__ Block decode_block(long long blk, const ProjParams& p) {
    Block b;
    const long long per_side = (long long)p.bh * p.mtiles;
    b.side = (int)(blk / per_side);
    const long long rem = blk - (long long)b.side * per_side;
    b.bhi = (int)(rem / p.mtiles);
    b.mt = (int)(rem - (long long)b.bhi * p.mtiles);
    b.h = b.bhi % p.H;
    return b;
}

// W^T of one head, split, into the K-major swizzled layout: row n (output
// channel), 32-column chunk c = k / 32, 16-byte unit u = (k mod 32) / 4 stored
// at unit u ^ (n mod 8) of the row.  Thread t builds row n = t (zero when
// n >= D), four consecutive k per store; the loads of a k row are coalesced
// over n.
template <int D>
__device__ __forceinline__ void build_wt(uint8_t* smem, const float* W, int n) {
#pragma unroll 4
    for (int k = 0; k < D; k += 4) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (n < D)
            x = make_float4(__ldg(W + (k + 0) * D + n), __ldg(W + (k + 1) * D + n),
                            __ldg(W + (k + 2) * D + n), __ldg(W + (k + 3) * D + n));
        const float4 hi = tf32_hi4(x);
        const float4 lo = make_float4(x.x - hi.x, x.y - hi.y, x.z - hi.z, x.w - hi.w);
        const int c = k >> 5, u = (k & 31) >> 2;
        const int off = c * kChunk + n * 128 + ((u ^ (n & 7)) << 4);
        *reinterpret_cast<float4*>(smem + kOffWhi + off) = hi;
        *reinterpret_cast<float4*>(smem + kOffWlo + off) = lo;
    }
}

template <int D>
__global__ void __launch_bounds__(kProjThreads, 1)
    project_tc_kernel(const __grid_constant__ ProjParams p) {
    constexpr int kHalves = D / 64;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* done = full + 1;
    uint64_t* acc_full = done + 1;       // [2]: a block's products are in accumulator a
    uint64_t* acc_empty = acc_full + 2;  // [2]: accumulator a has been read back
    uint64_t* drain = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const int tid = threadIdx.x, warp = tid >> 5;

    const long long per = (p.blocks + gridDim.x - 1) / gridDim.x;
    const long long b0 = (long long)blockIdx.x * per;
    const long long b1 = b0 + per < p.blocks ? b0 + per : p.blocks;

    if (tid == 0) {
        mbar_init(full, 1);
        mbar_init(done, 1);
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);  // one arrival per epilogue warp
        }
        mbar_init(drain, 32);  // every lane of warp 0 commits once at the end
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);  // two 128-column accumulators
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp < 4) {
        // ==================================================== split, W^T, products
        const uint32_t base = smem_addr(smem);
        // copy of half hk of block blk, the g-th half of this CTA, into raw buffer g & 1
        auto issue_load = [&](long long blk, int hk, int g) {
            const Block b = decode_block(blk, p);
            const CUtensorMap* map = b.side ? &p.mapK : &p.mapQ;
            const int row = b.bhi * p.rows_bh + b.mt * 128;
            uint8_t* dst = smem + kOffRaw + (g & 1) * kHalfBytes;
            mbar_arrive_expect_tx(full, kHalfBytes);
            tma_load_2d(dst, map, full, hk * 64, row);
            tma_load_2d(dst + kChunk, map, full, hk * 64 + 32, row);
        };
        int g = 0;      // halves multiplied so far: the phase of `full` and `done`
        int loads = 0;  // halves whose copy has been issued (the same count in warps 0..3)
        bool ok = true;
        int cur = -1;   // side * H + h of the W^T held in shared memory
        if (b0 < b1) {
            if (warp == 0) {
                if (elect_one()) issue_load(b0, 0, 0);
                __syncwarp();
            }
            loads = 1;
        }
        int lb = 0;  // block of this CTA: accumulator lb & 1, its use lb >> 1
        for (long long blk = b0; blk < b1 && ok; ++blk, ++lb) {
            const Block b = decode_block(blk, p);
            const int acc = lb & 1, use = lb >> 1;
            if (b.side * p.H + b.h != cur) {
                // every earlier product has completed (waited below): W^T may be rewritten
                build_wt<D>(smem, (b.side ? p.Wk : p.Wq) + (size_t)b.h * D * D, tid);
                fence_proxy_async_smem();
                cur = b.side * p.H + b.h;
            }
            // the epilogue warps have read this accumulator's previous block
            if (use > 0) {
                ok = named_barrier_and(kBarMain, 128,
                                       wait_bar(&acc_empty[acc], (use - 1) & 1, p, abort_flag));
                if (!ok) break;
            }
            for (int hk = 0; hk < kHalves; ++hk) {
                ok = named_barrier_and(kBarMain, 128, wait_bar(full, g & 1, p, abort_flag));
                if (!ok) break;
                // split the raw half: hi in place, lo into the lo buffer (whose previous
                // readers, the products of half g - 1, have completed)
                float4* raw = reinterpret_cast<float4*>(smem + kOffRaw + (g & 1) * kHalfBytes);
                float4* lo = reinterpret_cast<float4*>(smem + kOffLo);
                for (int i = tid; i < kHalfBytes / 16; i += 128) {
                    const float4 x = raw[i];
                    const float4 h4 = tf32_hi4(x);
                    raw[i] = h4;
                    lo[i] = make_float4(x.x - h4.x, x.y - h4.y, x.z - h4.z, x.w - h4.w);
                }
                fence_proxy_async_smem();
                named_barrier_sync(kBarMain, 128);
                const bool more = hk + 1 < kHalves || blk + 1 < b1;
                if (warp == 0) {
                    if (elect_one()) {
                        tc_fence_after();
                        const uint32_t rb = base + kOffRaw + (g & 1) * kHalfBytes;
                        const uint32_t lbuf = base + kOffLo;
                        const uint32_t dacc = tbase + acc * 128;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const int c = kk >> 2, w = (kk & 3) * 32;
                            const int kc = hk * 2 + c;  // 32-column chunk of K
                            const uint64_t a_hi =
                                smem_desc_sw128(base + kOffWhi + kc * kChunk + w, 16, 1024);
                            const uint64_t a_lo =
                                smem_desc_sw128(base + kOffWlo + kc * kChunk + w, 16, 1024);
                            const uint64_t b_hi = smem_desc_sw128(rb + c * kChunk + w, 16, 1024);
                            const uint64_t b_lo = smem_desc_sw128(lbuf + c * kChunk + w, 16, 1024);
                            mma_tf32_ss(dacc, a_hi, b_hi, kIdescProj, (hk > 0 || kk > 0) ? 1u : 0u);
                            mma_tf32_ss(dacc, a_hi, b_lo, kIdescProj, 1u);
                            mma_tf32_ss(dacc, a_lo, b_hi, kIdescProj, 1u);
                        }
                        mma_commit(done);
                        if (hk + 1 == kHalves) mma_commit(&acc_full[acc]);
                        // the other raw buffer was freed by the products of half g - 1:
                        // the next half's copy lands while these products run
                        if (hk + 1 < kHalves) issue_load(blk, hk + 1, g + 1);
                        else if (blk + 1 < b1) issue_load(blk + 1, 0, g + 1);
                    }
                    __syncwarp();
                }
                if (more) ++loads;
                ok = named_barrier_and(kBarMain, 128, wait_bar(done, g & 1, p, abort_flag));
                ++g;
                if (!ok) break;
            }
        }
        // drain: no copy or product of this CTA may be in flight when it exits
        if (warp == 0) {
            if (loads > g) {
                if (elect_one()) drain_bar(full, (loads - 1) & 1, p);
                __syncwarp();
            }
            mma_commit(drain);  // every lane: arrives once its own products, if any, are done
            __syncwarp();
            if (tid == 0) drain_bar(drain, 0, p);
            __syncwarp();
        }
    } else {
        // ==================================================== epilogue (warps 4..7)
        // tensor-memory lane n = output channel n (lane quarter warp & 3);
        // column = block row m
        const int q = warp & 3;
        const int n = q * 32 + (tid & 31);
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        int lb = 0;
        for (long long blk = b0; blk < b1; ++blk, ++lb) {
            const int acc = lb & 1, use = lb >> 1;
            // after an abort an accumulator may be incomplete: nothing more is written
            if (!warp_wait_bar(&acc_full[acc], use & 1, p, abort_flag) ||
                __any_sync(0xffffffffu, *abort_flag != 0))
                break;  // the whole warp leaves: the tensor-memory loads below are warp-wide
            tc_fence_after();
            const Block b = decode_block(blk, p);
            float* out = b.side ? p.kt : p.qt;
            const int m0 = b.mt * 128;
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tbase + lane_off + acc * 128 + cc * 32, v);
                tmem_wait_ld();
                if (n < D) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int m = m0 + cc * 32 + e;  // statistics row m = 3j + s of (b, h)
                        if (m < p.rows_bh) {
                            const int j = m / 3, s = m - 3 * j;
                            float* row = out + ((size_t)b.bhi * p.nT + j) * (9 * D) + s * D + n;
                            const float x = __uint_as_float(v[e]);
                            const float hi = tf32_hi(x), lo = x - hi;
                            row[0] = hi;
                            row[3 * D] = b.side ? lo : hi;
                            row[6 * D] = b.side ? hi : lo;
                        }
                    }
                }
            }
            // the accumulator is read: the products of the block after next may start
            tc_fence_before();
            __syncwarp();
            if ((tid & 31) == 0) mbar_arrive(&acc_empty[acc]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, 256);
    }
}

template <int D>
veda_status launch_project_d(const ProjParams& prm, cudaStream_t s) {
    cudaError_t err = cudaFuncSetAttribute(project_tc_kernel<D>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kProjSmem);
    if (err != cudaSuccess) return cuda_check(err, "projection smem attribute");
    const long long ctas = prm.blocks < sm_count() ? prm.blocks : sm_count();
    project_tc_kernel<D><<<(unsigned)ctas, kProjThreads, kProjSmem, s>>>(prm);
    return cuda_check(cudaGetLastError(), "projection launch");
}

}  // namespace

veda_status launch_project_pair(const Problem& pr, const float* statsQ, const float* statsK,
                                const float* Wq, const float* Wk, float* qt, float* kt,
                                int* status, cudaStream_t s) {
    ProjParams prm;
    memset(&prm, 0, sizeof(prm));
    const long long rows = (long long)pr.B * pr.H * 3 * pr.nT;
    veda_status st;
    if ((st = encode_rows_map(&prm.mapQ, statsQ, rows, pr.d, 128)) != VEDA_OK) return st;
    if ((st = encode_rows_map(&prm.mapK, statsK, rows, pr.d, 128)) != VEDA_OK) return st;
    prm.Wq = Wq;
    prm.Wk = Wk;
    prm.qt = qt;
    prm.kt = kt;
    prm.status = status;
    prm.H = pr.H;
    prm.nT = pr.nT;
    prm.rows_bh = 3 * pr.nT;
    prm.mtiles = (prm.rows_bh + 127) / 128;
    prm.bh = pr.B * pr.H;
    prm.blocks = 2LL * prm.bh * prm.mtiles;
    prm.wait_limit_ns = wait_limit_ns();
    return pr.d == 128 ? launch_project_d<128>(prm, s) : launch_project_d<64>(prm, s);
}

}  // namespace veda
