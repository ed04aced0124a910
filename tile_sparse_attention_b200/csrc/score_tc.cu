// score_tc.cu -- the tile-pair score matrix on the tensor cores.
//
// "Veda: Scalable Video Diffusion via Distilled Sparse Attention" (project
// page), "Attention Structure Distillation", Estimator:
//   S[i, j] = sum over s in {avg, max, min} of <q~_{i,s}, k~_{j,s}>,
// an nT x nT x 3d contraction per head.
//
// The decision that follows (Top-k) wants fp32-grade scores, so the product
// runs as a three-term TF32 split: every fp32 value x is written by the
// projection as hi = x rounded to TF32 and lo = x - hi, with
//   q^ = [q_hi | q_hi | q_lo],  k^ = [k_hi | k_lo | k_hi]   (length 9d),
// so that q^ . k^ = q_hi k_hi + q_hi k_lo + q_lo k_hi, which differs from the
// fp32 product by at most about 3 * 2^-21 |q||k| per term (the dropped lo*lo
// term and the TF32 truncation of lo); accumulation is fp32 in tensor memory.
// S = q^ k^^T is then one kind::tf32 GEMM with K = 9d:
//   * one CTA per 128 x BN block of S of one head (BN = 256 for large score
//     matrices: the operands come from L2 at about the rate TMA can move
//     them, and a wider block loads each q^ row for twice the columns;
//     BN = 128 when 256 would pad the columns by more than a tenth or leave
//     fewer than two blocks per SM); 128 threads;
//   * warp 0 lane 0 streams 32-wide K blocks of q^ (128 rows) and k^ (BN
//     rows), 128 B per row with the 128-byte swizzle, by TMA into a ring;
//   * warp 1 allocates BN TMEM columns; one of its lanes, chosen by
//     elect.sync, issues 4 tcgen05.mma (M = 128, N = BN, K = 8) per K block;
//   * all four warps read the accumulator back (thread = row) and store S.
// Every S element accumulates the same products in the same order for
// either BN, so the two block widths give identical S.
// Waits are bounded (VEDA_ERR_TIMEOUT in the status word, then a bounded drain
// of the copies and products in flight before tensor memory is freed; S is not
// written by a CTA that gave up).
#include "internal.h"
#include "kernel_common.cuh"
#include "ptx.cuh"

namespace veda {

namespace {

constexpr int kScoreThreads = 128;

template <int BN>
struct ScoreCfg {
    static constexpr int kStages = BN == 256 ? 4 : 3;
    static constexpr int kTileA = 128 * 128;  // 128 rows x 32 fp32
    static constexpr int kTileB = BN * 128;   // BN rows x 32 fp32
    static constexpr int kStageBytes = kTileA + kTileB;
    static constexpr int kSmemBytes = kStages * kStageBytes + 256 + 1024;
    // kind::tf32, fp32 accumulate, both operands K-major, M = 128, N = BN
    static constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) |
                                       ((uint32_t)(BN >> 3) << 17) | ((128u >> 4) << 24);
};

struct __align__(64) ScoreParams {
    CUtensorMap mapA;  // q^: rows B*H*nT, K = 9d
    CUtensorMap mapB;  // k^
    float* S;
    int* status;
    int nT, kblocks;
    unsigned long long wait_limit_ns;
    int withhold_fill;  // failure-detection test only: the first K block is never loaded
};

template <int BN>
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_tc_kernel(const __grid_constant__ ScoreParams p) {
    using C = ScoreCfg<BN>;
    constexpr int kStages = C::kStages;
    constexpr int kStageBytes = C::kStageBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* done = empty + kStages;
    uint64_t* drain = done + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j0 = blockIdx.x * BN, i0 = blockIdx.y * 128, bh = blockIdx.z;
    const int rowA = bh * p.nT + i0, rowB = bh * p.nT + j0;
    const int KB = p.kblocks;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, BN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    bool ok = true;
    if (warp == 0 && lane == 0) {
        // ---------------------------------------------------------- producer
        tma_prefetch_desc(&p.mapA);
        tma_prefetch_desc(&p.mapB);
        int issued = 0;
        for (int kb = 0; kb < KB; ++kb) {
            const int st = kb % kStages, n = kb / kStages;
            if (n > 0 && !wait_bar(&empty[st], (n - 1) & 1, p, abort_flag)) break;
            if (p.withhold_fill && kb == 0) {
                // test hook: stage 0's first fill never happens, so the issuer's
                // wait on it runs out (and stage 0 is never refilled)
                issued = 1;
                continue;
            }
            uint8_t* a = smem + st * kStageBytes;
            mbar_arrive_expect_tx(&full[st], kStageBytes);
            tma_load_2d(a, &p.mapA, &full[st], kb * 32, rowA);
            tma_load_2d(a + C::kTileA, &p.mapB, &full[st], kb * 32, rowB);
            issued = kb + 1;
        }
        for (int st = 0; st < kStages; ++st)  // drain: the last fill of every stage
            if (st < issued && !(p.withhold_fill && st == 0))
                drain_bar(&full[st], ((issued - 1 - st) / kStages) & 1, p);
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        // (one lane chosen by elect.sync: a branch on the lane index costs the
        // issuing thread more per tcgen05.mma than the product takes)
        if (elect_one()) {
            const uint32_t base = smem_addr(smem);
            for (int kb = 0; kb < KB && ok; ++kb) {
                const int st = kb % kStages;
                if (!wait_bar(&full[st], (kb / kStages) & 1, p, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a = base + st * kStageBytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = smem_desc_sw128(a + kk * 32, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(a + C::kTileA + kk * 32, 16, 1024);
                    mma_tf32_ss(tbase, ad, bd, C::kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&empty[st]);
            }
            mma_commit(done);
            mma_commit(drain);
            drain_bar(drain, 0, p);
        }
    }
    __syncwarp();

    // -------------------------------------------------------------- epilogue
    int got = 0;
    // after an abort the accumulator is incomplete: S is not written
    if (lane == 0) got = (wait_bar(done, 0, p, abort_flag) && !*abort_flag) ? 1 : 0;
    got = __shfl_sync(0xffffffffu, got, 0);
    __syncwarp();
    if (got) {
        tc_fence_after();
        const int r = warp * 32 + lane;
        const int i = i0 + r;
        const uint32_t taddr = tbase + (static_cast<uint32_t>(warp * 32) << 16);
        float* srow = p.S + ((size_t)bh * p.nT + i) * p.nT;
        const bool vec = (p.nT % 4) == 0;
#pragma unroll
        for (int cc = 0; cc < BN / 32; ++cc) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(taddr + cc * 32, v);
            tmem_wait_ld();
            const int jb = j0 + cc * 32;
            if (i < p.nT) {
                if (vec && jb + 32 <= p.nT) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4*>(srow + jb + e) =
                            make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                        __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (jb + e < p.nT) srow[jb + e] = __uint_as_float(v[e]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, BN);
    }
}

template <int BN>
veda_status launch_score_bn(ScoreParams& prm, const Problem& pr, const float* kext, long long rows,
                            int kx, cudaStream_t s) {
    using C = ScoreCfg<BN>;
    veda_status st;
    if ((st = encode_rows_map(&prm.mapB, kext, rows, kx, BN)) != VEDA_OK) return st;
    cudaError_t err = cudaFuncSetAttribute(score_tc_kernel<BN>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (err != cudaSuccess) return cuda_check(err, "score smem attribute");
    dim3 grid((pr.nT + BN - 1) / BN, (pr.nT + 127) / 128, pr.B * pr.H);
    score_tc_kernel<BN><<<grid, kScoreThreads, C::kSmemBytes, s>>>(prm);
    return cuda_check(cudaGetLastError(), "score launch");
}

}  // namespace

veda_status launch_score(const Problem& pr, const float* qext, const float* kext, float* S,
                         int* status, cudaStream_t s) {
    ScoreParams prm;
    memset(&prm, 0, sizeof(prm));
    const long long rows = (long long)pr.B * pr.H * pr.nT;
    const int kx = 9 * pr.d;
    veda_status st;
    if ((st = encode_rows_map(&prm.mapA, qext, rows, kx)) != VEDA_OK) return st;
    prm.S = S;
    prm.status = status;
    prm.nT = pr.nT;
    prm.kblocks = kx / 32;
    prm.wait_limit_ns = wait_limit_ns();
    // Test hook for the bounded waits (nothing in normal use sets the variable).
    prm.withhold_fill = getenv("VEDA_TEST_WITHHOLD_ARRIVE") != nullptr ? 1 : 0;
    // 256-column blocks when they pad the columns by at most a tenth more than
    // 128-column ones and still give every SM two blocks
    const long long pad128 = (pr.nT + 127) / 128 * 128, pad256 = (pr.nT + 255) / 256 * 256;
    const long long blocks256 = (pad256 / 256) * ((pr.nT + 127) / 128) * (long long)pr.B * pr.H;
    if (pad256 * 10 <= pad128 * 11 && blocks256 >= 2LL * sm_count())
        return launch_score_bn<256>(prm, pr, kext, rows, kx, s);
    return launch_score_bn<128>(prm, pr, kext, rows, kx, s);
}

}  // namespace veda
