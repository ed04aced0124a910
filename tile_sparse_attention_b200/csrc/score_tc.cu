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
// S = q^ k^^T is then one kind::tf32 GEMM with K = 9d, in a persistent kernel
// (one CTA per SM, 192 threads) that walks 128 x BN blocks of S round-robin,
// the column block fastest so that the CTAs running at one time share q^ rows
// in L2:
//   * BN = 256 for large score matrices (each q^ row block is loaded once for
//     twice the columns), BN = 128 when 256 would pad the columns by more
//     than a tenth or leave fewer than two blocks per SM;
//   * warp 0 (one elected lane) streams 32-wide K blocks of q^ (128 rows) and
//     k^ (BN rows), 128 B per row with the 128-byte swizzle, by TMA into a
//     ring that runs on across blocks;
//   * warp 1 allocates two BN-column accumulators in tensor memory; one lane,
//     chosen by elect.sync, issues 4 tcgen05.mma (M = 128, N = BN, K = 8) per
//     K block into the accumulator of the block's parity;
//   * warps 2..5 (thread = row, one warp per TMEM lane quarter) read a finished
//     accumulator back and store S while the next block's products run in
//     the other accumulator.
// Every S element accumulates the same products in the same order for either
// BN, so the two block widths give identical S.
// Barrier phases: full / empty of ring stage st complete once per fill (the
// ring position g = K blocks so far, fill g / stages); acc_full / acc_empty of
// accumulator a once per block of parity a (use u = local block >> 1).  The
// issuer waits acc_empty(u - 1) before it fills use u, and acc_empty(u)
// needs the epilogue to have waited acc_full(u), so neither side runs two
// phases ahead.  Waits are bounded (VEDA_ERR_TIMEOUT in the status word, then
// a bounded drain of the copies and products in flight before tensor memory
// is freed); no block is written once the CTA has given up.
#include "internal.h"
#include "kernel_common.cuh"
#include "ptx.cuh"

namespace veda {

namespace {

constexpr int kScoreWarps = 6;  // 0: TMA, 1: tensor memory + MMA issue, 2..5: epilogue
constexpr int kScoreThreads = 32 * kScoreWarps;
constexpr int kRingBytes = 192 * 1024;

template <int BN>
struct ScoreCfg {
    static constexpr int kTileA = 128 * 128;  // 128 rows x 32 fp32
    static constexpr int kTileB = BN * 128;   // BN rows x 32 fp32
    static constexpr int kStageBytes = kTileA + kTileB;
    static constexpr int kStages = kRingBytes / kStageBytes;  // 4 (BN = 256) or 6
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
    int tiles_i, tiles_j, ntiles;  // 128-row blocks, BN-column blocks, blocks in all
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
    uint64_t* acc_full = empty + kStages;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = p.kblocks;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);  // one arrival per epilogue warp
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 2 * BN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (elect_one()) {
            tma_prefetch_desc(&p.mapA);
            tma_prefetch_desc(&p.mapB);
            int last_fill[kStages];  // last fill issued into each stage (-1: none)
            for (int st = 0; st < kStages; ++st) last_fill[st] = -1;
            int g = 0;  // ring position: K blocks so far
            bool ok = true;
            for (int t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x) {
                const int jb = t % p.tiles_j, rest = t / p.tiles_j;
                const int ib = rest % p.tiles_i, bh = rest / p.tiles_i;
                const int rowA = bh * p.nT + ib * 128, rowB = bh * p.nT + jb * BN;
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    const int st = g % kStages, n = g / kStages;
                    if (n > 0 && !wait_bar(&empty[st], (n - 1) & 1, p, abort_flag)) {
                        ok = false;
                        break;
                    }
                    // test hook: the first fill never happens, so the issuer's wait
                    // on it runs out (and its stage is never refilled)
                    if (p.withhold_fill && g == 0) continue;
                    uint8_t* a = smem + st * kStageBytes;
                    mbar_arrive_expect_tx(&full[st], kStageBytes);
                    tma_load_2d(a, &p.mapA, &full[st], kb * 32, rowA);
                    tma_load_2d(a + C::kTileA, &p.mapB, &full[st], kb * 32, rowB);
                    last_fill[st] = n;
                }
            }
            for (int st = 0; st < kStages; ++st)  // drain: the last fill of every stage
                if (last_fill[st] >= 0) drain_bar(&full[st], last_fill[st] & 1, p);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        // (one lane chosen by elect.sync: a branch on the lane index costs the
        // issuing thread more per tcgen05.mma than the product takes)
        if (elect_one()) {
            const uint32_t base = smem_addr(smem);
            int g = 0, lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x, ++lt) {
                const int acc = lt & 1, use = lt >> 1;
                if (use > 0 && !wait_bar(&acc_empty[acc], (use - 1) & 1, p, abort_flag)) break;
                tc_fence_after();
                const uint32_t dacc = tbase + acc * BN;
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    const int st = g % kStages;
                    if (!wait_bar(&full[st], (g / kStages) & 1, p, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a = base + st * kStageBytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = smem_desc_sw128(a + kk * 32, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(a + C::kTileA + kk * 32, 16, 1024);
                        mma_tf32_ss(dacc, ad, bd, C::kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&empty[st]);
                }
                if (ok) mma_commit(&acc_full[acc]);
            }
            // drain: all tensor-core work issued by this thread has completed
            mma_commit(drain);
            drain_bar(drain, 0, p);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;  // TMEM lane quarter of this warp
        const int r = q * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        const bool vec = (p.nT % 4) == 0;
        int lt = 0;
        for (int t = blockIdx.x; t < p.ntiles; t += gridDim.x, ++lt) {
            const int acc = lt & 1, use = lt >> 1;
            // after an abort an accumulator may be incomplete: no more blocks are written
            if (!warp_wait_bar(&acc_full[acc], use & 1, p, abort_flag) ||
                __any_sync(0xffffffffu, *abort_flag != 0))
                break;  // the whole warp leaves: the tensor-memory loads below are warp-wide
            tc_fence_after();
            const int jb = t % p.tiles_j, rest = t / p.tiles_j;
            const int ib = rest % p.tiles_i, bh = rest / p.tiles_i;
            const int i = ib * 128 + r, j0 = jb * BN;
            float* srow = p.S + ((size_t)bh * p.nT + i) * p.nT;
#pragma unroll
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tbase + lane_off + acc * BN + cc * 32, v);
                tmem_wait_ld();
                const int jb0 = j0 + cc * 32;
                if (i < p.nT) {
                    if (vec && jb0 + 32 <= p.nT) {
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            *reinterpret_cast<float4*>(srow + jb0 + e) =
                                make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                            __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (jb0 + e < p.nT) srow[jb0 + e] = __uint_as_float(v[e]);
                    }
                }
            }
            // the accumulator is read: the issuer may start the block after next in it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, 2 * BN);
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
    prm.tiles_i = (pr.nT + 127) / 128;
    prm.tiles_j = (pr.nT + BN - 1) / BN;
    const long long ntiles = (long long)prm.tiles_i * prm.tiles_j * pr.B * pr.H;
    if (ntiles > (1LL << 30)) return fail(VEDA_ERR_UNSUPPORTED, "score matrix too large");
    prm.ntiles = (int)ntiles;
    const int ctas = prm.ntiles < sm_count() ? prm.ntiles : sm_count();
    score_tc_kernel<BN><<<ctas, kScoreThreads, C::kSmemBytes, s>>>(prm);
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
