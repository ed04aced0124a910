// sparse_attn_dual.cu -- tile-skipping attention for d = 128 and 128-token
// tiles: one query tile per CTA, two softmax groups taking alternate 64-key
// chunks (sm_100a: tcgen05 + TMEM + TMA).
//
// "Veda: Scalable Video Diffusion via Distilled Sparse Attention" (project
// page): "Attention Structure Distillation", Execution (only the selected K/V
// tiles are fetched); "Principle 03 Tile-Sparse Kernel" (TMA gathers of the
// selected tiles overlapped with the tensor-core products); "Theoretical
// Rationale" 1 (Softmax Geometry: the kept keys are renormalised among
// themselves; the two groups' partial results are merged with their own
// maxima and sums, which is exact).
//
// Per 128-key tile and SM, the exponentials (16,384 on the MUFU at 16 per
// clock) and the two products (8.4 MFLOP on the tensor core) both take about
// 1,024 cycles.  With a single softmax warp per sub-partition, S load ->
// exponentials -> P store -> hand-off run in series and bound the kernel.
// Here each sub-partition runs two softmax warps that work on different
// chunks of the same query tile, so one warp's exponentials overlap the
// other's loads, stores and hand-offs, and the tensor core is fed from both.
//
//   * CTA = query tile i of one (b, h); 384 threads:
//       warp 0, 2   TMA producers: the K and V halves of the selected key tiles
//                   j = 0, 2, 4, ... (warp 0) and j = 1, 3, 5, ... (warp 2),
//                   each into its own 3-stage ring;
//       warp 1      allocates the 512 TMEM columns; one elected lane issues
//                   every tcgen05.mma (A operand Q or P in tensor memory;
//                   issuing from an elected lane keeps up with the tensor
//                   core, a lane-index branch does not);
//       warp 3      loads Q by TMA;
//       warps 4-7   softmax group 0: chunks n = 0, 2, 4, ... (thread r owns
//                   query row r), accumulator O_0;
//       warps 8-11  softmax group 1: chunks n = 1, 3, 5, ..., accumulator O_1.
//   * Chunk n = 2j + h is half h of selected key tile j: 64 keys whose K and
//     V (16 KB each) arrive by ONE 5-D TMA copy each (box: half the tile's
//     shape times both 64-channel chunks; the tile is split along its
//     outermost dimension longer than one; rows may come in any order as long
//     as K and V agree).
//   * Tensor memory: S buffers 0-2 (64 fp32 columns each; P written over S as
//     bf16 pairs), Q (64 columns of bf16 pairs), O_0 and O_1 (128 fp32
//     columns each).  Chunk n uses S buffer n mod 3.
//   * Issue order: S(0), S(1), S(2); then per chunk n: wait P(n), O_{n mod 2}
//     += P(n) V, commits that release the ring stage and mark the group's
//     P V done, then S(n+3) = Q K^T into the buffer that P(n) V has just read
//     (one thread issues both, and tcgen05.mma executes in issue order).  A
//     group's next S is computed while the other group works, so each
//     group's chunks run nearly back to back.
//   * A group rescales its O (running max grew by more than 2^8) only after
//     its previous P V completed (pv_done[g]), and reads it in the epilogue
//     after its last one (o_done[g]).
//   * Epilogue: the groups exchange (max, sum) per row through shared memory,
//     each combines half of the 128 channels of O_0 and O_1, divides by the
//     merged sum and writes bf16 straight from registers (a row is one
//     token's 256 contiguous bytes); lse per token.
// Every mbarrier wait is bounded; on expiry the CTA raises its abort flag,
// writes VEDA_ERR_TIMEOUT to the status word, drains its copies and products
// (again bounded), frees tensor memory and exits.  Out-of-range index-list
// entries are replaced by tile 0 and reported as VEDA_ERR_BAD_INDEX.
#include <cuda_bf16.h>

#include "internal.h"
#include "kernel_common.cuh"
#include "ptx.cuh"

namespace veda {

namespace {

constexpr int kThreads = 384;
constexpr int kSoftmaxWarp0 = 4;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kD = 128;                    // head dimension
constexpr int kHB = 64;                    // keys per chunk (half a 128-token tile)
constexpr int kRing = 3;                   // stages per producer
constexpr int kStages = 2 * kRing;
constexpr int kHalfChunk = kHB * 128;        // one 64-channel, 128-byte-swizzled plane
constexpr int kHalfBytes = 2 * kHalfChunk;   // K or V of 64 keys
constexpr int kStageBytes = 2 * kHalfBytes;  // K half + V half
constexpr int kQChunk = 128 * 128;
constexpr int kQBytes = 2 * kQChunk;
constexpr int kQStage = kStages - 1;  // Q staged in the last stage (producer 1's third)
constexpr int kOffBar = kStages * kStageBytes;
// barriers: q_full, q_tmem, kv_full[6], kv_empty[6], s_full[3],
// p_full[3], pv_done[2], o_done[2], drain
constexpr int kNumBars = 2 + 2 * kStages + 3 + 3 + 2 + 2 + 1;
constexpr int kOffML = kOffBar + 512;          // per-row (max, sum) of both groups
constexpr int kOffMisc = kOffML + 2 * 128 * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
static_assert(kNumBars * 8 <= 512, "barrier area");
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
static_assert(kQBytes == kStageBytes, "Q staging fills one ring stage");
// tensor memory columns
constexpr int kTmemS = 0;    // S buffer b at 64 b
constexpr int kTmemQ = 192;
constexpr int kTmemO = 256;  // O_g at kTmemO + 128 g
constexpr int kTmemCols = 512;
constexpr uint32_t kIdescQK = idesc_bf16_f32(128, kHB, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, kD, true);

struct __align__(64) DualParams {
    CUtensorMap tmQ[kMaxShapes];  // box: the whole tile, both channel chunks
    CUtensorMap tmK[kMaxShapes];  // box: half the tile, both channel chunks
    CUtensorMap tmV[kMaxShapes];
    int shape[kMaxShapes][3];
    int split[kMaxShapes];        // dimension halved for the K/V box: 0 = t, 1 = y, 2 = x
    unsigned char head_shape[kMaxHeads];
    const int32_t* idx;  // [B,H,nT,k] or null (dense schedule)
    uint16_t* O;
    float* lse;          // [B,H,N] or null
    int* status;
    int H, T, Hs, Ws, N, nT, k;
    float scale_log2;
    unsigned long long wait_limit_ns;
    int withhold_arrive;  // failure-detection test only: warp 4 skips its first P-ready arrival
};

struct Bars {
    uint64_t* q_full;
    uint64_t* q_tmem;
    uint64_t* kv_full;
    uint64_t* kv_empty;
    uint64_t* s_full;
    uint64_t* p_full;
    uint64_t* pv_done;
    uint64_t* o_done;
    uint64_t* drain;
};

// Ring position of chunk n = 2j + h: producer p = j mod 2 fills its local
// sequence m = 2 (j div 2) + h into stage 3p + m mod 3 (use m div 3).
__device__ __forceinline__ void chunk_stage(int n, int& stage, int& use) {
    const int j = n >> 1, h = n & 1;
    const int m = 2 * (j >> 1) + h;
    stage = kRing * (j & 1) + m % kRing;
    use = m / kRing;
}

// Every tcgen05.mma of the CTA, from one thread: S(0), S(1), S(2), then per
// chunk n: wait P(n), O_{n mod 2} += P(n) V, S(n + 3) = Q K^T into the buffer
// P(n) V has just read.  Ends with a drain of the products.
__device__ __forceinline__ void issue_all(const DualParams& p, const Bars& bars, uint8_t* smem,
                                          uint32_t tbase, volatile int* abort_flag, int chunks) {
    const uint32_t ring = smem_addr(smem);
    // S(n) = Q K^T over the 64 keys of chunk n into buffer n mod 3: A = Q in
    // tensor memory, B = the K half (K-major, two planes)
    auto issue_qk = [&](int n) -> bool {
        int st, u;
        chunk_stage(n, st, u);
        if (!wait_bar(&bars.kv_full[st], u & 1, p, abort_flag)) return false;
        tc_fence_after();
        const uint32_t kaddr = ring + st * kStageBytes;
        const uint32_t dS = tbase + kTmemS + 64 * (n % 3);
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
            const uint64_t bd =
                smem_desc_sw128(kaddr + (ks >> 2) * kHalfChunk + (ks & 3) * 32, 16, 1024);
            mma_bf16_ts(dS, tbase + kTmemQ + ks * 8, bd, kIdescQK, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars.s_full[n % 3]);
        return true;
    };
    bool ok = wait_bar(bars.q_tmem, 0, p, abort_flag);
    for (int n = 0; n < 3 && n < chunks && ok; ++n) ok = issue_qk(n);
    for (int n = 0; n < chunks && ok; ++n) {
        const int b = n % 3, g = n & 1;
        int st, u;
        chunk_stage(n, st, u);
        // the V half landed with the K half (one barrier), whose wait S(n) passed
        if (!wait_bar(&bars.p_full[b], (n / 3) & 1, p, abort_flag)) break;
        tc_fence_after();
        // O_g += P(n) V: A = P(n) (bf16 pairs over S buffer b), B = the V half
        // (MN-major: 64-channel planes 8 KB apart, 16 keys per 2 KB)
        const uint32_t vaddr = ring + st * kStageBytes + kHalfBytes;
#pragma unroll
        for (int ks = 0; ks < kHB / 16; ++ks) {
            const uint64_t bd = smem_desc_sw128(vaddr + ks * 2048, kHalfChunk, 1024);
            mma_bf16_ts(tbase + kTmemO + 128 * g, tbase + kTmemS + 64 * b + ks * 8, bd, kIdescPV,
                        (n >= 2 || ks > 0) ? 1u : 0u);
        }
        mma_commit(&bars.kv_empty[st]);
        mma_commit(&bars.pv_done[g]);
        if (n + 2 >= chunks) mma_commit(&bars.o_done[g]);  // the group's last chunk
        if (n + 3 < chunks) ok = issue_qk(n + 3);
    }
    // Drain: all tensor-core work issued by this thread has completed.
    mma_commit(bars.drain);
    drain_bar(bars.drain, 0, p);
}

// Barrier phase bookkeeping:
//   q_full              Q landed: once
//   q_tmem              all eight softmax warps wrote their half of Q into
//                       tensor memory: once; also gates the first fill of the
//                       Q staging stage
//   kv_full[st]         use u of stage st (K and V halves) has landed:
//                       parity u & 1
//   kv_empty[st]        the P V of use u is done (one commit): parity u & 1
//   s_full[b], p_full[b]  chunk n is use n div 3 of buffer b = n mod 3:
//                       parity (n div 3) & 1
//   pv_done[g]          the i-th P V of group g is done: parity i & 1
// A parity wait for completion c is right only while completion c - 1 has
// happened and c + 1 has not; every wait here is placed so:
//   * the issuer waits P(n) in chunk order; S(n + 3) and P(n + 3) need that
//     wait to have passed;
//   * a group waits S(n) after it saw S(n - 2), whose commit (issued after
//     Q K^T(n - 3)) tracks S(n - 3);
//   * S(n) is issued right after P(n - 3) V, so when the group sees S(n) its
//     P V number i - 2 (chunk n - 4) is complete and number i needs its next
//     P: a rescale waits number i - 1;
//   o_done[g]           the group's last P V is done (so are all before it):
//                       once; the epilogue waits it (after the last P, its
//                       last two P V could have completed, which a parity
//                       wait on pv_done[g] cannot tell apart from neither);
//   * producers and the issuer wait each ring stage's uses in order.
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_dual_kernel(const __grid_constant__ DualParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bar_base = reinterpret_cast<uint64_t*>(smem + kOffBar);
    Bars bars;
    bars.q_full = bar_base;
    bars.q_tmem = bar_base + 1;
    bars.kv_full = bar_base + 2;
    bars.kv_empty = bars.kv_full + kStages;
    bars.s_full = bars.kv_empty + kStages;
    bars.p_full = bars.s_full + 3;
    bars.pv_done = bars.p_full + 3;
    bars.o_done = bars.pv_done + 2;
    bars.drain = bars.o_done + 2;
    float2* ml = reinterpret_cast<float2*>(smem + kOffML);  // [2][128] (max, sum)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i_tile = blockIdx.x;
    const int bh = blockIdx.y;
    const int h = bh % p.H;
    const int slot = p.head_shape[h];
    const int pt = p.shape[slot][0], ph = p.shape[slot][1], pw = p.shape[slot][2];
    const int k = p.k;
    const int chunks = 2 * k;

    // ---------------------------------------------------------------- set-up
    if (threadIdx.x == 0) {
        mbar_init(bars.q_full, 1);
        mbar_init(bars.q_tmem, 8);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars.kv_full[s], 1);
            mbar_init(&bars.kv_empty[s], 1);
        }
        for (int b = 0; b < 3; ++b) {
            mbar_init(&bars.s_full[b], 1);
            mbar_init(&bars.p_full[b], 4);
        }
        mbar_init(&bars.pv_done[0], 1);
        mbar_init(&bars.pv_done[1], 1);
        mbar_init(&bars.o_done[0], 1);
        mbar_init(&bars.o_done[1], 1);
        mbar_init(bars.drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == 3) {
        // ============================================================ Q load
        if (lane == 0) {
            tma_prefetch_desc(&p.tmQ[slot]);
            int t0, y0, x0;
            tile_origin(i_tile, pt, ph, pw, p.Hs, p.Ws, t0, y0, x0);
            mbar_arrive_expect_tx(bars.q_full, kQBytes);
            tma_load_5d(smem + kQStage * kStageBytes, &p.tmQ[slot], bars.q_full, 0, x0, y0,
                        bh * p.T + t0, 0);
        }
        __syncwarp();
        if (lane == 0) drain_bar(bars.q_full, 0, p);  // the Q copy has landed
    } else if (warp == 0 || warp == 2) {
        // ============================================================ producers
        const int pr = warp >> 1;  // key tiles j = pr, pr + 2, ...
        int fills = 0;             // local fills issued (lane 0)
        if (lane == 0) {
            tma_prefetch_desc(&p.tmK[slot]);
            tma_prefetch_desc(&p.tmV[slot]);
        }
        const int sd = p.split[slot];
        const int dt = sd == 0 ? pt / 2 : 0, dy = sd == 1 ? ph / 2 : 0, dx = sd == 2 ? pw / 2 : 0;
        const int32_t* irow = p.idx ? p.idx + ((size_t)bh * p.nT + i_tile) * k : nullptr;
        bool ok = true;
        for (int jb = 0; jb < k && ok; jb += 64) {
            // lane l: key tile jb + 2l + pr and its origin (divisions on all lanes)
            const int j_l = jb + 2 * lane + pr;
            int my_t = 0;
            if (j_l < k) {
                my_t = irow ? irow[j_l] : j_l;
                if (my_t < 0 || my_t >= p.nT) {
                    atomicCAS(p.status, 0, (int)VEDA_ERR_BAD_INDEX);
                    my_t = 0;
                }
            }
            int mt0, my0, mx0;
            tile_origin(my_t, pt, ph, pw, p.Hs, p.Ws, mt0, my0, mx0);
            mt0 += bh * p.T;
            for (int jj = 0; jj < 32 && ok; ++jj) {
                if (jb + 2 * jj + pr >= k) break;  // uniform across the warp
                const int t0 = __shfl_sync(0xffffffffu, mt0, jj);
                const int y0 = __shfl_sync(0xffffffffu, my0, jj);
                const int x0 = __shfl_sync(0xffffffffu, mx0, jj);
                int good = 1;
                if (lane == 0) {
                    for (int hh = 0; hh < 2 && good; ++hh) {
                        const int m = jb + 2 * jj + hh;  // local fill index
                        const int st = kRing * pr + m % kRing, u = m / kRing;
                        if (u > 0)
                            good = wait_bar(&bars.kv_empty[st], (u - 1) & 1, p, abort_flag);
                        else if (st == kQStage)
                            good = wait_bar(bars.q_tmem, 0, p, abort_flag);
                        if (good) {
                            uint8_t* sk = smem + st * kStageBytes;
                            mbar_arrive_expect_tx(&bars.kv_full[st], 2 * kHalfBytes);
                            tma_load_5d(sk, &p.tmK[slot], &bars.kv_full[st], 0, x0 + hh * dx,
                                        y0 + hh * dy, t0 + hh * dt, 0);
                            tma_load_5d(sk + kHalfBytes, &p.tmV[slot], &bars.kv_full[st], 0,
                                        x0 + hh * dx, y0 + hh * dy, t0 + hh * dt, 0);
                            fills = m + 1;
                        }
                    }
                }
                good = __shfl_sync(0xffffffffu, good, 0);
                if (!good) ok = false;
            }
        }
        if (lane == 0) {
            // Drain: every copy this warp issued has landed before the CTA exits.
            for (int r = 0; r < kRing; ++r) {
                if (r < fills) {
                    const uint32_t par = ((fills - 1 - r) / kRing) & 1;
                    drain_bar(&bars.kv_full[kRing * pr + r], par, p);
                }
            }
        }
    } else if (warp == 1) {
        // ============================================================ MMA issuer
        if (elect_one()) issue_all(p, bars, smem, tbase, abort_flag, chunks);
        __syncwarp();
    } else if (warp >= kSoftmaxWarp0) {
        // ============================================================ softmax
        const int g = (warp - kSoftmaxWarp0) >> 2;  // group: chunks n = g, g + 2, ...
        const int wq = warp & 3;                    // TMEM lane quarter
        const int r = wq * 32 + lane;               // query row of the tile
        const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tQ = tbase + lane_off + kTmemQ;
        const uint32_t tO = tbase + lane_off + kTmemO + 128 * g;
        const float c2 = p.scale_log2;
        float m_run = 0.f, l_run = 0.f;
        bool ok = warp_wait_bar(bars.q_full, 0, p, abort_flag);
        if (ok) ok = __all_sync(0xffffffffu, mbar_try_wait(bars.q_full, 0));
        if (ok) {
            // channel chunk g of Q row r: shared-memory staging (128-byte
            // swizzle) -> tensor memory (32 columns of bf16 pairs)
            const uint8_t* sQ = smem + kQStage * kStageBytes + g * kQChunk;
            uint32_t v[32];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint4 q = *reinterpret_cast<const uint4*>(sQ + r * 128 + ((u ^ (r & 7)) << 4));
                v[4 * u] = q.x;
                v[4 * u + 1] = q.y;
                v[4 * u + 2] = q.z;
                v[4 * u + 3] = q.w;
            }
            tmem_st_32x32b_x32(tQ + g * 32, v);
            tmem_wait_st();
            tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.q_tmem);  // even after a failed wait: nobody waits long
        int i = 0;  // chunks done by this group
        for (int n = g; n < chunks && ok; n += 2, ++i) {
            const int b = n % 3;
            const uint32_t tS = tbase + lane_off + kTmemS + 64 * b;
            if (!warp_wait_bar(&bars.s_full[b], (n / 3) & 1, p, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t s[kHB];
            tmem_ld_32x32b_x32(tS, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
            tmem_ld_32x32b_x32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
            tmem_wait_ld();

            // row max: eight independent chains, then a short tree
            float mx8[8];
#pragma unroll
            for (int a = 0; a < 8; ++a) mx8[a] = fmaxf(__uint_as_float(s[a]), __uint_as_float(s[a + 8]));
#pragma unroll
            for (int e = 16; e < kHB; e += 16)
#pragma unroll
                for (int a = 0; a < 8; ++a)
                    mx8[a] = fmax3(mx8[a], __uint_as_float(s[e + a]), __uint_as_float(s[e + 8 + a]));
            const float mx = fmaxf(fmax3(mx8[0], mx8[1], mx8[2]),
                                   fmax3(fmax3(mx8[3], mx8[4], mx8[5]), mx8[6], mx8[7]));
            const float m_tile = mx * c2;
            bool need;
            float m_use, alpha;
            if (i == 0) {
                need = false;
                m_use = m_tile;
                alpha = 0.f;
            } else {
                const float m_new = fmaxf(m_run, m_tile);
                need = m_new > m_run + kRescaleThreshold;
                m_use = need ? m_new : m_run;
                alpha = 1.f;
                // the MUFU is shared with the other group's exponentials on
                // this sub-partition: only a rescale pays for this one
                if (__any_sync(0xffffffffu, need) && need) alpha = fast_exp2(m_run - m_new);
            }
            // p = 2^(s*c2 - m): packed fp32x2 scale-and-shift, MUFU ex2, four
            // independent packed partial sums
            uint32_t pk[kHB / 2];
            const uint64_t c2x2 = f32x2_pack(c2, c2);
            const uint64_t negm = f32x2_pack(-m_use, -m_use);
            uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int e = 0; e < kHB; e += 2) {
                const uint64_t xv = f32x2_fma(
                    f32x2_pack(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), c2x2, negm);
                float x0, x1;
                f32x2_unpack(xv, x0, x1);
                const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
                acc[(e >> 1) & 3] = f32x2_add(acc[(e >> 1) & 3], f32x2_pack(p0, p1));
                pk[e / 2] = pack_bf16x2(p0, p1);
            }
            float a0, a1, a2, a3;
            f32x2_unpack(f32x2_add(acc[0], acc[1]), a0, a1);
            f32x2_unpack(f32x2_add(acc[2], acc[3]), a2, a3);
            const float lsum = (a0 + a2) + (a1 + a3);
            l_run = (i == 0) ? lsum : fmaf(l_run, alpha, lsum);
            m_run = m_use;
            if (__any_sync(0xffffffffu, need)) {
                // O_g must hold the group's previous P V (number i - 1) first
                if (!warp_wait_bar(&bars.pv_done[g], (i - 1) & 1, p, abort_flag)) {
                    ok = false;
                    break;
                }
                {
                    tc_fence_after();
#pragma unroll
                    for (int cc = 0; cc < kD / 32; ++cc) {
                        uint32_t o[32];
                        tmem_ld_32x32b_x32(tO + cc * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st_32x32b_x32(tO + cc * 32, o);
                    }
                }
            }

            // P(n) over S(n) (this thread has read its row of S(n))
            tmem_st_32x32b_x32(tS, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && !(p.withhold_arrive && n == 0 && wq == 0))
                mbar_arrive(&bars.p_full[b]);
        }
        // every P V of the group is done (see the phase notes)
        if (ok) ok = warp_wait_bar(&bars.o_done[g], 0, p, abort_flag);
        ml[g * 128 + r] = make_float2(m_run, l_run);
        // both groups' accumulators are complete once all 256 softmax threads
        // pass this barrier with ok; every thread gets here (all waits are bounded)
        if (named_barrier_and(1, 256, ok)) {
            tc_fence_after();
            // ---------------------------------------------------- epilogue
            const float2 s0 = ml[r], s1 = ml[128 + r];
            const float m = fmaxf(s0.x, s1.x);
            const float f0 = fast_exp2(s0.x - m), f1 = fast_exp2(s1.x - m);
            const float l = s0.y * f0 + s1.y * f1;
            const float w0 = f0 / l, w1 = f1 / l;
            int i_t0, i_y0, i_x0;
            tile_origin(i_tile, pt, ph, pw, p.Hs, p.Ws, i_t0, i_y0, i_x0);
            const int lt = r / (ph * pw), lh = (r / pw) % ph, lw = r % pw;
            const int tok = ((i_t0 + lt) * p.Hs + (i_y0 + lh)) * p.Ws + (i_x0 + lw);
            // group g writes channels [64 g, 64 g + 64) of its row: 128 bytes
            uint4* orow = reinterpret_cast<uint4*>(p.O + ((size_t)bh * p.N + tok) * kD + 64 * g);
            const uint32_t tO0 = tbase + lane_off + kTmemO + 64 * g;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t o0[32], o1[32];
                tmem_ld_32x32b_x32(tO0 + cc * 32, o0);
                tmem_ld_32x32b_x32(tO0 + 128 + cc * 32, o1);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        y[e] = __uint_as_float(o0[8 * q + e]) * w0 + __uint_as_float(o1[8 * q + e]) * w1;
                    uint4 vv;
                    vv.x = pack_bf16x2(y[0], y[1]);
                    vv.y = pack_bf16x2(y[2], y[3]);
                    vv.z = pack_bf16x2(y[4], y[5]);
                    vv.w = pack_bf16x2(y[6], y[7]);
                    orow[cc * 4 + q] = vv;
                }
            }
            if (g == 0 && p.lse != nullptr)
                p.lse[(size_t)bh * p.N + tok] = (m + log2f(l)) * 0.69314718055994531f;
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

}  // namespace

bool dual_attn_supported(const Problem& pr) { return pr.d == kD && pr.Bt == 128; }

veda_status launch_sparse_attn_dual(const Problem& pr, const uint16_t* Q, const uint16_t* K,
                                    const uint16_t* V, const int32_t* idx, int k, uint16_t* O,
                                    float* lse, int* status, cudaStream_t s) {
    if (!dual_attn_supported(pr))
        return fail(VEDA_ERR_UNSUPPORTED, "two-group attention kernel needs d = 128 and Bt = 128");
    DualParams prm;
    memset(&prm, 0, sizeof(prm));
    for (int sh = 0; sh < pr.nshapes; ++sh) {
        const int* shape = pr.shape[sh];
        // split the outermost dimension longer than one (all are powers of two)
        const int sd = shape[0] > 1 ? 0 : (shape[1] > 1 ? 1 : 2);
        int half[3] = {shape[0], shape[1], shape[2]};
        half[sd] /= 2;
        veda_status st;
        if ((st = encode_tile_map_2c(&prm.tmQ[sh], Q, pr, shape)) != VEDA_OK) return st;
        if ((st = encode_tile_map_2c(&prm.tmK[sh], K, pr, half)) != VEDA_OK) return st;
        if ((st = encode_tile_map_2c(&prm.tmV[sh], V, pr, half)) != VEDA_OK) return st;
        for (int q = 0; q < 3; ++q) prm.shape[sh][q] = shape[q];
        prm.split[sh] = sd;
    }
    for (int h = 0; h < pr.H; ++h) prm.head_shape[h] = (unsigned char)pr.head_shape[h];
    prm.idx = idx;
    prm.O = O;
    prm.lse = lse;
    prm.status = status;
    prm.H = pr.H;
    prm.T = pr.T;
    prm.Hs = pr.Hs;
    prm.Ws = pr.Ws;
    prm.N = pr.N;
    prm.nT = pr.nT;
    prm.k = k;
    prm.scale_log2 = pr.scale * 1.4426950408889634f;
    prm.wait_limit_ns = wait_limit_ns();
    // Test hook for the bounded waits: with VEDA_TEST_WITHHOLD_ARRIVE set, one
    // arrival never happens, the MMA issuer's wait runs out and every CTA
    // reports VEDA_ERR_TIMEOUT (nothing in normal use sets the variable).
    prm.withhold_arrive = getenv("VEDA_TEST_WITHHOLD_ARRIVE") != nullptr ? 1 : 0;
    cudaError_t err = cudaFuncSetAttribute(sparse_attn_dual_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return cuda_check(err, "two-group attention smem attribute");
    dim3 grid(pr.nT, pr.B * pr.H);
    sparse_attn_dual_kernel<<<grid, kThreads, kSmemBytes, s>>>(prm);
    return cuda_check(cudaGetLastError(), "two-group attention launch");
}

}  // namespace veda
