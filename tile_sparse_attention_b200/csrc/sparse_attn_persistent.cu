// sparse_attn_persistent.cu -- tile-skipping attention for short key lists:
// persistent CTAs that carry the pipeline from one query tile to the next.
//
// "Veda: Scalable Video Diffusion via Distilled Sparse Attention" (project
// page): "Attention Structure Distillation", Execution (only the selected K/V
// tiles are fetched); "Principle 03 Tile-Sparse Kernel" (TMA gathers overlap
// the tensor-core products); "Theoretical Rationale" 1 (the kept keys are
// renormalised among themselves).  It computes exactly what the one-CTA-per-
// query-tile kernel (sparse_attn.cu) computes, with the same products in the
// same order per query tile.
//
// With one CTA per query tile, every CTA pays a fixed cost outside its tile
// loop (tensor-memory allocation, the Q load and copy, filling the pipeline,
// the epilogue): about 15,000 SM cycles, against ~2,000 per key tile.  That is
// 7% of the work at k = 96 but most of it at k <= 12.  Here one CTA per SM
// loops over query tiles u = c, c + G, c + 2G, ... (G CTAs), and everything
// continues across tiles:
//   * warp 0 (TMA producer) streams Q of each query tile into one staging
//     buffer, and the selected K and V tiles of all its query tiles through
//     one NS-deep ring (the key tiles of the CTA form one stream g = n*k + j);
//   * warp 1 allocates tensor memory once; one elected lane issues S_g = Q_n K_g^T
//     (A = Q_n from one of two TMEM Q buffers, B = K from the ring) and
//     O += P_g V_g, with S_{g+2} queued behind P_g V_g across tile boundaries;
//   * warps 4..7 (thread = query row) run the online softmax of tile n, copy
//     Q of tile n+1 into the other TMEM Q buffer as soon as the last P of tile
//     n is written (so the first products of tile n+1 run during tile n's
//     epilogue), then normalise O and write it straight from registers.
// The pipeline's steady state costs about 5% more per key tile than the
// one-CTA-per-tile kernel (measured), while the per-tile fixed cost drops to
// ~6,000 cycles, so the library uses this kernel for k <= 64 and the other
// one above.
// Every wait on an mbarrier is bounded by a time limit; on expiry the CTA sets
// VEDA_ERR_TIMEOUT in the status word, drains its outstanding copies and
// tensor-core work (again with a limit), frees its tensor memory and exits.
#include <cuda_bf16.h>

#include "internal.h"
#include "kernel_common.cuh"
#include "ptx.cuh"

namespace veda {

namespace {

constexpr int kThreads = 256;
constexpr int kSoftmaxWarp0 = 4;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct __align__(64) AttnParams {
    CUtensorMap tmQ[kMaxShapes];
    CUtensorMap tmK[kMaxShapes];
    CUtensorMap tmV[kMaxShapes];
    int shape[kMaxShapes][3];
    unsigned char head_shape[kMaxHeads];
    const int32_t* idx;  // [B,H,nT,k] or null (dense schedule)
    uint16_t* O;         // [B,H,N,d]
    float* lse;          // [B,H,N] or null
    int* status;
    int H, T, Hs, Ws, N, nT, k;
    int total_tiles;     // B * H * nT query tiles, shared out over the persistent CTAs
    float scale_log2;
    unsigned long long wait_limit_ns;
    int withhold_arrive;  // failure-detection test only: warp 4 skips its first P-ready arrival
};

template <int D, int BT, int NS>
struct Cfg {
    static constexpr int kChunks = D / 64;           // 64-channel (128-byte) chunks
    static constexpr int kQChunk = 128 * 128;        // bytes per Q staging chunk (128 rows x 128 B)
    static constexpr int kQBytes = kChunks * kQChunk;
    static constexpr int kKVBytes = BT * D * 2;      // one K or V tile
    static constexpr int kKVChunk = BT * 128;        // bytes per K/V chunk
    static constexpr int kOffQ = 0;                  // Q staging
    static constexpr int kOffK = kQBytes;
    static constexpr int kOffV = kOffK + NS * kKVBytes;
    static constexpr int kOffBar = kOffV + NS * kKVBytes;
    // barriers: q_full, q_free, q_tmem[2], k_full[NS], v_full[NS], kv_empty[NS],
    // s_full[2], p_full[2], drain
    static constexpr int kNumBars = 4 + 3 * NS + 2 + 2 + 1;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
    // tensor memory columns: S/P buffers 0 and 1 (S_g in buffer g mod 2, then
    // P_g, bf16 pairs, over its first BT/2 columns), two Q buffers (bf16 pairs,
    // D/2 columns each; query tile n uses buffer n mod 2), the O accumulator
    static constexpr int kTmemS = 0;
    static constexpr int kTmemQ = 2 * BT;
    static constexpr int kTmemO = 2 * BT + D;
    static constexpr int kTmemCols = (kTmemO + D) <= 256 ? 256 : 512;
    static_assert(kTmemO + D <= 512, "tensor memory budget");
    static constexpr uint32_t kIdescQK = idesc_bf16_f32(128, BT, false);
    static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, true);
};

struct Bars {
    uint64_t* q_full;
    uint64_t* q_free;
    uint64_t* q_tmem;
    uint64_t* k_full;
    uint64_t* v_full;
    uint64_t* kv_empty;
    uint64_t* s_full;
    uint64_t* p_full;
    uint64_t* drain;
};

// Query tile u of the flattened (b*H + h, i) space: its head's tile shape and
// the grid origin of the query tile.
struct QueryTile {
    int bh, i, slot, pt, ph, pw, t0, y0, x0;
};

__device__ __forceinline__ QueryTile query_tile(const AttnParams& p, int u) {
    QueryTile q;
    q.bh = u / p.nT;
    q.i = u - q.bh * p.nT;
    q.slot = p.head_shape[q.bh % p.H];
    q.pt = p.shape[q.slot][0];
    q.ph = p.shape[q.slot][1];
    q.pw = p.shape[q.slot][2];
    tile_origin(q.i, q.pt, q.ph, q.pw, p.Hs, p.Ws, q.t0, q.y0, q.x0);
    return q;
}

// Persistent schedule: CTA c handles query tiles u = c, c + G, c + 2G, ...
// (G = gridDim.x); its n-th tile is u_n.  Every query tile has k key tiles, so
// the key tiles of all of the CTA's query tiles form one stream, g = n*k + j.
// Barrier phase bookkeeping (each barrier completes once per use):
//   q_full      Q of tile n is in the staging buffer: parity n & 1
//   q_free      the softmax has copied Q of tile n out of the staging: n & 1
//   q_tmem[b]   Q of tile n (b = n mod 2) is in tensor memory: (n >> 1) & 1
//   k_full/v_full[st], kv_empty[st]   key tile g in stage st = g mod NS, fill
//               g / NS: parity (g / NS) & 1 (kv_empty: P_g V_g is done)
//   s_full[b], p_full[b]   S_g / P_g in buffer b = g mod 2: (g >> 1) & 1
// Every barrier's next completion needs its waiter to have passed its current
// wait, so no waiter is two phases behind.  The softmax also reads "P_g V_g
// done" from kv_empty (O rescale within a tile; before the epilogue); the
// next completion of that stage is P_{g+NS} V_{g+NS}, which needs the softmax
// to have finished tile g+NS.  Ordering inside the tensor pipe: Q K_{g+2}^T
// overwrites S buffer g mod 2 after P_g V_g has read P_g, and the first
// P V product of tile n+1 overwrites O (accumulate off) after the softmax has
// read O for tile n's epilogue (it issues only once P of that product is
// ready, which the softmax writes after the epilogue).  Q of tile n+2 is
// written into the Q buffer of tile n after the softmax has seen the last S
// of tile n+1, so every product of tile n is done.
template <int D, int BT, int NS>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_persistent_kernel(const __grid_constant__ AttnParams p) {
    using C = Cfg<D, BT, NS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;
    uint64_t* bar_base = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    Bars bars;
    bars.q_full = bar_base;
    bars.q_free = bar_base + 1;
    bars.q_tmem = bar_base + 2;
    bars.k_full = bar_base + 4;
    bars.v_full = bars.k_full + NS;
    bars.kv_empty = bars.v_full + NS;
    bars.s_full = bars.kv_empty + NS;
    bars.p_full = bars.s_full + 2;
    bars.drain = bars.p_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int k = p.k;
    const int G = gridDim.x;
    const int n_tiles = blockIdx.x < p.total_tiles ? (p.total_tiles - 1 - blockIdx.x) / G + 1 : 0;
    const int total_g = n_tiles * k;

    // ---------------------------------------------------------------- set-up
    if (threadIdx.x == 0) {
        mbar_init(bars.q_full, 1);
        mbar_init(bars.q_free, 4);
        mbar_init(&bars.q_tmem[0], 4);
        mbar_init(&bars.q_tmem[1], 4);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&bars.k_full[s], 1);
            mbar_init(&bars.v_full[s], 1);
            mbar_init(&bars.kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars.s_full[b], 1);
            mbar_init(&bars.p_full[b], 4);
        }
        mbar_init(bars.drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
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
        int q_issued = 0, k_fills = 0, v_fills = 0;  // copies issued (lane 0)
        if (lane == 0)
            for (int sl = 0; sl < kMaxShapes; ++sl) {
                tma_prefetch_desc(&p.tmQ[sl]);
                tma_prefetch_desc(&p.tmK[sl]);
                tma_prefetch_desc(&p.tmV[sl]);
            }
        bool ok = true;
        for (int n = 0; n < n_tiles && ok; ++n) {
            const QueryTile qt = query_tile(p, blockIdx.x + n * G);
            if (lane == 0) {
                // Q of tile n into the staging buffer, once the softmax has
                // copied Q of tile n-1 out of it
                int good = 1;
                if (n > 0) good = wait_bar(bars.q_free, (n - 1) & 1, p, abort_flag);
                if (good) {
                    mbar_arrive_expect_tx(bars.q_full, BT * D * 2);
#pragma unroll
                    for (int c = 0; c < C::kChunks; ++c)
                        tma_load_5d(sQ + c * C::kQChunk, &p.tmQ[qt.slot], bars.q_full, c * 64,
                                    qt.x0, qt.y0, qt.t0, qt.bh);
                    q_issued = n + 1;
                } else {
                    ok = false;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            const int32_t* irow = p.idx ? p.idx + ((size_t)qt.bh * p.nT + qt.i) * k : nullptr;
            for (int j0 = 0; j0 < k && ok; j0 += 32) {
                int my_t = 0;
                if (j0 + lane < k) {
                    my_t = irow ? irow[j0 + lane] : j0 + lane;
                    if (my_t < 0 || my_t >= p.nT) {
                        atomicCAS(p.status, 0, (int)VEDA_ERR_BAD_INDEX);
                        my_t = 0;
                    }
                }
                const int cnt = min(32, k - j0);
                for (int jj = 0; jj < cnt; ++jj) {
                    const int t = __shfl_sync(0xffffffffu, my_t, jj);
                    int good = 1;
                    if (lane == 0) {
                        const int g = n * k + j0 + jj, st = g % NS, f = g / NS;
                        int t0, y0, x0;
                        tile_origin(t, qt.pt, qt.ph, qt.pw, p.Hs, p.Ws, t0, y0, x0);
                        if (f > 0) good = wait_bar(&bars.kv_empty[st], (f - 1) & 1, p, abort_flag);
                        if (good) {
                            mbar_arrive_expect_tx(&bars.k_full[st], C::kKVBytes);
#pragma unroll
                            for (int c = 0; c < C::kChunks; ++c)
                                tma_load_5d(sK + st * C::kKVBytes + c * C::kKVChunk,
                                            &p.tmK[qt.slot], &bars.k_full[st], c * 64, x0, y0, t0,
                                            qt.bh);
                            k_fills = g + 1;
                            mbar_arrive_expect_tx(&bars.v_full[st], C::kKVBytes);
#pragma unroll
                            for (int c = 0; c < C::kChunks; ++c)
                                tma_load_5d(sV + st * C::kKVBytes + c * C::kKVChunk,
                                            &p.tmV[qt.slot], &bars.v_full[st], c * 64, x0, y0, t0,
                                            qt.bh);
                            v_fills = g + 1;
                        }
                    }
                    good = __shfl_sync(0xffffffffu, good, 0);
                    if (!good) {
                        ok = false;
                        break;
                    }
                }
            }
        }
        if (lane == 0) {
            // Drain: every copy this warp issued has landed before the CTA exits.
            if (q_issued > 0) drain_bar(bars.q_full, (q_issued - 1) & 1, p);
            for (int st = 0; st < NS; ++st) {
                if (st < k_fills) drain_bar(&bars.k_full[st], ((k_fills - 1 - st) / NS) & 1, p);
                if (st < v_fills) drain_bar(&bars.v_full[st], ((v_fills - 1 - st) / NS) & 1, p);
            }
        }
    } else if (warp == 1) {
        // ============================================================ MMA issuer
        if (elect_one()) {
            const uint32_t tS = tbase + C::kTmemS;
            const uint32_t tQ = tbase + C::kTmemQ;
            const uint32_t tO = tbase + C::kTmemO;
            const uint32_t k_addr = smem_addr(sK);
            const uint32_t v_addr = smem_addr(sV);
            // S_g = Q_n K_g^T into buffer g & 1: A = Q_n from tensor memory, B = K
            // tile (K-major, swizzled).  The first product of a query tile waits
            // for its Q in tensor memory.  (qk_g, qk_n, qk_j): the next product
            // to issue, as a global key-tile index, query tile and key tile;
            // counters instead of divisions keep the issue path short.
            int qk_g = 0, qk_n = 0, qk_j = 0;
            auto issue_next_qk = [&]() -> bool {
                const int st = qk_g % NS, b = qk_g & 1;
                if (qk_j == 0 &&
                    !wait_bar(&bars.q_tmem[qk_n & 1], (qk_n >> 1) & 1, p, abort_flag))
                    return false;
                if (!wait_bar(&bars.k_full[st], (qk_g / NS) & 1, p, abort_flag)) return false;
                tc_fence_after();
                const uint32_t tq = tQ + (qk_n & 1) * (D / 2);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const int c = ks >> 2, w = ks & 3;
                    const uint64_t bd = smem_desc_sw128(
                        k_addr + st * C::kKVBytes + c * C::kKVChunk + w * 32, 16, 1024);
                    mma_bf16_ts(tS + b * BT, tq + ks * 8, bd, C::kIdescQK, ks > 0 ? 1u : 0u);
                }
                mma_commit(&bars.s_full[b]);
                ++qk_g;
                if (++qk_j == k) {
                    qk_j = 0;
                    ++qk_n;
                }
                return true;
            };
            bool ok = true;
            if (total_g > 0) ok = issue_next_qk();
            if (ok && total_g > 1) ok = issue_next_qk();
            int j = 0;  // key tile of g within its query tile
            for (int g = 0; g < total_g && ok; ++g) {
                const int st = g % NS, b = g & 1;
                if (!wait_bar(&bars.p_full[b], (g >> 1) & 1, p, abort_flag)) break;
                if (!wait_bar(&bars.v_full[st], (g / NS) & 1, p, abort_flag)) break;
                tc_fence_after();
                // O += P_g V_g (the first key tile of a query tile starts O afresh)
#pragma unroll
                for (int ks = 0; ks < BT / 16; ++ks) {
                    const uint64_t bd =
                        smem_desc_sw128(v_addr + st * C::kKVBytes + ks * 2048, C::kKVChunk, 1024);
                    mma_bf16_ts(tO, tS + b * BT + ks * 8, bd, C::kIdescPV,
                                (j > 0 || ks > 0) ? 1u : 0u);
                }
                mma_commit(&bars.kv_empty[st]);
                if (++j == k) j = 0;
                if (qk_g < total_g && !issue_next_qk()) break;
            }
            // Drain: all tensor-core work issued by this thread has completed.
            mma_commit(bars.drain);
            drain_bar(bars.drain, 0, p);
        }
        __syncwarp();
    } else if (warp >= kSoftmaxWarp0) {
        // ============================================================ softmax
        const int wq = warp & 3;                 // TMEM lane quarter of this warp
        const int r = wq * 32 + lane;            // query row of the tile
        const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tS = tbase + lane_off + C::kTmemS;
        const uint32_t tQ = tbase + lane_off + C::kTmemQ;
        const uint32_t tO = tbase + lane_off + C::kTmemO;
        const float c2 = p.scale_log2;
        bool ok = true;
        // Q of tile n: staging (128-byte swizzle) -> tensor memory buffer n & 1;
        // rows BT..127 are zero rows of the 128-row MMA operand.
        auto copy_q = [&](int n) -> bool {
            if (!warp_wait_bar(bars.q_full, n & 1, p, abort_flag)) return false;
            // lane 0 saw the copy land; each lane observes the completed phase
            // itself (one test, which succeeds) before reading the staged tile
            if (!__all_sync(0xffffffffu, mbar_try_wait(bars.q_full, n & 1))) return false;
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c) {
                uint32_t v[32];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    uint4 x = make_uint4(0, 0, 0, 0);
                    if (r < BT)
                        x = *reinterpret_cast<const uint4*>(sQ + c * C::kQChunk + r * 128 +
                                                            ((u ^ (r & 7)) << 4));
                    v[4 * u] = x.x;
                    v[4 * u + 1] = x.y;
                    v[4 * u + 2] = x.z;
                    v[4 * u + 3] = x.w;
                }
                tmem_st_32x32b_x32(tQ + (n & 1) * (D / 2) + c * 32, v);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars.q_tmem[n & 1]);
                mbar_arrive(bars.q_free);  // the staging buffer may take the next Q
            }
            return true;
        };
        if (n_tiles > 0) ok = copy_q(0);
        for (int n = 0; n < n_tiles && ok; ++n) {
            float m_run = 0.f, l_run = 0.f;
            for (int j = 0; j < k && ok; ++j) {
                const int g = n * k + j, b = g & 1;
                if (!warp_wait_bar(&bars.s_full[b], (g >> 1) & 1, p, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t s[BT];
#pragma unroll
                for (int cc = 0; cc < BT / 32; ++cc)
                    tmem_ld_32x32b_x32(tS + b * BT + cc * 32,
                                       *reinterpret_cast<uint32_t(*)[32]>(&s[cc * 32]));
                tmem_wait_ld();

                // row max: eight independent three-input chains, then a short tree
                float mx8[8];
#pragma unroll
                for (int a = 0; a < 8; ++a)
                    mx8[a] = fmaxf(__uint_as_float(s[a]), __uint_as_float(s[a + 8]));
#pragma unroll
                for (int e = 16; e < BT; e += 16)
#pragma unroll
                    for (int a = 0; a < 8; ++a)
                        mx8[a] = fmax3(mx8[a], __uint_as_float(s[e + a]),
                                       __uint_as_float(s[e + 8 + a]));
                const float mx = fmaxf(fmax3(mx8[0], mx8[1], mx8[2]),
                                       fmax3(fmax3(mx8[3], mx8[4], mx8[5]), mx8[6], mx8[7]));
                const float m_tile = mx * c2;
                bool need;
                float m_use, alpha;
                if (j == 0) {
                    need = false;
                    m_use = m_tile;
                    alpha = 0.f;
                } else {
                    const float m_new = fmaxf(m_run, m_tile);
                    need = m_new > m_run + kRescaleThreshold;
                    m_use = need ? m_new : m_run;
                    alpha = need ? fast_exp2(m_run - m_new) : 1.f;
                }
                // p = 2^(s*c2 - m): packed fp32x2 scale-and-shift, MUFU ex2, four
                // independent packed partial sums
                uint32_t pk[BT / 2];
                const uint64_t c2x2 = f32x2_pack(c2, c2);
                const uint64_t negm = f32x2_pack(-m_use, -m_use);
                uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int e = 0; e < BT; e += 2) {
                    const uint64_t x = f32x2_fma(
                        f32x2_pack(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), c2x2, negm);
                    float x0, x1;
                    f32x2_unpack(x, x0, x1);
                    const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
                    acc[(e >> 1) & 3] = f32x2_add(acc[(e >> 1) & 3], f32x2_pack(p0, p1));
                    pk[e / 2] = pack_bf16x2(p0, p1);
                }
                float a0, a1, a2, a3;
                f32x2_unpack(f32x2_add(acc[0], acc[1]), a0, a1);
                f32x2_unpack(f32x2_add(acc[2], acc[3]), a2, a3);
                const float lsum = (a0 + a2) + (a1 + a3);
                l_run = (j == 0) ? lsum : fmaf(l_run, alpha, lsum);
                m_run = m_use;

                if (__any_sync(0xffffffffu, need)) {
                    // rescale O: P_{g-1} V_{g-1} must have landed first
                    if (!warp_wait_bar(&bars.kv_empty[(g - 1) % NS], ((g - 1) / NS) & 1, p,
                                       abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll 1
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t o[32];
                        tmem_ld_32x32b_x32(tO + cc * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st_32x32b_x32(tO + cc * 32, o);
                    }
                }
                // P_g over S_g in buffer b (this thread has read its row of S_g)
#pragma unroll
                for (int cc = 0; cc < BT / 64; ++cc)
                    tmem_st_32x32b_x32(tS + b * BT + cc * 32,
                                       *reinterpret_cast<uint32_t(*)[32]>(&pk[cc * 32]));
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0 && !(p.withhold_arrive && g == 0 && wq == 0))
                    mbar_arrive(&bars.p_full[b]);
            }
            if (!ok) break;
            // the next query tile's Q goes into tensor memory now, so its first
            // products run on the tensor core while this tile's epilogue runs
            if (n + 1 < n_tiles && !copy_q(n + 1)) {
                ok = false;
                break;
            }
            const int g_last = n * k + k - 1;
            if (!warp_wait_bar(&bars.kv_empty[g_last % NS], (g_last / NS) & 1, p, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // ------------------------------------------------ epilogue of tile n
            // O / l -> bf16, written straight from registers: row r is one token,
            // its D channels 2*D contiguous bytes
            const QueryTile qt = query_tile(p, blockIdx.x + n * G);
            const float inv_l = 1.f / l_run;
            const int lt = r / (qt.ph * qt.pw), lh = (r / qt.pw) % qt.ph, lw = r % qt.pw;
            const int tok = ((qt.t0 + lt) * p.Hs + (qt.y0 + lh)) * p.Ws + (qt.x0 + lw);
            uint4* orow = reinterpret_cast<uint4*>(p.O + ((size_t)qt.bh * p.N + tok) * D);
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                tmem_ld_32x32b_x32(tO + cc * 32, o);
                tmem_wait_ld();
                if (r < BT) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv_l,
                                          __uint_as_float(o[8 * q + 1]) * inv_l);
                        v.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv_l,
                                          __uint_as_float(o[8 * q + 3]) * inv_l);
                        v.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv_l,
                                          __uint_as_float(o[8 * q + 5]) * inv_l);
                        v.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv_l,
                                          __uint_as_float(o[8 * q + 7]) * inv_l);
                        orow[cc * 4 + q] = v;
                    }
                }
            }
            if (p.lse != nullptr && r < BT)
                p.lse[(size_t)qt.bh * p.N + tok] = (m_run + log2f(l_run)) * 0.69314718055994531f;
            // the next tile's first P V product overwrites O: the reads above are
            // complete (wait::ld) before this warp's next P-ready arrival
            tc_fence_before();
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, C::kTmemCols);
    }
}

// ---------------------------------------------------------------- host side
template <int D, int BT, int NS>
veda_status launch_cfg(const AttnParams& prm, const Problem& pr, cudaStream_t s) {
    using C = Cfg<D, BT, NS>;
    static_assert(C::kSmemBytes <= 227 * 1024, "shared memory budget");
    cudaError_t err = cudaFuncSetAttribute(sparse_attn_persistent_kernel<D, BT, NS>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           C::kSmemBytes);
    if (err != cudaSuccess) return cuda_check(err, "sparse_attn smem attribute");
    // persistent: one CTA per SM (shared memory allows one), at most one per tile
    const int total = prm.total_tiles;
    const int ctas = total < sm_count() ? total : sm_count();
    sparse_attn_persistent_kernel<D, BT, NS><<<ctas, kThreads, C::kSmemBytes, s>>>(prm);
    return cuda_check(cudaGetLastError(), "sparse_attn launch");
}

}  // namespace

veda_status launch_sparse_attn_persistent(const Problem& pr, const uint16_t* Q,
                                          const uint16_t* K, const uint16_t* V,
                                          const int32_t* idx, int k, uint16_t* O, float* lse,
                                          int* status, cudaStream_t s) {
    AttnParams prm;
    memset(&prm, 0, sizeof(prm));
    for (int sh = 0; sh < pr.nshapes; ++sh) {
        veda_status st;
        if ((st = encode_tile_map(&prm.tmQ[sh], Q, pr, pr.shape[sh])) != VEDA_OK) return st;
        if ((st = encode_tile_map(&prm.tmK[sh], K, pr, pr.shape[sh])) != VEDA_OK) return st;
        if ((st = encode_tile_map(&prm.tmV[sh], V, pr, pr.shape[sh])) != VEDA_OK) return st;
        for (int q = 0; q < 3; ++q) prm.shape[sh][q] = pr.shape[sh][q];
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
    prm.total_tiles = pr.B * pr.H * pr.nT;
    prm.scale_log2 = pr.scale * 1.4426950408889634f;
    prm.wait_limit_ns = wait_limit_ns();
    // Test hook for the bounded waits: with VEDA_TEST_WITHHOLD_ARRIVE set, one
    // arrival never happens, the MMA issuer's wait runs out and every CTA
    // reports VEDA_ERR_TIMEOUT (nothing in normal use sets the variable).
    prm.withhold_arrive = getenv("VEDA_TEST_WITHHOLD_ARRIVE") != nullptr ? 1 : 0;
    if (pr.d == 128 && pr.Bt == 128) return launch_cfg<128, 128, 3>(prm, pr, s);
    if (pr.d == 128 && pr.Bt == 64) return launch_cfg<128, 64, 4>(prm, pr, s);
    if (pr.d == 64 && pr.Bt == 128) return launch_cfg<64, 128, 4>(prm, pr, s);
    return launch_cfg<64, 64, 4>(prm, pr, s);
}

}  // namespace veda
