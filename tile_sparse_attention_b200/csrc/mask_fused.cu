// mask_fused.cu -- tile scores and head-aware Top-k in one kernel: the score
// matrix S never leaves the chip.
//
// "Veda: Scalable Video Diffusion via Distilled Sparse Attention" (project
// page), "Attention Structure Distillation", Estimator (S[i, j] = sum over
// the three statistics of <q~_{i,s}, k~_{j,s}>) and Execution (Top-k per query
// tile gives the tile mask); "Theoretical Rationale" 4.  Ties go to the lower
// tile index; -0.0 and +0.0 tie.
//
// One CTA owns 128 query tiles (rows) of one head and walks the key tiles in
// chunks of 128 columns:
//   * warp 4 lane 0 streams 32-wide K blocks of q^ (the CTA's rows) and k^ (the
//     chunk's rows) by TMA into a 3-stage ring -- the same operands, in the
//     same order, as the stand-alone score kernel, so every S value is
//     bit-identical to it;
//   * warp 5 owns 256 TMEM columns (two S chunk buffers); one elected lane issues the
//     kind::tf32 MMAs of chunk c into buffer c mod 2;
//   * warps 0..3 (thread = row) read their row of chunk c out of tensor memory,
//     release the buffer, and fold the 128 scores into a running Top-k: a
//     binary min-heap of k entries per row in shared memory.  An entry is the
//     64-bit value (order key << 32) | (2^32 - 1 - j): a larger value is a
//     larger score, or an equal score at a lower index, so "keep the k largest
//     values" is exactly the selection rule, and the values of a row are all
//     distinct: the heap ends with the same k entries whatever order the
//     columns arrive in.  A column replaces the heap minimum only if its value
//     is larger.
//   * the chunks are visited starting with the block's own diagonal chunk and
//     then in rotation: where nearby key tiles score high (local attention),
//     the heap threshold is high from the start and later columns rarely
//     enter the heap (each entry costs a sift through shared memory, taken by
//     the whole warp whenever one of its rows needs it).
// After the last chunk the shared memory of the TMA ring holds one bitmap row
// of nT bits per query tile; each warp then writes the ascending index lists
// (ballot prefix counts over bitmap words) and the 0/1 mask rows of 32 rows.
//
// Limits: k <= 128 (heap capacity) and nT <= 6144 (bitmaps fit the ring).
// Waits are bounded (VEDA_ERR_TIMEOUT in the status word, then a bounded drain
// of the copies and products in flight before tensor memory is freed).
#include "internal.h"
#include "kernel_common.cuh"
#include "ptx.cuh"

namespace veda {

namespace {

constexpr int kThreadsF = 192;
constexpr int kSelectWarps = 4;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kStagesF = 3;
constexpr int kTileBytesF = 128 * 128;            // 128 rows x 32 fp32
constexpr int kStageBytesF = 2 * kTileBytesF;     // A and B
constexpr int kRingBytesF = kStagesF * kStageBytesF;
constexpr int kMaxKF = 128;
constexpr int kMaxNTF = kRingBytesF * 8 / 128;    // bitmap rows of nT bits in the ring
constexpr int kOffHeap = kRingBytesF;
constexpr int kOffBarF = kOffHeap + kMaxKF * 128 * 8;
// barriers: full[3], empty[3], s_full[2], s_free[2], drain
constexpr int kNumBarsF = 2 * kStagesF + 2 + 2 + 1;
constexpr int kOffMiscF = kOffBarF + kNumBarsF * 8;
constexpr int kSmemBytesF = kOffMiscF + 16 + 1024;  // + alignment slack
static_assert(kSmemBytesF <= 227 * 1024, "shared memory budget");
static_assert(kMaxNTF == 6144, "bitmap capacity");
// kind::tf32, fp32 accumulate, both operands K-major, M = N = 128
constexpr uint32_t kIdescTF32F = (1u << 4) | (2u << 7) | (2u << 10) | ((128u >> 3) << 17) |
                                 ((128u >> 4) << 24);

struct __align__(64) FusedParams {
    CUtensorMap mapA;  // q^: rows B*H*nT, K = 9d
    CUtensorMap mapB;  // k^
    uint8_t* mask;     // [B,H,nT,nT] or null
    int32_t* idx;      // [B,H,nT,k]
    int* status;
    int nT, k, kblocks, nchunks;
    unsigned long long wait_limit_ns;
};

// Min-heap of `n` entries of one row: entry e at heap[e * 128] (entry-major,
// so the 128 rows' heaps interleave and equal positions hit distinct banks).
__device__ __forceinline__ void sift_down(uint64_t* heap, int pos, int n) {
    const uint64_t v = heap[pos * 128];
    while (true) {
        int c = 2 * pos + 1;
        if (c >= n) break;
        uint64_t cv = heap[c * 128];
        if (c + 1 < n) {
            const uint64_t c2 = heap[(c + 1) * 128];
            if (c2 < cv) {
                cv = c2;
                ++c;
            }
        }
        if (cv >= v) break;
        heap[pos * 128] = cv;
        pos = c;
    }
    heap[pos * 128] = v;
}

// Builds the heap from its n entries; returns the minimum.
__device__ __noinline__ uint64_t heap_build(uint64_t* heap, int n) {
    for (int s = n / 2 - 1; s >= 0; --s) sift_down(heap, s, n);
    return heap[0];
}

// Replaces the minimum by v (> minimum); returns the new minimum.
__device__ __noinline__ uint64_t heap_replace_min(uint64_t* heap, uint64_t v, int n) {
    heap[0] = v;
    sift_down(heap, 0, n);
    return heap[0];
}

__global__ void __launch_bounds__(kThreadsF, 1)
    score_topk_kernel(const __grid_constant__ FusedParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* heap_all = reinterpret_cast<uint64_t*>(smem + kOffHeap);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBarF);
    uint64_t* empty = full + kStagesF;
    uint64_t* s_full = empty + kStagesF;
    uint64_t* s_free = s_full + 2;
    uint64_t* drain = s_free + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMiscF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMiscF + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i0 = blockIdx.x * 128, bh = blockIdx.y;
    const int nT = p.nT, k = p.k, KB = p.kblocks, NC = p.nchunks;
    const int rowA = bh * nT + i0;
    const int c0 = blockIdx.x % NC;  // the block's diagonal chunk comes first

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesF; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_free[b], kSelectWarps);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == kProducerWarp) {
        // ============================================================ producer
        if (lane == 0) {
            tma_prefetch_desc(&p.mapA);
            tma_prefetch_desc(&p.mapB);
            int issued = 0;
            bool ok = true;
            for (int t = 0; t < NC && ok; ++t) {
                const int c = (c0 + t) % NC;  // chunk visited at step t
                const int rowB = bh * nT + c * 128;
                for (int kb = 0; kb < KB; ++kb) {
                    const int g = t * KB + kb, st = g % kStagesF, n = g / kStagesF;
                    if (n > 0 && !wait_bar(&empty[st], (n - 1) & 1, p, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t* a = smem + st * kStageBytesF;
                    mbar_arrive_expect_tx(&full[st], kStageBytesF);
                    tma_load_2d(a, &p.mapA, &full[st], kb * 32, rowA);
                    tma_load_2d(a + kTileBytesF, &p.mapB, &full[st], kb * 32, rowB);
                    issued = g + 1;
                }
            }
            // drain: every copy issued has landed before the CTA exits
            for (int st = 0; st < kStagesF; ++st)
                if (st < issued) drain_bar(&full[st], ((issued - 1 - st) / kStagesF) & 1, p);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ============================================================ MMA issuer
        if (elect_one()) {
            const uint32_t base = smem_addr(smem);
            bool ok = true;
            for (int t = 0; t < NC && ok; ++t) {
                const int b = t & 1;
                // buffer b was last read by the select warps at step t - 2
                if (t >= 2 && !wait_bar(&s_free[b], ((t - 2) >> 1) & 1, p, abort_flag)) break;
                for (int kb = 0; kb < KB; ++kb) {
                    const int g = t * KB + kb, st = g % kStagesF;
                    if (!wait_bar(&full[st], (g / kStagesF) & 1, p, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a = base + st * kStageBytesF;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = smem_desc_sw128(a + kk * 32, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(a + kTileBytesF + kk * 32, 16, 1024);
                        mma_tf32_ss(tbase + b * 128, ad, bd, kIdescTF32F, (kb > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&empty[st]);
                }
                if (ok) mma_commit(&s_full[b]);
            }
            // drain: all tensor-core work issued by this thread has completed
            mma_commit(drain);
            drain_bar(drain, 0, p);
        }
        __syncwarp();
    } else {
        // ============================================================ select
        const int r = warp * 32 + lane;  // query tile i0 + r; TMEM lane r
        const int i = i0 + r;
        const bool active = i < nT;
        const uint32_t taddr = tbase + (static_cast<uint32_t>(warp * 32) << 16);
        uint64_t* heap = heap_all + r;
        int count = 0;
        uint64_t thr = 0;  // heap minimum once the heap holds k entries
        bool ok = true;
        for (int t = 0; t < NC; ++t) {
            const int b = t & 1;
            const int c = (c0 + t) % NC;  // chunk of step t
            if (!warp_wait_bar(&s_full[b], (t >> 1) & 1, p, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t v[128];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
                tmem_ld_32x32b_x32(taddr + b * 128 + cc * 32,
                                   *reinterpret_cast<uint32_t(*)[32]>(&v[cc * 32]));
            tmem_wait_ld();
            // the chunk is in registers: buffer b may take chunk c + 2
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[b]);
            if (active) {
                const int jn = min(128, nT - c * 128);
#pragma unroll
                for (int e = 0; e < 128; ++e) {
                    if (e < jn) {
                        const uint32_t j = static_cast<uint32_t>(c * 128 + e);
                        const uint64_t val =
                            (static_cast<uint64_t>(order_key(__uint_as_float(v[e]))) << 32) |
                            (0xffffffffu - j);
                        if (count < k) {
                            heap[count * 128] = val;
                            if (++count == k) thr = heap_build(heap, k);
                        } else if (val > thr) {
                            thr = heap_replace_min(heap, val, k);
                        }
                    }
                }
            }
        }
        // all select threads get here (every wait is bounded); the output is
        // written only if the four warps saw every chunk
        if (named_barrier_and(1, kSelectWarps * 32, ok)) {
            // Every product is done (the last s_full commit covers them) and
            // every copy has landed, so the ring's shared memory is free: one
            // bitmap row of W words per query tile.
            const int W = (nT + 31) / 32;
            uint32_t* bm = reinterpret_cast<uint32_t*>(smem);
            uint32_t* my = bm + (size_t)r * W;
            for (int w = 0; w < W; ++w) my[w] = 0u;
            if (active)
                for (int e = 0; e < count; ++e) {
                    const uint32_t j = 0xffffffffu - static_cast<uint32_t>(heap[e * 128]);
                    my[j >> 5] |= 1u << (j & 31);
                }
            named_barrier_sync(2, kSelectWarps * 32);
            // warp w writes rows w, w + 4, ...: ascending index list by ballot
            // prefix counts over bitmap words, and the mask row
            for (int rr = warp; rr < 128; rr += kSelectWarps) {
                const int ii = i0 + rr;
                if (ii >= nT) break;
                const uint32_t* row = bm + (size_t)rr * W;
                int32_t* out = p.idx + ((size_t)bh * nT + ii) * k;
                int pos = 0;
                for (int w0 = 0; w0 < W; w0 += 32) {
                    const uint32_t word = (w0 + lane < W) ? row[w0 + lane] : 0u;
                    const int cnt = __popc(word);
                    int incl = cnt;
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const int t = __shfl_up_sync(0xffffffffu, incl, off);
                        if (lane >= off) incl += t;
                    }
                    int o = pos + incl - cnt;
                    uint32_t bits = word;
                    while (bits) {
                        const int bpos = __ffs(bits) - 1;
                        out[o++] = (w0 + lane) * 32 + bpos;
                        bits &= bits - 1;
                    }
                    pos += __shfl_sync(0xffffffffu, incl, 31);
                }
                if (p.mask != nullptr) {
                    uint8_t* mrow = p.mask + ((size_t)bh * nT + ii) * nT;
                    for (int j = lane; j < nT; j += 32)
                        mrow[j] = static_cast<uint8_t>((row[j >> 5] >> (j & 31)) & 1u);
                }
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tbase, 256);
    }
}

}  // namespace

bool fused_mask_supported(const Problem& pr) {
    return pr.k >= 1 && pr.k <= kMaxKF && pr.nT <= kMaxNTF;
}

veda_status launch_score_topk(const Problem& pr, const float* qext, const float* kext,
                              uint8_t* mask, int32_t* idx, int* status, cudaStream_t s) {
    if (!fused_mask_supported(pr))
        return fail(VEDA_ERR_UNSUPPORTED, "fused mask: needs k <= 128 and nT <= 6144");
    FusedParams prm;
    memset(&prm, 0, sizeof(prm));
    const long long rows = (long long)pr.B * pr.H * pr.nT;
    const int kx = 9 * pr.d;
    veda_status st;
    if ((st = encode_rows_map(&prm.mapA, qext, rows, kx)) != VEDA_OK) return st;
    if ((st = encode_rows_map(&prm.mapB, kext, rows, kx)) != VEDA_OK) return st;
    prm.mask = mask;
    prm.idx = idx;
    prm.status = status;
    prm.nT = pr.nT;
    prm.k = pr.k;
    prm.kblocks = kx / 32;
    prm.nchunks = (pr.nT + 127) / 128;
    prm.wait_limit_ns = wait_limit_ns();
    cudaError_t err = cudaFuncSetAttribute(score_topk_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytesF);
    if (err != cudaSuccess) return cuda_check(err, "fused mask smem attribute");
    dim3 grid((pr.nT + 127) / 128, pr.B * pr.H);
    score_topk_kernel<<<grid, kThreadsF, kSmemBytesF, s>>>(prm);
    return cuda_check(cudaGetLastError(), "fused mask launch");
}

}  // namespace veda
