// topk.cu -- head-aware Top-k of the tile scores into a 0/1 tile mask and an
// ascending index list.
//
// "Veda: Scalable Video Diffusion via Distilled Sparse Attention" (project
// page), "Attention Structure Distillation", Execution: Top-k selection per
// query tile produces the tile mask handed to the tile-skipping kernel.  Ties
// go to the lower tile index; -0.0 and +0.0 tie.
//
// One warp per row, in one of two kernels.  Rows of up to 2048 scores stay in
// registers (topk_reg_kernel, described where it is defined).  Longer rows are
// read with 16-byte loads (up to sixteen in flight per lane) into shared
// memory (topk_kernel).  The selection is exact and integer-valued:
//   1. Bucketing: every score goes to one of 256 buckets spread linearly over
//      [row min, row max].  The bucket index is computed with correctly
//      rounded fp32 operations from the score alone, so it is a
//      non-decreasing function of the score (equal scores, -0.0 and +0.0
//      included, share a bucket).  A histogram gives the bucket b* holding
//      the k-th largest score and the count of scores in higher buckets, all
//      of which are selected.
//   2. Within b* (a handful of scores for smooth score distributions), the
//      exact threshold key K* (order-preserving 32-bit keys, larger score ->
//      larger key) and how many keys equal to K* are kept: pairwise ranks for
//      at most 32 candidates, else a radix select (8 bits per pass, most
//      significant varying bit first) over the candidates.
//   3. One pass in ascending index order emits the mask (four bytes per lane
//      store) and, through warp ballots and prefix pop-counts, the index list
//      already sorted; of the keys equal to K*, the lowest-index ones are kept.
#include <cfloat>

#include "internal.h"
#include "kernel_common.cuh"

namespace veda {

namespace {

constexpr int kBins = 256;     // buckets of the first pass and radix digits
constexpr int kCandCap = 256;  // candidate keys kept in shared memory per row

struct TopkParams {
    const float* S;
    uint8_t* mask;
    int32_t* idx;
    long long rows;
    int nT, k;
};

// Shared-memory words of one warp: the row (rounded up to groups of four),
// the histogram, the candidate list and its counter (padded to 16 bytes).
__host__ __device__ inline size_t topk_warp_words(int nT) {
    return (size_t)4 * ((nT + 3) >> 2) + kBins + kCandCap + 4;
}

// Bucket of score x among kBins linear buckets over [mn, mn + kBins / inv];
// inv >= 0 and finite, x >= mn, so t is finite and >= 0 and the result is
// non-decreasing in x.
__device__ __forceinline__ int bucket_of(float x, float mn, float inv) {
    const float t = __fmul_rn(__fsub_rn(x, mn), inv);
    return t < (float)(kBins - 1) ? (int)t : kBins - 1;
}

// The bin holding the kr-th largest element of a kBins-bin histogram (bins in
// ascending value order, so the scan runs from the top bin down); `above`
// receives the number of elements in higher bins.  kr must not exceed the
// histogram's total.
__device__ __forceinline__ uint32_t select_bin(const uint32_t* hist, int kr, int lane,
                                               uint32_t& above) {
    // lane l owns bins 255-8l ... 248-8l (descending)
    uint32_t cnt[8];
    uint32_t local = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        cnt[e] = hist[kBins - 1 - 8 * lane - e];
        local += cnt[e];
    }
    uint32_t incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    const uint32_t hit = __ballot_sync(0xffffffffu, incl >= (uint32_t)kr);
    const int src = __ffs(hit) - 1;
    uint32_t bin = 0, ab = 0;
    if (lane == src) {
        uint32_t run = incl - local;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (run + cnt[e] >= (uint32_t)kr) {
                bin = kBins - 1 - 8 * lane - e;
                ab = run;
                break;
            }
            run += cnt[e];
        }
    }
    above = __shfl_sync(0xffffffffu, ab, src);
    return __shfl_sync(0xffffffffu, bin, src);
}

// Exact radix select of the kr-th largest key among the candidates.  each(f)
// calls f(key) for every candidate key held by this lane (a shared-memory list
// or registers).  Returns that key; kr becomes the number of candidates equal
// to it that are kept (ranked among equal keys).
template <class Each>
__device__ uint32_t radix_select(const Each& each, int& kr, uint32_t* hist, int lane) {
    // Bits above the highest bit in which the candidates differ are common to
    // all of them: the passes start below them.
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    each([&](uint32_t key) {
        kmin = min(kmin, key);
        kmax = max(kmax, key);
    });
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, off));
    }
    const int top = 32 - __clz(kmin ^ kmax);  // number of bits that vary (0..32)
    uint32_t pmask = top == 32 ? 0u : ~((1u << top) - 1u);
    uint32_t prefix = kmin & pmask;
#pragma unroll 1
    for (int hi = top; hi > 0; hi -= 8) {
        const int shift = hi >= 8 ? hi - 8 : 0;
        const uint32_t dmask = hi >= 8 ? 255u : (1u << hi) - 1u;
        for (int b = lane; b < kBins; b += 32) hist[b] = 0;
        __syncwarp();
        each([&](uint32_t key) {
            if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
        });
        __syncwarp();
        uint32_t above;
        const uint32_t digit = select_bin(hist, kr, lane, above);
        kr -= (int)above;
        prefix |= digit << shift;
        pmask |= dmask << shift;
        __syncwarp();
    }
    return prefix;
}

// Threshold among the c candidate keys of cand[] (c >= kr >= 1): pairwise
// ranks for at most 32 (the lanes holding the kr-th largest key see fewer than
// kr larger keys and at least kr larger-or-equal ones), else a radix select.
// Returns the key; kr becomes the number of keys equal to it that are kept.
__device__ __forceinline__ uint32_t candidate_threshold(const uint32_t* cand, int c, int& kr,
                                                       uint32_t* hist, int lane) {
    const unsigned full = 0xffffffffu;
    if (c <= 32) {
        const uint32_t mine = lane < c ? cand[lane] : 0u;
        int gt = 0, eq = 0;
        for (int m = 0; m < c; ++m) {
            const uint32_t o = __shfl_sync(full, mine, m);
            gt += o > mine ? 1 : 0;
            eq += o == mine ? 1 : 0;
        }
        const bool hit = lane < c && gt < kr && gt + eq >= kr;
        const int src = __ffs(__ballot_sync(full, hit)) - 1;
        kr -= __shfl_sync(full, gt, src);
        return __shfl_sync(full, mine, src);
    }
    return radix_select(
        [&](auto&& f) {
            for (int j = lane; j < c; j += 32) f(cand[j]);
        },
        kr, hist, lane);
}

// Score of an order key (inverse of order_key; the key of -0.0 maps to +0.0).
__device__ __forceinline__ float key_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key ^ 0x80000000u) : ~key);
}

// LOADS: 16-byte loads in flight per lane (16 for long rows; 8 keeps the
// register count, and so the warps per SM, up for rows of up to 1024 scores).
template <int WARPS, int LOADS>
__global__ void __launch_bounds__(WARPS * 32) topk_kernel(const __grid_constant__ TopkParams p) {
    extern __shared__ __align__(16) uint32_t smem_u[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * WARPS + warp;
    if (row >= p.rows) return;
    const int nT = p.nT;
    const int nG = (nT + 3) >> 2;  // groups of four scores
    uint32_t* base = smem_u + (size_t)warp * topk_warp_words(nT);
    float* vals = reinterpret_cast<float*>(base);
    float4* v4 = reinterpret_cast<float4*>(base);
    uint32_t* hist = base + 4 * nG;
    uint32_t* cand = hist + kBins;
    uint32_t* ncand = cand + kCandCap;
    const float* srow = p.S + row * nT;
    const unsigned full = 0xffffffffu;

    // ---- 1. the row into shared memory, with its min and max
    float mn = INFINITY, mx = -INFINITY;
    if ((nT & 3) == 0) {  // rows start on 16-byte boundaries (S is 16-byte aligned)
        const float4* s4 = reinterpret_cast<const float4*>(srow);
        for (int g = lane; g < nG; g += 32 * LOADS) {
            float4 t[LOADS];
#pragma unroll
            for (int u = 0; u < LOADS; ++u)
                if (g + 32 * u < nG) t[u] = __ldcs(s4 + g + 32 * u);
#pragma unroll
            for (int u = 0; u < LOADS; ++u)
                if (g + 32 * u < nG) {
                    v4[g + 32 * u] = t[u];
                    mn = fminf(mn, fminf(fminf(t[u].x, t[u].y), fminf(t[u].z, t[u].w)));
                    mx = fmaxf(mx, fmaxf(fmaxf(t[u].x, t[u].y), fmaxf(t[u].z, t[u].w)));
                }
        }
    } else {
        for (int j = lane; j < nT; j += 32 * 8) {
            float t[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (j + 32 * u < nT) t[u] = __ldcs(srow + j + 32 * u);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (j + 32 * u < nT) {
                    vals[j + 32 * u] = t[u];
                    mn = fminf(mn, t[u]);
                    mx = fmaxf(mx, t[u]);
                }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(full, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(full, mx, off));
    }
    // kBins buckets over [mn, mx]; a zero or non-finite range puts every score
    // in bucket 0 (still exact: the candidates are then the whole row)
    const float range = __fsub_rn(mx, mn);
    const float inv = (range > 0.f && range <= FLT_MAX) ? fminf((float)kBins / range, FLT_MAX) : 0.f;
    __syncwarp();

    // ---- 2. bucket histogram and the bucket of the k-th largest score
    for (int b = lane; b < kBins; b += 32) hist[b] = 0;
    __syncwarp();
    for (int g = lane; g < nG; g += 32) {
        const float4 x = v4[g];
        const int j = 4 * g;
        atomicAdd(&hist[bucket_of(x.x, mn, inv)], 1u);
        if (j + 1 < nT) atomicAdd(&hist[bucket_of(x.y, mn, inv)], 1u);
        if (j + 2 < nT) atomicAdd(&hist[bucket_of(x.z, mn, inv)], 1u);
        if (j + 3 < nT) atomicAdd(&hist[bucket_of(x.w, mn, inv)], 1u);
    }
    __syncwarp();
    uint32_t above;
    const int bstar = (int)select_bin(hist, p.k, lane, above);
    int kr = p.k - (int)above;  // rank of the k-th largest score within bucket b*
    __syncwarp();

    // ---- 3. the keys of bucket b* (in any order), and the exact threshold among them
    if (lane == 0) *ncand = 0;
    __syncwarp();
    for (int g = lane; g < nG; g += 32) {
        const float4 x = v4[g];
        const float xe[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if (4 * g + e < nT && bucket_of(xe[e], mn, inv) == bstar) {
                const uint32_t pos = atomicAdd(ncand, 1u);
                if (pos < (uint32_t)kCandCap) cand[pos] = order_key(xe[e]);
            }
    }
    __syncwarp();
    const int c = (int)*ncand;  // candidates (warp-uniform)
    uint32_t thr;
    if (c <= kCandCap) {
        thr = candidate_threshold(cand, c, kr, hist, lane);
    } else {
        thr = radix_select(
            [&](auto&& f) {
                for (int j = lane; j < nT; j += 32) {
                    const float x = vals[j];
                    if (bucket_of(x, mn, inv) == bstar) f(order_key(x));
                }
            },
            kr, hist, lane);
    }

    // scores above and equal to the threshold, compared as floats (order keys
    // compare like the scores, with -0.0 equal to +0.0)
    const float tv = key_value(thr);

    // ---- 4. mask and ascending index list; keep the kr lowest-index scores equal to tv
    const unsigned lt_mask = (1u << lane) - 1u;
    int eq_seen = 0, sel_seen = 0;
    int32_t* irow = p.idx + row * p.k;
    uint8_t* mrow = p.mask ? p.mask + row * nT : nullptr;
    for (int g0 = 0; g0 < nG; g0 += 32) {
        const int g = g0 + lane;
        const bool gv = g < nG;
        const float4 x = gv ? v4[g] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float xe[4] = {x.x, x.y, x.z, x.w};
        bool eq[4], sel[4];
        int neq = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool valid = gv && 4 * g + e < nT;
            eq[e] = valid && xe[e] == tv;
            sel[e] = valid && xe[e] > tv;
            neq += eq[e] ? 1 : 0;
        }
        if (__any_sync(full, neq > 0)) {
            int r = eq_seen, tot = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const unsigned b = __ballot_sync(full, eq[e]);
                r += __popc(b & lt_mask);
                tot += __popc(b);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (eq[e] && r < kr) sel[e] = true;
                r += eq[e] ? 1 : 0;
            }
            eq_seen += tot;
        }
        int pos = sel_seen, tot = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const unsigned b = __ballot_sync(full, sel[e]);
            pos += __popc(b & lt_mask);
            tot += __popc(b);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if (sel[e]) {
                if (pos < p.k) irow[pos] = 4 * g + e;  // exactly k are selected
                ++pos;
            }
        sel_seen += tot;
        if (mrow != nullptr) {
            if ((nT & 3) == 0) {
                if (gv)
                    reinterpret_cast<uchar4*>(mrow)[g] =
                        make_uchar4(sel[0] ? 1 : 0, sel[1] ? 1 : 0, sel[2] ? 1 : 0, sel[3] ? 1 : 0);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (gv && 4 * g + e < nT) mrow[4 * g + e] = sel[e] ? 1 : 0;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Rows of up to 2048 scores (1024 for rows that do not start on a 16-byte
// boundary): the row stays in registers.
//
// Lane l holds the float4 groups l, l + 32, ... (G of them), and the next row
// is loaded into the same registers once the current one's bucket-b* scores
// have been gathered, so its loads land while this row's selection finishes.
// The scores become 7-bit buckets,
//   bucket(x) = floor(127 * sat(fl(fl(x - min) * inv))),  inv = 1 / (max - min),
// a non-decreasing function of x in which equal scores (-0.0 and +0.0
// included) share a bucket; `sat` clamps to [0, 1] and sends NaN to 0, so the
// padding of a short last group (NaN) lands in bucket 0 and never counts.  Four
// buckets are packed per register, each byte with its top bit set, so that
// byte-wise `b >= P` is the top bit of the byte after subtracting P (no byte
// borrows).  Then, with no shared-memory histogram:
//   1. a binary search over the 128 buckets, each probe a byte-parallel count
//      reduced over the warp, gives the bucket b* of the k-th largest score and
//      the number of scores above it;
//   2. the scores of bucket b* (a handful for smooth rows) are gathered from
//      the registers and their exact threshold found as in the kernel above
//      (pairwise ranks for up to 32, an 8-bit radix select otherwise, or over
//      the whole row, re-read, if more than kCandCap share the bucket); the
//      chosen ones of b* are marked in a bitmap;
//   3. the selected bytes of every packed word (buckets above b*, plus the
//      bitmap) give per-lane counts, whose prefix over the warp comes from four
//      counts per 32-bit word in one scan, and the index list is written
//      already ascending.

constexpr int kRegWarps = 4;
constexpr int kRegMaxG = 16;                 // rows of up to 128 * 16 = 2048 scores
constexpr int kRegBitmapWords = 2048 / 32;   // one bit per score
// per warp: histogram, candidate keys, candidate indices, bitmap, counter (16 B)
constexpr int kRegWarpWords = kBins + 2 * kCandCap + kRegBitmapWords + 4;

// Bit pattern of fl(2^23 + 127 t), rounded toward zero, for t = sat(fl(fl(x - mn) * inv)):
// its low byte is floor(127 t), the bucket of x (0..127).
__device__ __forceinline__ uint32_t bucket7_bits(float x, float mn, float inv) {
    float d, t, r;
    asm("sub.rn.f32 %0, %1, %2;" : "=f"(d) : "f"(x), "f"(mn));
    asm("mul.rn.sat.f32 %0, %1, %2;" : "=f"(t) : "f"(d), "f"(inv));
    asm("fma.rz.f32 %0, %1, 0f42FE0000, 0f4B000000;" : "=f"(r) : "f"(t));  // 127, 2^23
    return __float_as_uint(r);
}

__device__ __forceinline__ uint32_t bucket7(float x, float mn, float inv) {
    return bucket7_bits(x, mn, inv) & 0x7fu;
}

// Four buckets in one word, each byte 0x80 | bucket.
__device__ __forceinline__ uint32_t pack_buckets(const float4& v, float mn, float inv) {
    const uint32_t lo = __byte_perm(bucket7_bits(v.x, mn, inv), bucket7_bits(v.y, mn, inv), 0x0040);
    const uint32_t hi = __byte_perm(bucket7_bits(v.z, mn, inv), bucket7_bits(v.w, mn, inv), 0x0040);
    return __byte_perm(lo, hi, 0x5410) | 0x80808080u;
}

// Group g (scores 4g .. 4g+3) of a row; scores beyond nT read as NaN.
template <bool ALIGNED>
__device__ __forceinline__ float4 load_group(const float* srow, int g, int nT) {
    const float qnan = __int_as_float(0x7fc00000);
    if (ALIGNED) {
        if (4 * g < nT) return __ldg(reinterpret_cast<const float4*>(srow) + g);
        return make_float4(qnan, qnan, qnan, qnan);
    }
    const int j = 4 * g;
    float4 v;
    v.x = j < nT ? __ldg(srow + j) : qnan;
    v.y = j + 1 < nT ? __ldg(srow + j + 1) : qnan;
    v.z = j + 2 < nT ? __ldg(srow + j + 2) : qnan;
    v.w = j + 3 < nT ? __ldg(srow + j + 3) : qnan;
    return v;
}

__device__ __forceinline__ float min3f(float a, float b, float c) {
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));  // NaN inputs ignored
    return r;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

template <int G, bool ALIGNED>
__global__ void __launch_bounds__(kRegWarps * 32, G >= 12 ? 4 : G >= 5 ? 5 : 6)
    topk_reg_kernel(const __grid_constant__ TopkParams p) {
    __shared__ __align__(16) uint32_t smem_u[kRegWarps * kRegWarpWords];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t* hist = smem_u + warp * kRegWarpWords;
    uint32_t* ck = hist + kBins;
    int32_t* ci = reinterpret_cast<int32_t*>(ck + kCandCap);
    uint32_t* bm = reinterpret_cast<uint32_t*>(ci + kCandCap);
    uint32_t* ncand = bm + kRegBitmapWords;
    const unsigned full = 0xffffffffu;
    const int nT = p.nT, k = p.k;
    const long long stride = (long long)gridDim.x * kRegWarps;
    long long row = (long long)blockIdx.x * kRegWarps + warp;

    float4 v[G];
    if (row < p.rows) {
#pragma unroll
        for (int u = 0; u < G; ++u) v[u] = load_group<ALIGNED>(p.S + row * nT, 32 * u + lane, nT);
    }
    for (; row < p.rows; row += stride) {
        const float* srow = p.S + row * nT;
        // ---- row min and max (the NaN padding is ignored)
        float mn0 = INFINITY, mn1 = INFINITY, mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int u = 0; u < G; ++u) {
            mn0 = min3f(mn0, v[u].x, v[u].y);
            mn1 = min3f(mn1, v[u].z, v[u].w);
            mx0 = max3f(mx0, v[u].x, v[u].y);
            mx1 = max3f(mx1, v[u].z, v[u].w);
        }
        float mn = fminf(mn0, mn1), mx = fmaxf(mx0, mx1);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(full, mn, off));
            mx = fmaxf(mx, __shfl_xor_sync(full, mx, off));
        }
        // a zero or non-finite range puts every score in bucket 0 (still exact)
        const float range = __fsub_rn(mx, mn);
        const float inv =
            (range > 0.f && range <= FLT_MAX) ? fminf(__frcp_rn(range), FLT_MAX) : 0.f;
        uint32_t pk[G];
#pragma unroll
        for (int u = 0; u < G; ++u) pk[u] = pack_buckets(v[u], mn, inv);
        for (int w = lane; w < kRegBitmapWords; w += 32) bm[w] = 0u;
        if (lane == 0) *ncand = 0u;

        // ---- 1. bucket b* of the k-th largest score:
        //      count(bucket >= lo) >= k > count(bucket >= hi)
        uint32_t lo = 0, hi = 128, above = 0;
#pragma unroll 1
        for (int it = 0; it < 7; ++it) {
            const uint32_t mid = (lo + hi) >> 1;
            const uint32_t T = mid * 0x01010101u;
            uint32_t acc[3] = {0u, 0u, 0u};  // three independent chains; bytes stay <= G
#pragma unroll
            for (int u = 0; u < G; ++u) acc[u % 3] += ((pk[u] - T) & 0x80808080u) >> 7;
            const uint32_t a = acc[0] + acc[1] + acc[2];
            const uint32_t c = __reduce_add_sync(full, (a * 0x01010101u) >> 24);
            if (c >= (uint32_t)k) {
                lo = mid;
            } else {
                hi = mid;
                above = c;
            }
        }
        const uint32_t bstar = lo;
        int kr = k - (int)above;  // rank of the k-th largest score within bucket b*
        __syncwarp();

        // ---- 2. the scores of bucket b*, taken from the registers
        const uint32_t Bs = bstar * 0x01010101u;
#pragma unroll
        for (int u = 0; u < G; ++u) {
            const uint32_t z = (pk[u] ^ Bs) & 0x7f7f7f7fu;
            uint32_t eq = ~(z + 0x7f7f7f7fu) & 0x80808080u;
            if (eq != 0u) {
                const int j0 = 4 * (32 * u + lane);
                do {
                    const int e = (__ffs(eq) - 8) >> 3;
                    eq &= eq - 1u;
                    if (j0 + e < nT) {
                        const float x =
                            e == 0 ? v[u].x : e == 1 ? v[u].y : e == 2 ? v[u].z : v[u].w;
                        const uint32_t pos = atomicAdd(ncand, 1u);
                        if (pos < (uint32_t)kCandCap) {
                            ck[pos] = order_key(x);
                            ci[pos] = j0 + e;
                        }
                    }
                } while (eq != 0u);
            }
        }
        // ---- the next row's loads go out now and land during the rest of this one
        {
            const long long nrow = row + stride;
            if (nrow < p.rows) {
#pragma unroll
                for (int u = 0; u < G; ++u)
                    v[u] = load_group<ALIGNED>(p.S + nrow * nT, 32 * u + lane, nT);
            }
        }
        __syncwarp();
        const int c = (int)*ncand;  // >= kr
        uint32_t thr;
        if (c <= kCandCap) {
            thr = candidate_threshold(ck, c, kr, hist, lane);
        } else {
            thr = radix_select(
                [&](auto&& f) {
                    for (int j = lane; j < nT; j += 32) {
                        const float x = __ldg(srow + j);
                        if (bucket7(x, mn, inv) == bstar) f(order_key(x));
                    }
                },
                kr, hist, lane);
        }
        // kr is now the number of scores equal to the threshold that are kept
        // (the lowest-index ones); mark the chosen scores of b* in the bitmap
        if (c <= kCandCap) {
            int neq = 0;
            for (int j = lane; j < c; j += 32) neq += ck[j] == thr ? 1 : 0;
            neq = __reduce_add_sync(full, neq);
            for (int j = lane; j < c; j += 32) {
                const uint32_t key = ck[j];
                const int id = ci[j];
                bool keep = key > thr;
                if (key == thr) {
                    if (neq == kr) {
                        keep = true;
                    } else {
                        int r = 0;
                        for (int m = 0; m < c; ++m) r += (ck[m] == thr && ci[m] < id) ? 1 : 0;
                        keep = r < kr;
                    }
                }
                if (keep) atomicOr(&bm[id >> 5], 1u << (id & 31));
            }
        } else {
            int eq_seen = 0;
            const unsigned lt = (1u << lane) - 1u;
            for (int j0 = 0; j0 < nT; j0 += 32) {
                const int j = j0 + lane;
                bool gt = false, eq = false;
                if (j < nT) {
                    const float x = __ldg(srow + j);
                    if (bucket7(x, mn, inv) == bstar) {
                        const uint32_t key = order_key(x);
                        gt = key > thr;
                        eq = key == thr;
                    }
                }
                const unsigned be = __ballot_sync(full, eq);
                const bool keep = gt || (eq && eq_seen + __popc(be & lt) < kr);
                eq_seen += __popc(be);
                const unsigned bk = __ballot_sync(full, keep);
                if (lane == 0) bm[j0 >> 5] = bk;
            }
        }
        __syncwarp();

        // ---- 3. selected bytes, their prefix over the warp, the ascending list and the mask
        const uint32_t T = (bstar + 1u) * 0x01010101u;
        constexpr int NS = (G + 3) / 4;
        uint32_t sw[NS];
#pragma unroll
        for (int q = 0; q < NS; ++q) sw[q] = 0u;
#pragma unroll
        for (int u = 0; u < G; ++u) {
            const int g = 32 * u + lane;
            const uint32_t nib = (bm[g >> 3] >> (4 * (g & 7))) & 0xfu;  // chosen scores of b*
            const uint32_t m =
                ((pk[u] - T) & 0x80808080u) | (((nib * 0x00204081u) & 0x01010101u) << 7);
            pk[u] = m;
            sw[u >> 2] |= (uint32_t)__popc(m) << (8 * (u & 3));
        }
        uint32_t excl[NS], tot[NS];
#pragma unroll
        for (int q = 0; q < NS; ++q) {
            uint32_t incl = sw[q];
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t t = __shfl_up_sync(full, incl, off);
                if (lane >= off) incl += t;  // each byte <= 32 * 4: no carries between counts
            }
            excl[q] = incl - sw[q];
            tot[q] = __shfl_sync(full, incl, 31);
        }
        int32_t* irow = p.idx + row * k;
        int run = 0;
#pragma unroll
        for (int u = 0; u < G; ++u) {
            const int g = 32 * u + lane;
            int q = run + (int)((excl[u >> 2] >> (8 * (u & 3))) & 0xffu);
            run += (int)((tot[u >> 2] >> (8 * (u & 3))) & 0xffu);
            const uint32_t m = pk[u];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if ((m >> (8 * e + 7)) & 1u) {
                    if (q < k) irow[q] = 4 * g + e;  // exactly k are selected
                    ++q;
                }
        }
        if (p.mask != nullptr) {
            uint8_t* mrow = p.mask + row * nT;
#pragma unroll
            for (int u = 0; u < G; ++u) {
                const int g = 32 * u + lane;
                const uint32_t flags = (pk[u] >> 7) & 0x01010101u;
                if (ALIGNED) {
                    if (4 * g < nT) reinterpret_cast<uint32_t*>(mrow)[g] = flags;
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (4 * g + e < nT) mrow[4 * g + e] = (uint8_t)((flags >> (8 * e)) & 1u);
                }
            }
        }
        __syncwarp();
    }
}

template <int G, bool ALIGNED>
veda_status launch_topk_reg(const TopkParams& prm, cudaStream_t s) {
    static const int per_sm = [] {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, topk_reg_kernel<G, ALIGNED>,
                                                          kRegWarps * 32, 0) != cudaSuccess || n < 1)
            n = 1;
        return n;
    }();
    const long long need = (prm.rows + kRegWarps - 1) / kRegWarps;
    const long long cap = (long long)per_sm * sm_count();
    const unsigned blocks = (unsigned)(need < cap ? need : cap);
    topk_reg_kernel<G, ALIGNED><<<blocks, kRegWarps * 32, 0, s>>>(prm);
    return cuda_check(cudaGetLastError(), "topk launch");
}

template <bool ALIGNED>
veda_status launch_topk_reg_g(const TopkParams& prm, int g, cudaStream_t s) {
    if (g <= 1) return launch_topk_reg<1, ALIGNED>(prm, s);
    if (g <= 2) return launch_topk_reg<2, ALIGNED>(prm, s);
    if (g <= 4) return launch_topk_reg<4, ALIGNED>(prm, s);
    if (g <= 5) return launch_topk_reg<5, ALIGNED>(prm, s);
    if constexpr (!ALIGNED) {
        return launch_topk_reg<8, ALIGNED>(prm, s);  // rows of up to 1024 scores
    } else {
        if (g <= 8) return launch_topk_reg<8, ALIGNED>(prm, s);
        if (g <= 12) return launch_topk_reg<12, ALIGNED>(prm, s);
        if (g <= 15) return launch_topk_reg<15, ALIGNED>(prm, s);
        return launch_topk_reg<16, ALIGNED>(prm, s);
    }
}

template <int W, int LOADS>
veda_status launch_topk_w(const TopkParams& prm, cudaStream_t s) {
    const size_t smem = topk_warp_words(prm.nT) * sizeof(uint32_t) * W;
    cudaError_t err = cudaFuncSetAttribute(topk_kernel<W, LOADS>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return cuda_check(err, "topk smem attribute");
    const unsigned blocks = (unsigned)((prm.rows + W - 1) / W);
    topk_kernel<W, LOADS><<<blocks, W * 32, smem, s>>>(prm);
    return cuda_check(cudaGetLastError(), "topk launch");
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
    // rows of up to 2048 scores (1024 when they do not start on 16-byte
    // boundaries: their single-score loads need more registers): in registers,
    // 128 scores per float4 group of every lane; longer rows: in shared
    // memory, four warps (rows) per block up to 4096 tiles (<= 74 KB), one
    // above (<= 66 KB at the 16384-tile limit)
    if ((pr.nT & 3) == 0 && pr.nT <= 128 * kRegMaxG)
        return launch_topk_reg_g<true>(prm, (pr.nT + 127) / 128, s);
    if ((pr.nT & 3) != 0 && pr.nT <= 1024)
        return launch_topk_reg_g<false>(prm, (pr.nT + 127) / 128, s);
    if (pr.nT <= 4096) return launch_topk_w<4, 16>(prm, s);
    return launch_topk_w<1, 16>(prm, s);
}

}  // namespace veda
