// index_check.cu -- optional validation of caller-supplied index lists.
//
// The tile-skipping attention reads, for query tile i, the key tiles listed in
// idx[b,h,i,:] ("Veda: Scalable Video Diffusion via Distilled Sparse Attention"
// (project page), "Attention Structure Distillation", Execution: the tile mask
// decides which K/V tiles are fetched).  The attention kernels always replace
// an out-of-range entry by tile 0 and report it; a repeated entry, though,
// would be fetched twice and counted twice in the softmax.  With the
// environment variable VEDA_DEBUG_CHECKS set (to anything but "0"),
// veda_sparse_attn first runs this kernel, which reports any row with an
// out-of-range or repeated entry as VEDA_ERR_BAD_INDEX in the status word
// (no trap: the status word is read back with veda_get_status).  The TMA
// coordinates of a copy are derived from a range-checked tile index, so they
// need no separate check.
#include <cstdlib>
#include <cstring>

#include "internal.h"

namespace veda {

namespace {

constexpr int kCheckWarps = 4;  // rows per block

// One warp per row: a bitmap of the row's tiles in shared memory; a tile seen
// twice (atomicOr finds its bit set) or outside [0, nT) marks the row bad.
__global__ void __launch_bounds__(kCheckWarps * 32)
    check_index_kernel(const int32_t* __restrict__ idx, long long rows, int k, int nT,
                       int* status) {
    extern __shared__ uint32_t seen_all[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kCheckWarps + warp;
    if (row >= rows) return;  // whole warp
    const int words = (nT + 31) >> 5;
    uint32_t* seen = seen_all + (size_t)warp * words;
    for (int w = lane; w < words; w += 32) seen[w] = 0u;
    __syncwarp();
    const int32_t* r = idx + row * k;
    bool bad = false;
    for (int j = lane; j < k; j += 32) {
        const int t = r[j];
        if (t < 0 || t >= nT) {
            bad = true;
        } else {
            const uint32_t bit = 1u << (t & 31);
            if (atomicOr(&seen[t >> 5], bit) & bit) bad = true;
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicCAS(status, 0, (int)VEDA_ERR_BAD_INDEX);
}

}  // namespace

bool debug_checks_enabled() {
    const char* env = getenv("VEDA_DEBUG_CHECKS");
    return env != nullptr && env[0] != '\0' && strcmp(env, "0") != 0;
}

veda_status launch_check_index(const int32_t* idx, long long rows, int k, int nT, int* status,
                               cudaStream_t s) {
    const size_t smem = (size_t)kCheckWarps * ((nT + 31) >> 5) * sizeof(uint32_t);
    const unsigned blocks = (unsigned)((rows + kCheckWarps - 1) / kCheckWarps);
    check_index_kernel<<<blocks, kCheckWarps * 32, smem, s>>>(idx, rows, k, nT, status);
    return cuda_check(cudaGetLastError(), "index check launch");
}

}  // namespace veda
