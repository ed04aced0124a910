// noalloc.cu -- a variant of veda_tile_score for callers that cannot allocate
// device memory.
//
// Some callers of this library have no way to obtain a device workspace: a
// host application embedded in another runtime that only hands it device
// pointers for the inputs and outputs, a plugin whose host forbids allocations
// after start-up, or a real-time loop that must not call cudaMalloc on its hot
// path because that call can synchronise the device.  For them,
// veda_tile_score_noalloc keeps its scratch (the status word and the projected
// statistics q~ and k~) in a fixed, file-scope device array instead of a
// caller-provided workspace.
//
// Properties:
//   * the array is kVedaNoallocScratchBytes (64 MiB); every GPU that loads the
//     library holds it until the process exits;
//   * problems that need more scratch than that are rejected with
//     VEDA_ERR_UNSUPPORTED before anything is launched;
//   * the first call on a device looks up the array's device address on that
//     device (cudaGetSymbolAddress, with that device current) and caches it;
//     make that first call before any stream capture;
//   * every call shares the one array, which keeps the last call's contents:
//     calls whose work overlaps on the GPU (other streams, other host threads)
//     race on it; the status word is cleared by each call;
//   * the device status word (VEDA_ERR_TIMEOUT when a bounded wait of the
//     score kernel gave up) lives in the array too: veda_noalloc_get_status
//     reads it back for the current device;
//   * nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <mutex>
#include <string>

#include "internal.h"

namespace {

constexpr size_t kVedaNoallocScratchBytes = size_t(64) << 20;
constexpr int kMaxDevices = 64;

// The scratch itself.  In host code this name is only a stand-in for the
// device symbol, never a device address: kernels receive the address that
// cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_veda_noalloc_scratch[kVedaNoallocScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

veda_status scratch_for_current_device(void** out) {
    int dev = -1;
    veda_status st = veda::cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
    if (st != VEDA_OK) return st;
    if (dev < 0 || dev >= kMaxDevices)
        return veda::fail(VEDA_ERR_UNSUPPORTED, "device ordinal out of range for the scratch table");
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* ptr = nullptr;
        cudaError_t err = cudaGetSymbolAddress(&ptr, g_veda_noalloc_scratch);
        if (err != cudaSuccess || ptr == nullptr)
            return veda::fail(VEDA_ERR_CUDA, std::string("cudaGetSymbolAddress of the scratch: ") +
                                                 cudaGetErrorString(err));
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return VEDA_OK;
}

}  // namespace

extern "C" {

size_t veda_noalloc_scratch_bytes(void) { return kVedaNoallocScratchBytes; }

veda_status veda_tile_score_noalloc(const veda_problem* p, const float* statsQ,
                                    const float* statsK, const float* Wq, const float* Wk,
                                    float* S, veda_stream_t stream) {
    veda::Problem pr;
    veda_status st;
    if ((st = veda::make_problem(p, false, &pr)) != VEDA_OK) return st;
    if ((st = veda::check_ptr(statsQ, "statsQ")) || (st = veda::check_ptr(statsK, "statsK")) ||
        (st = veda::check_ptr(Wq, "Wq")) || (st = veda::check_ptr(Wk, "Wk")) ||
        (st = veda::check_ptr(S, "S")))
        return st;
    // Same scratch layout as veda_tile_score's workspace: status word, q^, k^.
    const size_t stats = veda::projected_bytes(pr);
    const size_t need = VEDA_STATUS_BYTES + 2 * stats;
    if (need > kVedaNoallocScratchBytes)
        return veda::fail(VEDA_ERR_UNSUPPORTED,
                          "veda_tile_score_noalloc needs " + std::to_string(need) +
                              " bytes of scratch, more than its fixed " +
                              std::to_string(kVedaNoallocScratchBytes) +
                              " bytes; use veda_tile_score with a workspace");
    void* scratch = nullptr;
    if ((st = scratch_for_current_device(&scratch)) != VEDA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    char* base = static_cast<char*>(scratch);
    float* qt = reinterpret_cast<float*>(base + VEDA_STATUS_BYTES);
    float* kt = reinterpret_cast<float*>(base + VEDA_STATUS_BYTES + stats);
    if ((st = veda::cuda_check(cudaMemsetAsync(base, 0, VEDA_STATUS_BYTES, s), "status reset")))
        return st;
    int* status = reinterpret_cast<int*>(base);
    if ((st = veda::launch_project_pair(pr, statsQ, statsK, Wq, Wk, qt, kt, status, s))) return st;
    return veda::launch_score(pr, qt, kt, S, status, s);
}

veda_status veda_noalloc_get_status(veda_stream_t stream, int32_t* device_status) {
    if (device_status == nullptr) return veda::fail(VEDA_ERR_INVALID_ARG, "device_status is NULL");
    void* scratch = nullptr;
    veda_status st;
    if ((st = scratch_for_current_device(&scratch)) != VEDA_OK) return st;
    if ((st = veda::cuda_check(cudaStreamSynchronize((cudaStream_t)stream), "stream sync")))
        return st;
    return veda::cuda_check(
        cudaMemcpy(device_status, scratch, sizeof(int32_t), cudaMemcpyDeviceToHost),
        "status read");
}

}  // extern "C"
