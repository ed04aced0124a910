// host_pipeline.cu -- the whole layer from host memory, pipelined by heads.
//
// Every step of the layer is independent per (batch entry, head) (project
// page, "Attention Structure Distillation": statistics, scores, Top-k and the
// tile-skipping attention of a head read only that head's Q, K, V), so the
// layer can run in chunks of heads: while chunk g is computed on the caller's
// stream, chunk g+1 is copied in on one copy stream and chunk g-1 is copied
// out on another.  The copies use cudaMemcpyAsync; with page-locked host
// buffers they overlap the kernels and each other (the host link is full
// duplex).  The results are the same as one veda_forward call on the whole
// problem: each chunk runs the same kernels on its own heads.
#include <map>
#include <mutex>
#include <vector>

#include "internal.h"

namespace veda {

namespace {

struct CopyStreams {
    cudaStream_t in = nullptr;
    cudaStream_t out = nullptr;
};

std::mutex g_streams_mu;
std::map<int, CopyStreams> g_streams;  // one pair per device, kept for the process

veda_status copy_streams(CopyStreams* cs) {
    int dev = 0;
    veda_status st;
    if ((st = cuda_check(cudaGetDevice(&dev), "current device"))) return st;
    std::lock_guard<std::mutex> lock(g_streams_mu);
    auto it = g_streams.find(dev);
    if (it == g_streams.end()) {
        CopyStreams n;
        if ((st = cuda_check(cudaStreamCreateWithFlags(&n.in, cudaStreamNonBlocking), "copy stream")))
            return st;
        if ((st = cuda_check(cudaStreamCreateWithFlags(&n.out, cudaStreamNonBlocking),
                             "copy stream")))
            return st;
        it = g_streams.emplace(dev, n).first;
    }
    *cs = it->second;
    return VEDA_OK;
}

// Events of one call, destroyed when the call returns (a destroyed event that
// is still pending is released once it completes).
struct EventSet {
    std::vector<cudaEvent_t> ev;
    ~EventSet() {
        for (cudaEvent_t e : ev) cudaEventDestroy(e);
    }
    veda_status make(cudaEvent_t* e) {
        veda_status st = cuda_check(cudaEventCreateWithFlags(e, cudaEventDisableTiming), "event");
        if (st == VEDA_OK) ev.push_back(*e);
        return st;
    }
};

}  // namespace

veda_status forward_host_impl(const veda_problem* p, const Problem& pr, const uint16_t* hQ,
                              const uint16_t* hK, const uint16_t* hV, const float* hWq,
                              const float* hWk, uint16_t* hO, float* hlse, uint16_t* dQ,
                              uint16_t* dK, uint16_t* dV, float* dWq, float* dWk, uint16_t* dO,
                              float* dlse, void* ws, int head_chunk, cudaStream_t s) {
    CopyStreams cs;
    veda_status st;
    if ((st = copy_streams(&cs))) return st;
    EventSet events;
    cudaEvent_t entry;
    if ((st = events.make(&entry))) return st;
    // device buffers may still be in use by earlier work on the caller's stream
    if ((st = cuda_check(cudaEventRecord(entry, s), "event record"))) return st;
    if ((st = cuda_check(cudaStreamWaitEvent(cs.in, entry, 0), "stream wait"))) return st;
    if ((st = cuda_check(cudaStreamWaitEvent(cs.out, entry, 0), "stream wait"))) return st;
    if ((st = cuda_check(cudaMemsetAsync(ws, 0, sizeof(int), s), "status reset"))) return st;
    // From here on copies may be queued on the copy streams: an error return
    // first makes the caller's stream wait for them (or, if even that fails,
    // waits on the host), so no copy touches the caller's buffers after the
    // caller's stream has completed.
    auto fail_joined = [&](veda_status err) -> veda_status {
        cudaEvent_t ein = nullptr, eout = nullptr;
        bool joined = events.make(&ein) == VEDA_OK && events.make(&eout) == VEDA_OK &&
                      cudaEventRecord(ein, cs.in) == cudaSuccess &&
                      cudaEventRecord(eout, cs.out) == cudaSuccess &&
                      cudaStreamWaitEvent(s, ein, 0) == cudaSuccess &&
                      cudaStreamWaitEvent(s, eout, 0) == cudaSuccess;
        if (!joined) {
            cudaStreamSynchronize(cs.in);
            cudaStreamSynchronize(cs.out);
        }
        return err;
    };

    const size_t tok = (size_t)pr.N * pr.d;  // elements of one head of Q, K, V or O
    const size_t wsz = (size_t)pr.d * pr.d;  // elements of one head's weight matrix
    for (int b = 0; b < pr.B; ++b) {
        for (int h0 = 0; h0 < pr.H; h0 += head_chunk) {
            const int hc = pr.H - h0 < head_chunk ? pr.H - h0 : head_chunk;
            veda_problem pc = *p;
            pc.B = 1;
            pc.H = hc;
            pc.tile_shapes = p->tile_shapes + 3 * h0;
            Problem sub;
            if ((st = make_problem(&pc, true, &sub))) return fail_joined(st);
            const size_t off = ((size_t)b * pr.H + h0) * tok;
            const size_t bytes = (size_t)hc * tok * sizeof(uint16_t);
            // in: this chunk's Q, K, V (and weights, once per head)
            if ((st = cuda_check(cudaMemcpyAsync(dQ + off, hQ + off, bytes, cudaMemcpyHostToDevice,
                                                 cs.in), "Q copy in")))
                return fail_joined(st);
            if ((st = cuda_check(cudaMemcpyAsync(dK + off, hK + off, bytes, cudaMemcpyHostToDevice,
                                                 cs.in), "K copy in")))
                return fail_joined(st);
            if ((st = cuda_check(cudaMemcpyAsync(dV + off, hV + off, bytes, cudaMemcpyHostToDevice,
                                                 cs.in), "V copy in")))
                return fail_joined(st);
            if (b == 0) {
                const size_t wb = (size_t)hc * wsz * sizeof(float);
                if ((st = cuda_check(cudaMemcpyAsync(dWq + h0 * wsz, hWq + h0 * wsz, wb,
                                                     cudaMemcpyHostToDevice, cs.in), "Wq copy in")))
                    return fail_joined(st);
                if ((st = cuda_check(cudaMemcpyAsync(dWk + h0 * wsz, hWk + h0 * wsz, wb,
                                                     cudaMemcpyHostToDevice, cs.in), "Wk copy in")))
                    return fail_joined(st);
            }
            cudaEvent_t landed, computed;
            if ((st = events.make(&landed)) || (st = events.make(&computed))) return fail_joined(st);
            if ((st = cuda_check(cudaEventRecord(landed, cs.in), "event record"))) return fail_joined(st);
            // compute: the whole layer on this chunk's heads
            if ((st = cuda_check(cudaStreamWaitEvent(s, landed, 0), "stream wait"))) return fail_joined(st);
            float* lse_c = dlse ? dlse + ((size_t)b * pr.H + h0) * pr.N : nullptr;
            if ((st = forward_impl(sub, dQ + off, dK + off, dV + off, dWq + h0 * wsz,
                                   dWk + h0 * wsz, dO + off, lse_c, nullptr, nullptr, ws, s)))
                return fail_joined(st);
            if ((st = cuda_check(cudaEventRecord(computed, s), "event record"))) return fail_joined(st);
            // out: this chunk's O (and lse)
            if ((st = cuda_check(cudaStreamWaitEvent(cs.out, computed, 0), "stream wait")))
                return fail_joined(st);
            if ((st = cuda_check(cudaMemcpyAsync(hO + off, dO + off, bytes, cudaMemcpyDeviceToHost,
                                                 cs.out), "O copy out")))
                return fail_joined(st);
            if (hlse != nullptr) {
                const size_t lo = ((size_t)b * pr.H + h0) * pr.N;
                if ((st = cuda_check(cudaMemcpyAsync(hlse + lo, dlse + lo,
                                                     (size_t)hc * pr.N * sizeof(float),
                                                     cudaMemcpyDeviceToHost, cs.out),
                                     "lse copy out")))
                    return fail_joined(st);
            }
        }
    }
    // the caller's stream completes only after the last copy out
    cudaEvent_t done;
    if ((st = events.make(&done))) return fail_joined(st);
    if ((st = cuda_check(cudaEventRecord(done, cs.out), "event record"))) return fail_joined(st);
    if ((st = cuda_check(cudaStreamWaitEvent(s, done, 0), "stream wait"))) return fail_joined(st);
    return VEDA_OK;
}

}  // namespace veda
