// monarch_host.cu -- monarch_attn_fwd_host_pipelined: the host-buffer entry
// point with the copies overlapped with the computation (include/monarch_attn.h).
//
// The (batch, head) problems are independent, so the call splits them into
// chunks of consecutive batch-heads ([B][heads][N][d] keeps each chunk
// contiguous) and pipelines: the upload of chunk c+1 runs while chunk c is
// computed and chunk c-1 is downloaded.  Uploads and downloads use two
// streams of their own (one pair per device, kept), so both copy directions
// run at once.
#include <cuda_runtime.h>

#include <cstdint>
#include <initializer_list>
#include <mutex>
#include <vector>

#include "../../include/monarch_attn.h"

namespace {

// Upload and download streams and the call's events, created once per device
// and kept (creating them costs about as much as a chunk's copy).  A call
// holds its device's lock from its first copy to its final synchronisation,
// so calls from several host threads on one device run one after another and
// never share an event while it is in use.
struct CopyState {
    cudaStream_t up = nullptr, down = nullptr;
    std::vector<cudaEvent_t> ev;  // grown as calls need more, never destroyed
    std::mutex mu;
};
constexpr int kMaxDevices = 64;
CopyState g_copy[kMaxDevices];

// The device's copy state with at least `nev` events; the caller holds cs->mu.
int copy_state(int dev, size_t nev, CopyState **out) {
    CopyState &c = g_copy[dev];
    if (!c.up && cudaStreamCreateWithFlags(&c.up, cudaStreamNonBlocking) != cudaSuccess) {
        c.up = nullptr;
        return MONARCH_ERR_CUDA;
    }
    if (!c.down && cudaStreamCreateWithFlags(&c.down, cudaStreamNonBlocking) != cudaSuccess) {
        c.down = nullptr;
        return MONARCH_ERR_CUDA;
    }
    while (c.ev.size() < nev) {
        cudaEvent_t e = nullptr;
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return MONARCH_ERR_CUDA;
        c.ev.push_back(e);
    }
    *out = &c;
    return MONARCH_OK;
}

}  // namespace

extern "C" int monarch_attn_fwd_host_pipelined(const void *h_q, const void *h_k, const void *h_v, void *h_out,
                                               void *d_q, void *d_k, void *d_v, void *d_out, int B, int heads,
                                               int T, int H, int W, int d, int factorisation, int tile_h,
                                               int tile_w, int dtype, int nchunks, void *stream) {
    if (!h_q || !h_k || !h_v || !h_out || !d_q || !d_k || !d_v || !d_out) return MONARCH_ERR_INVALID_ARG;
    if (B < 1 || heads < 1 || T < 1 || H < 1 || W < 1 || nchunks < 1) return MONARCH_ERR_INVALID_ARG;
    if (dtype != MONARCH_DTYPE_F32 && dtype != MONARCH_DTYPE_BF16 && dtype != MONARCH_DTYPE_F16)
        return MONARCH_ERR_INVALID_ARG;
    const long long bh = static_cast<long long>(B) * heads;
    const long long n = bh < nchunks ? bh : nchunks;
    const size_t es = dtype == MONARCH_DTYPE_F32 ? 4 : 2;
    const size_t per_bh = static_cast<size_t>(T) * H * W * d * es;
    // each chunk's call validates its own slices; the whole output buffer may
    // not overlap a whole input buffer either
    const size_t total = static_cast<size_t>(bh) * per_bh;
    const uintptr_t o = reinterpret_cast<uintptr_t>(d_out);
    for (const void *in : {static_cast<const void *>(d_q), static_cast<const void *>(d_k),
                           static_cast<const void *>(d_v)}) {
        const uintptr_t x = reinterpret_cast<uintptr_t>(in);
        if (x < o + total && o < x + total) return MONARCH_ERR_INVALID_ARG;
    }
    cudaStream_t compute = static_cast<cudaStream_t>(stream);
    int devi = 0;
    if (cudaGetDevice(&devi) != cudaSuccess || devi < 0 || devi >= kMaxDevices) return MONARCH_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_copy[devi].mu);
    CopyState *cs = nullptr;
    if (copy_state(devi, static_cast<size_t>(2 * n + 1), &cs) != MONARCH_OK) return MONARCH_ERR_CUDA;
    CopyState &s = *cs;
    const std::vector<cudaEvent_t> &ev = s.ev;
    // the computation must not start before earlier work on the caller's stream
    // is done with the device buffers: uploads wait for it
    cudaEvent_t start = ev[2 * n];
    if (cudaEventRecord(start, compute) != cudaSuccess || cudaStreamWaitEvent(s.up, start, 0) != cudaSuccess)
        return MONARCH_ERR_CUDA;
    int st = MONARCH_OK;
    for (long long c = 0; c < n && st == MONARCH_OK; ++c) {
        const long long b0 = bh * c / n, b1 = bh * (c + 1) / n;
        const size_t off = static_cast<size_t>(b0) * per_bh, bytes = static_cast<size_t>(b1 - b0) * per_bh;
        auto dev = [&](void *p) { return static_cast<void *>(static_cast<uint8_t *>(p) + off); };
        auto host = [&](const void *p) { return static_cast<const void *>(static_cast<const uint8_t *>(p) + off); };
        cudaEvent_t in = ev[2 * c], out = ev[2 * c + 1];
        if (cudaMemcpyAsync(dev(d_q), host(h_q), bytes, cudaMemcpyHostToDevice, s.up) != cudaSuccess ||
            cudaMemcpyAsync(dev(d_k), host(h_k), bytes, cudaMemcpyHostToDevice, s.up) != cudaSuccess ||
            cudaMemcpyAsync(dev(d_v), host(h_v), bytes, cudaMemcpyHostToDevice, s.up) != cudaSuccess ||
            cudaEventRecord(in, s.up) != cudaSuccess || cudaStreamWaitEvent(compute, in, 0) != cudaSuccess) {
            st = MONARCH_ERR_CUDA;
            break;
        }
        // chunk c as its own call: batch 1, (b1 - b0) heads
        st = monarch_attn_fwd(dev(d_q), dev(d_k), dev(d_v), dev(d_out), 1, static_cast<int>(b1 - b0), T, H, W, d,
                              factorisation, tile_h, tile_w, dtype, compute);
        if (st != MONARCH_OK) break;
        if (cudaEventRecord(out, compute) != cudaSuccess || cudaStreamWaitEvent(s.down, out, 0) != cudaSuccess ||
            cudaMemcpyAsync(static_cast<uint8_t *>(h_out) + off, dev(d_out), bytes, cudaMemcpyDeviceToHost,
                            s.down) != cudaSuccess)
            st = MONARCH_ERR_CUDA;
    }
    // the events are reused by the next call only after all queued work is done
    const cudaError_t e1 = cudaStreamSynchronize(s.up), e2 = cudaStreamSynchronize(compute),
                      e3 = cudaStreamSynchronize(s.down);
    if (st == MONARCH_OK && (e1 != cudaSuccess || e2 != cudaSuccess || e3 != cudaSuccess)) st = MONARCH_ERR_CUDA;
    return st;
}
