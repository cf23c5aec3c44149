// The forward from host buffers (wkv4_forward_host): the sequence is cut
// into chunks of T, and while the kernels run on chunk i, chunk i + 1's
// inputs come in and chunk i - 1's outputs go out.  The state is the whole
// history of the sequence and one call's final state is the next call's
// initial state ("An RNN that claims to match transformers, now in chatbot
// form", "The interesting bit"; the fp32 state of "RWKV in a self-built
// engine: a second non-attention paradigm (WKV/RNN)", Methods table,
// "Precision"), so the chunks are plain forward calls chained through one
// device state buffer.  Nothing here computes: the copies are CUDA runtime
// copies, every step of the recurrence runs in the forward's kernels.
//
// Streams: the caller's stream runs the kernels; two streams of the
// library's own (one pair per device) carry host -> device and device ->
// host copies (the two directions of the link at once).  Two workspace slots
// alternate between the chunks:
//   in (i):   copies of k, v (r) of chunk i into slot i % 2, once the kernels
//             of chunk i - 2 have read that slot;
//   run (i):  the forward of chunk i from the device state, in place, once
//             its inputs are in and the outputs of chunk i - 2 have left
//             slot i % 2;
//   out (i):  the copy of chunk i's y to the host, once it is written.
// The copy streams start after the work queued on `stream` before the call,
// and `stream` waits for the call's last copy, so the whole call is ordered
// on `stream` like any other call of the library (a call's first chunks
// follow the end of the call before it; the events' waits stay inside one
// call).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "../../include/wkv4.h"

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

size_t dtype_bytes(int dtype) { return dtype == WKV4_F32 ? 4 : 2; }

// Steps a chunk: the caller's choice, else about a sixteenth of the call's
// input bytes and at least 16 MB of them, at most T.  Each chunk costs a few
// copy calls, events and a launch, and the link moves both directions at
// once at a lower rate each (measured on B200: 55 GB/s in, 50 out, 42 + 42
// at once), so chunks of a few MB lose to fewer, larger ones; the first
// chunk's inputs and the last one's outputs are not overlapped, which a
// sixteenth keeps small on long calls.
int64_t chunk_steps_for(int64_t B, int64_t T, int64_t C, int dtype, bool gated, int64_t want) {
    if (T <= 0) return 0;
    if (want > 0) return std::min(want, T);
    const int64_t row = B * C * (int64_t)dtype_bytes(dtype) * (gated ? 3 : 2);  // input bytes a step
    if (row <= 0) return T;
    const int64_t by_share = (T + 15) / 16;
    const int64_t by_floor = ((int64_t)16 << 20) / row + 1;
    return std::min(T, std::max(by_share, by_floor));
}

struct Plan {
    int64_t tc = 0;  // steps a chunk
    size_t io = 0;   // bytes of one [B][tc][C] tensor in a slot
    size_t slot = 0; // bytes of a slot: k, v (r), y
    size_t state = 0;
    size_t total = 0;
};

Plan plan_for(int64_t B, int64_t T, int64_t C, int dtype, bool gated, int64_t want) {
    Plan p;
    p.tc = chunk_steps_for(B, T, C, dtype, gated, want);
    p.io = align_up((size_t)B * (size_t)p.tc * (size_t)C * dtype_bytes(dtype));
    p.slot = p.io * (gated ? 4 : 3);
    p.state = align_up((size_t)3 * B * C * 4);
    p.total = 2 * p.slot + p.state;
    return p;
}

// The copy streams and the events of the pipeline, made once per device and
// kept for the process (streams and events, no memory).  Calls on one device
// issue their work under the device's lock, so the events' records and
// waits of two calls never interleave; the work itself runs asynchronously.
struct DeviceResources {
    std::mutex lock;
    bool ready = false;
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, end = nullptr, in_done = nullptr;
    cudaEvent_t in_ready[2] = {nullptr, nullptr}, in_free[2] = {nullptr, nullptr};
    cudaEvent_t y_ready[2] = {nullptr, nullptr}, y_free[2] = {nullptr, nullptr};
    cudaError_t create() {
        if (ready) return cudaSuccess;
        cudaError_t e;
        if (!in && (e = cudaStreamCreateWithFlags(&in, cudaStreamNonBlocking)) != cudaSuccess) return e;
        if (!out && (e = cudaStreamCreateWithFlags(&out, cudaStreamNonBlocking)) != cudaSuccess) return e;
        cudaEvent_t* all[] = {&start, &end, &in_done, &in_ready[0], &in_ready[1], &in_free[0],
                              &in_free[1], &y_ready[0], &y_ready[1], &y_free[0], &y_free[1]};
        for (cudaEvent_t* ev : all)
            if (!*ev && (e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return e;
        ready = true;
        return cudaSuccess;
    }
};

constexpr int kMaxDevices = 64;

DeviceResources* device_resources(int dev) {
    static DeviceResources res[kMaxDevices];
    return dev >= 0 && dev < kMaxDevices ? &res[dev] : nullptr;
}

// A [B][n][C] block starting at step t0 of a [B][T][C] host tensor, to or
// from a contiguous [B][n][C] device block (unified addressing tells the
// direction: host memory, pinned or not, or device memory).
cudaError_t copy_block(void* dst, size_t dpitch, const void* src, size_t spitch, size_t width,
                       int64_t B, cudaMemcpyKind kind, cudaStream_t s) {
    if (B == 1 || (dpitch == width && spitch == width))
        return cudaMemcpyAsync(dst, src, width * (size_t)B, kind, s);
    return cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, (size_t)B, kind, s);
}

int cuda_rc(cudaError_t e) {
    if (e == cudaSuccess) return WKV4_OK;
    cudaGetLastError();
    return WKV4_ERR_CUDA;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || !na || !nb) return false;
    const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
    return x < y + nb && y < x + na;
}

}  // namespace

namespace {

// The copies and forward calls of wkv4_forward_host, chunk by chunk, on the
// device's copy streams and `cs` (see the top of the file); returns at the
// first error, leaving what it queued to the caller's join.
int issue_chunks(DeviceResources& res, int64_t B, int64_t T, int64_t C, const float* w,
                 const float* u, const void* k, const void* v, const void* r,
                 const float* state_in, void* y, float* state_out, const Plan& pl,
                 unsigned char* ws, int dtype, cudaStream_t cs) {
    const wkv4_stream_t stream = (wkv4_stream_t)cs;
    const bool gated = r != nullptr;
    const size_t es = dtype_bytes(dtype);
    const size_t st_bytes = (size_t)3 * B * C * 4;
    float* dstate = reinterpret_cast<float*>(ws + 2 * pl.slot);
    auto slot_k = [&](int s) { return ws + (size_t)s * pl.slot; };
    auto slot_v = [&](int s) { return slot_k(s) + pl.io; };
    auto slot_y = [&](int s) { return slot_k(s) + 2 * pl.io; };
    auto slot_r = [&](int s) { return slot_k(s) + 3 * pl.io; };
    const size_t spitch = (size_t)T * C * es;  // a batch row of a host tensor
    cudaError_t e;
    // the copies follow whatever the caller queued on `stream` before
    if ((e = cudaEventRecord(res.start, cs)) != cudaSuccess) return cuda_rc(e);
    if ((e = cudaStreamWaitEvent(res.in, res.start, 0)) != cudaSuccess) return cuda_rc(e);
    if ((e = cudaStreamWaitEvent(res.out, res.start, 0)) != cudaSuccess) return cuda_rc(e);
    if (state_in &&
        (e = cudaMemcpyAsync(dstate, state_in, st_bytes, cudaMemcpyDefault, res.in)) != cudaSuccess)
        return cuda_rc(e);
    const int64_t nchunks = (T + pl.tc - 1) / pl.tc;
    for (int64_t i = 0; i < nchunks; ++i) {
        const int s = (int)(i & 1);
        const int64_t t0 = i * pl.tc, n = std::min(pl.tc, T - t0);
        const size_t width = (size_t)n * C * es;  // a batch row of the chunk
        const size_t off = (size_t)t0 * C * es;
        // in (i)
        if (i >= 2 && (e = cudaStreamWaitEvent(res.in, res.in_free[s], 0)) != cudaSuccess) return cuda_rc(e);
        if ((e = copy_block(slot_k(s), width, static_cast<const unsigned char*>(k) + off, spitch, width,
                            B, cudaMemcpyDefault, res.in)) != cudaSuccess)
            return cuda_rc(e);
        if ((e = copy_block(slot_v(s), width, static_cast<const unsigned char*>(v) + off, spitch, width,
                            B, cudaMemcpyDefault, res.in)) != cudaSuccess)
            return cuda_rc(e);
        if (gated && (e = copy_block(slot_r(s), width, static_cast<const unsigned char*>(r) + off, spitch,
                                     width, B, cudaMemcpyDefault, res.in)) != cudaSuccess)
            return cuda_rc(e);
        if ((e = cudaEventRecord(res.in_ready[s], res.in)) != cudaSuccess) return cuda_rc(e);
        // run (i): chunk 0 starts from state_in (or the empty state), every
        // later chunk from the state the one before left
        if ((e = cudaStreamWaitEvent(cs, res.in_ready[s], 0)) != cudaSuccess) return cuda_rc(e);
        if (i >= 2 && (e = cudaStreamWaitEvent(cs, res.y_free[s], 0)) != cudaSuccess) return cuda_rc(e);
        const float* sin = (i == 0 && !state_in) ? nullptr : dstate;
        const int rc = gated ? wkv4_forward_gated(B, n, C, w, u, slot_k(s), slot_v(s), slot_r(s), sin,
                                                  slot_y(s), dstate, stream, dtype)
                             : wkv4_forward(B, n, C, w, u, slot_k(s), slot_v(s), sin, slot_y(s), dstate,
                                            stream, dtype);
        if (rc != WKV4_OK) return rc;
        if ((e = cudaEventRecord(res.in_free[s], cs)) != cudaSuccess) return cuda_rc(e);
        if ((e = cudaEventRecord(res.y_ready[s], cs)) != cudaSuccess) return cuda_rc(e);
        // out (i)
        if ((e = cudaStreamWaitEvent(res.out, res.y_ready[s], 0)) != cudaSuccess) return cuda_rc(e);
        if ((e = copy_block(static_cast<unsigned char*>(y) + off, spitch, slot_y(s), width, width, B,
                            cudaMemcpyDefault, res.out)) != cudaSuccess)
            return cuda_rc(e);
        if ((e = cudaEventRecord(res.y_free[s], res.out)) != cudaSuccess) return cuda_rc(e);
    }
    // the final state leaves after the last chunk's kernels (the out stream
    // waited for them)
    if (state_out &&
        (e = cudaMemcpyAsync(state_out, dstate, st_bytes, cudaMemcpyDefault, res.out)) != cudaSuccess)
        return cuda_rc(e);
    return WKV4_OK;
}

}  // namespace

extern "C" {

size_t wkv4_forward_host_workspace(int64_t B, int64_t T, int64_t C, int dtype, int gated,
                                   int64_t chunk_steps) {
    if (B <= 0 || T < 0 || C <= 0 || chunk_steps < 0) return 0;
    if (dtype != WKV4_F32 && dtype != WKV4_F16 && dtype != WKV4_BF16) return 0;
    if (T == 0) return align_up((size_t)3 * B * C * 4);  // the empty state's way out
    return plan_for(B, T, C, dtype, gated != 0, chunk_steps).total;
}

int wkv4_forward_host(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                      const void* k, const void* v, const void* r, const float* state_in,
                      void* y, float* state_out, void* workspace, size_t workspace_bytes,
                      int64_t chunk_steps, wkv4_stream_t stream, int dtype) {
    if (B < 0 || T < 0 || C < 0 || chunk_steps < 0) return WKV4_ERR_ARG;
    if (dtype != WKV4_F32 && dtype != WKV4_F16 && dtype != WKV4_BF16) return WKV4_ERR_DTYPE;
    if (B == 0 || C == 0) return WKV4_OK;
    const cudaStream_t cs = (cudaStream_t)stream;
    const size_t st_bytes = (size_t)3 * B * C * 4;
    const size_t es = dtype_bytes(dtype);
    const size_t io_bytes = (size_t)B * T * C * es;
    if (T == 0) {
        // the state passes through unchanged (the empty state without one)
        if (!state_out) return WKV4_OK;
        if (state_in) {
            if (state_in == state_out) return WKV4_OK;
            if (overlaps(state_in, st_bytes, state_out, st_bytes)) return WKV4_ERR_ALIAS;
            return cuda_rc(cudaMemcpyAsync(state_out, state_in, st_bytes, cudaMemcpyDefault, cs));
        }
        if (!workspace || workspace_bytes < align_up(st_bytes)) return WKV4_ERR_ARG;
        int rc = wkv4_forward(B, 0, C, w, u, nullptr, nullptr, nullptr, nullptr,
                              static_cast<float*>(workspace), stream, dtype);
        if (rc != WKV4_OK) return rc;
        return cuda_rc(cudaMemcpyAsync(state_out, workspace, st_bytes, cudaMemcpyDefault, cs));
    }
    const bool gated = r != nullptr;
    if (!w || !u || !k || !v || !y || !workspace) return WKV4_ERR_ARG;
    const Plan pl = plan_for(B, T, C, dtype, gated, chunk_steps);
    if (workspace_bytes < pl.total) return WKV4_ERR_ARG;
    // host outputs must not overlap the host inputs (the in-place state
    // excepted), nor the workspace anything
    if (overlaps(y, io_bytes, k, io_bytes) || overlaps(y, io_bytes, v, io_bytes) ||
        overlaps(y, io_bytes, r, gated ? io_bytes : 0) || overlaps(y, io_bytes, state_in, st_bytes) ||
        overlaps(y, io_bytes, state_out, st_bytes))
        return WKV4_ERR_ALIAS;
    if (overlaps(state_out, st_bytes, k, io_bytes) || overlaps(state_out, st_bytes, v, io_bytes) ||
        overlaps(state_out, st_bytes, r, gated ? io_bytes : 0) ||
        (state_in != state_out && overlaps(state_out, st_bytes, state_in, st_bytes)))
        return WKV4_ERR_ALIAS;
    const void* host[] = {k, v, r, state_in, y, state_out, w, u};
    const size_t host_n[] = {io_bytes, io_bytes, gated ? io_bytes : 0, st_bytes, io_bytes,
                             st_bytes, (size_t)C * 4, (size_t)C * 4};
    for (int i = 0; i < 8; ++i)
        if (overlaps(workspace, pl.total, host[i], host_n[i])) return WKV4_ERR_ALIAS;

    unsigned char* ws = static_cast<unsigned char*>(workspace);

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_rc(e);
    DeviceResources* rp = device_resources(dev);
    if (!rp) return WKV4_ERR_CUDA;
    std::lock_guard<std::mutex> guard(rp->lock);
    DeviceResources& res = *rp;
    if ((e = res.create()) != cudaSuccess) return cuda_rc(e);
    const int rc = issue_chunks(res, B, T, C, w, u, k, v, r, state_in, y, state_out, pl, ws, dtype, cs);
    // `stream` waits for whatever this call queued on the copy streams -- after an error too, so
    // that no copy of the call is still in flight once `stream` has passed it
    cudaError_t e1 = cudaEventRecord(res.end, res.out);
    if (e1 == cudaSuccess) e1 = cudaStreamWaitEvent(cs, res.end, 0);
    cudaError_t e2 = cudaEventRecord(res.in_done, res.in);
    if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(cs, res.in_done, 0);
    if (rc != WKV4_OK) return rc;
    return cuda_rc(e1 != cudaSuccess ? e1 : e2);
}

}  // extern "C"
