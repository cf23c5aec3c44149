// Host-side interface between the C ABI (wkv4_api.cpp) and the kernels
// (wkv4_kernels.cu).  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace wkv4 {

// Bits of the device error word (set by the kernels, read by wkv4_device_error).
constexpr unsigned kErrTmaWait = 2u;       // a TMA copy did not land in time
constexpr unsigned kErrExchangeWait = 4u;  // a cluster peer's aggregate did not land in time
constexpr unsigned kErrSlot = 8u;          // a slot-indexed decode row named a slot outside the pool
constexpr unsigned kErrBounds = 16u;       // checked builds: a global index outside its buffer

struct FwdArgs {
    int64_t B, T, C;
    const float* w;
    const float* u;
    const void* k;
    const void* v;
    const float* state_in;
    void* y;
    float* state_out;
    int dtype;  // WKV4_F32 / WKV4_F16 / WKV4_BF16
    cudaStream_t stream;
    const void* r = nullptr;  // receptance [B][T][C] of the gated forward (y = sigmoid(r) wkv), or NULL
};

// Tile geometry of a kernel for one dtype: channels and steps per TMA box.
struct Geom {
    int box_c;      // channels per box (innermost TMA dimension)
    int box_t;      // time steps per box
    int threads;    // threads per CTA
    size_t smem;    // dynamic shared memory per CTA (bytes)
};

Geom seq_geom(int dtype);
size_t dtype_size(int dtype);

// Encoder of a 3-D [B][T][C] tensor map with a box of box_c channels x
// box_t steps (false on failure).
typedef bool (*EncodeFn)(CUtensorMap* map, const void* ptr, int dtype, int64_t B, int64_t T,
                         int64_t C, int box_c, int box_t);

// Launchers.  The scan picks its shape, then encodes its tensor maps with
// `encode` (tma) or loads element-wise (!tma).
cudaError_t launch_scan(const FwdArgs& a, bool tma, EncodeFn encode);
cudaError_t launch_seq(const FwdArgs& a, const CUtensorMap* tk, const CUtensorMap* tv,
                       const CUtensorMap* tr);  // tr: the receptance's map when a.r is given
cudaError_t launch_step(const FwdArgs& a);     // exact per-step kernel, any T >= 1
// token shift: out[i] = mix[i] x_t + (1 - mix[i]) x_{t-1} for the non-null mix[i]
struct ShiftArgs {
    int64_t B, T, C;
    const void* x;
    const void* x_prev;
    const float* mix[3];
    void* out[3];
    void* x_last;
    int dtype;
    cudaStream_t stream;
};
cudaError_t launch_token_shift(const ShiftArgs& a);  // T >= 1, B, C >= 1

cudaError_t launch_decode(const FwdArgs& a);   // T == 1, vectorised when aligned
// T == 1 over rows slots[b] of a state pool of S rows (a.state_in == a.state_out == the pool)
cudaError_t launch_decode_slots(const FwdArgs& a, const int32_t* slots, int64_t S);
cudaError_t launch_copy_state(const FwdArgs& a);  // T == 0
// out <- x (NULL: empty) followed by a segment of n steps whose state is y
cudaError_t launch_state_combine(int64_t B, int64_t C, const float* w, int64_t n, const float* x,
                                 const float* y, float* out, cudaStream_t stream);

// Device error word of the current device (synchronous read; optional reset).
cudaError_t read_device_error(unsigned* bits, bool reset);

}  // namespace wkv4
