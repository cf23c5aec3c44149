// Token shift of the RWKV-4 time mix: each output mixes the current token's
// channels with the previous token's ("RWKV in a self-built engine: a second
// non-attention paradigm (WKV/RNN)", Reproducibility / Provenance,
// "Implementation": token-shift, "mix current and previous token"):
//   out[b,t,c] = mix[c] x[b,t,c] + (1 - mix[c]) x[b,t-1,c],
// with x[b,-1,c] the previous call's last token (x_prev) or zero, for up to
// three mix vectors (k, v, r) in one pass over x.
//
// An HBM stream: each thread owns V channels (16 bytes) of one batch row and
// walks a run of steps, keeping the previous token in registers, so x is read
// once (plus one row per run) and each output written once.  The launcher
// sizes the runs so that the grid is one wave of the CTAs the GPU holds at
// once (no tail of a second, partial wave).  Computed in fp32 as
// x_prev + mix (x - x_prev) and rounded once to the I/O type.
#pragma once

#include "wkv4_device.cuh"

namespace wkv4 {

struct ShiftParams {
    int64_t B, T, C;
    const void* x;
    const void* x_prev;  // [B][C] or null (zero)
    const float* mix[3];  // k, v, r; r may be null
    void* out[3];        // xk, xv, xr (xr null when mix r is)
    void* x_last;        // [B][C] or null
    int64_t run;         // steps a thread walks
};

constexpr int kShiftThreads = 128;  // threads a CTA: channel groups of 128 V
constexpr int kShiftMinRun = 8;     // shortest run (each run reads one row twice)

// V fp32 values from p (16-byte pieces when V > 1).
template <int V>
__device__ __forceinline__ void load_f32(const float* p, float (&o)[V]) {
    if constexpr (V <= 4) {
        load_vec<float, V>(p, o);
    } else {
        static_assert(V % 4 == 0, "16-byte pieces");
#pragma unroll
        for (int q = 0; q < V / 4; ++q) {
            float t[4];
            load_vec<float, 4>(p + 4 * q, t);
#pragma unroll
            for (int j = 0; j < 4; ++j) o[4 * q + j] = t[j];
        }
    }
}

// grid: x = channel groups of kShiftThreads V, y = runs of p.run steps, z =
// batch rows.  The caller checks that C % V == 0 and every pointer is 16-byte
// aligned when V > 1.
template <typename IO, int V>
__global__ void __launch_bounds__(kShiftThreads) wkv4_token_shift_kernel(const ShiftParams p) {
    allow_dependents();
    grid_dependency_wait();
    const int64_t c = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * V;
    if (c >= p.C) return;
    const int64_t b = blockIdx.z;
    const int64_t t0 = (int64_t)blockIdx.y * p.run;
    const int64_t t1 = min(p.T, t0 + p.run);
    const IO* x = static_cast<const IO*>(p.x);
    // every access is (b T + t) C + c .. + V - 1 for t in [t0 - 1, t1), or a
    // [B][C] row at b C + c (checked builds)
    if (!in_range(c + V - 1, p.C) || !in_range(b, p.B) || !in_range(t1 - 1, p.T)) return;
    float xp[V], xt[V], o[V];
    if (t0 > 0) {
        load_vec<IO, V>(x + (b * p.T + t0 - 1) * p.C + c, xp);
    } else if (p.x_prev) {
        load_vec<IO, V>(static_cast<const IO*>(p.x_prev) + b * p.C + c, xp);
    } else {
#pragma unroll
        for (int j = 0; j < V; ++j) xp[j] = 0.f;
    }
    const int nout = p.mix[2] ? 3 : 2;
    float m[3][V];
#pragma unroll
    for (int i = 0; i < 3; ++i)
        if (i < nout) load_f32<V>(p.mix[i] + c, m[i]);
#pragma unroll 4
    for (int64_t t = t0; t < t1; ++t) {
        const int64_t off = (b * p.T + t) * p.C + c;
        load_vec<IO, V>(x + off, xt);
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            if (i < nout) {
#pragma unroll
                for (int j = 0; j < V; ++j) o[j] = fmaf(m[i][j], xt[j] - xp[j], xp[j]);
                store_vec<IO, V>(static_cast<IO*>(p.out[i]) + off, o);
            }
        }
#pragma unroll
        for (int j = 0; j < V; ++j) xp[j] = xt[j];
    }
    if (t1 == p.T && p.x_last) store_vec<IO, V>(static_cast<IO*>(p.x_last) + b * p.C + c, xp);
}

}  // namespace wkv4
