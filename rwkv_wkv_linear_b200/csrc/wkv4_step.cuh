// Per-step kernels: the max-trick one step at a time, in natural units.
//
//   wkv4_step_kernel    one thread per channel, any T (the recurrence as the
//                       pages state it, step after step).
//   wkv4_decode_kernel  T = 1 with V channels per thread and vector accesses;
//                       the state may be updated in place (RNN mode); with
//                       kSlots, row b's state is row slots[b] of a pool of
//                       S rows (state_in == state_out == the pool).
//   wkv4_copy_state_kernel  T = 0: state_out <- state_in (or the empty state).
#pragma once

#include "wkv4_device.cuh"

namespace wkv4 {

struct StepParams {
    int64_t B, T, C;
    const float* w;
    const float* u;
    const void* k;
    const void* v;
    const float* state_in;
    void* y;
    float* state_out;
    const int32_t* slots;  // decode from a state pool: row b uses pool row slots[b]
    int64_t S;             // pool rows
};

template <typename IO>
__global__ void __launch_bounds__(256) wkv4_step_kernel(const StepParams p) {
    const int64_t BC = p.B * p.C;
    const int64_t ch = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (ch >= BC) return;
    const int64_t b = ch / p.C, c = ch - b * p.C;
    St s = p.state_in ? St{p.state_in[ch], p.state_in[BC + ch], (double)p.state_in[2 * BC + ch]}
                      : St{0.f, 0.f, (double)kEmptyMaxNat};
    const float w = p.w[c], u = p.u[c];
    const IO* kg = static_cast<const IO*>(p.k);
    const IO* vg = static_cast<const IO*>(p.v);
    IO* yg = static_cast<IO*>(p.y);
    for (int64_t t = 0; t < p.T; ++t) {
        const int64_t off = (b * p.T + t) * p.C + c;
        const float y = step_nat(s, Io<IO>::to_f(kg[off]), Io<IO>::to_f(vg[off]), w, u);
        yg[off] = Io<IO>::from_f(y);
    }
    if (p.state_out) store_state_nat_d(p.state_out, BC, ch, s.a, s.b, s.p);
}

// The caller checks that C % V == 0 and every pointer is aligned to its
// vector width.
template <typename IO, int V, bool kSlots = false>
__global__ void __launch_bounds__(256) wkv4_decode_kernel(const StepParams p) {
    const int64_t BC = p.B * p.C;
    const int64_t ch = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * V;
    if (ch >= BC) return;
    const int64_t c = ch % p.C;
    float kk[V], vv[V], yy[V], a[V], bb[V], pp[V], w[V], u[V];
    load_vec<IO, V>(static_cast<const IO*>(p.k) + ch, kk);
    load_vec<IO, V>(static_cast<const IO*>(p.v) + ch, vv);
    load_vec<float, V>(p.w + c, w);
    load_vec<float, V>(p.u + c, u);
    // state plane stride and this thread's offset in a plane (with kSlots the
    // row's slot, read while the loads above are in flight)
    int64_t SC = BC, sch = ch;
    if constexpr (kSlots) {
        const int64_t b = ch / p.C;
        const int64_t slot = p.slots[b];
        if (slot < 0 || slot >= p.S) {
            if (c == 0) atomicOr(&g_device_error, kErrSlot);
            return;
        }
        SC = p.S * p.C;
        sch = slot * p.C + c;
    }
    if (p.state_in) {
        load_vec<float, V>(p.state_in + sch, a);
        load_vec<float, V>(p.state_in + SC + sch, bb);
        load_vec<float, V>(p.state_in + 2 * SC + sch, pp);
    } else {
#pragma unroll
        for (int j = 0; j < V; ++j) {
            a[j] = 0.f;
            bb[j] = 0.f;
            pp[j] = kEmptyMaxNat;
        }
    }
#pragma unroll
    for (int j = 0; j < V; ++j) {
        St s = {a[j], bb[j], (double)pp[j]};
        yy[j] = step_nat(s, kk[j], vv[j], w[j], u[j]);
        const float pf = (float)s.p;
        const float d = (float)(s.p - (double)pf);  // fold the max's rounding into a, b
        a[j] = fmaf(s.a, d, s.a);
        bb[j] = fmaf(s.b, d, s.b);
        pp[j] = pf;
    }
    store_vec<IO, V>(static_cast<IO*>(p.y) + ch, yy);
    if (p.state_out) {
        store_vec<float, V>(p.state_out + sch, a);
        store_vec<float, V>(p.state_out + SC + sch, bb);
        store_vec<float, V>(p.state_out + 2 * SC + sch, pp);
    }
}

__global__ void __launch_bounds__(256) wkv4_copy_state_kernel(const float* in, float* out, int64_t BC) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= BC) return;
    if (in) {
        out[i] = in[i];
        out[BC + i] = in[BC + i];
        out[2 * BC + i] = in[2 * BC + i];
    } else {
        out[i] = 0.f;
        out[BC + i] = 0.f;
        out[2 * BC + i] = kEmptyMaxNat;
    }
}

}  // namespace wkv4
