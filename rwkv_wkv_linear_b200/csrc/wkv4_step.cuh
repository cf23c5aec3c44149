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
    const void* r;         // receptance, laid out as k, of the gated step (kGate), else NULL
};

// kGate: y = sigmoid(r) wkv, the receptance gate of the time mix.
template <typename IO, bool kGate = false>
__global__ void __launch_bounds__(256) wkv4_step_kernel(const StepParams p) {
    allow_dependents();
    grid_dependency_wait();
    const int64_t BC = p.B * p.C;
    const int64_t ch = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (ch >= BC) return;
    const int64_t b = ch / p.C, c = ch - b * p.C;
    if (!in_range(c, p.C) || !in_range(b, p.B)) return;
    St s = p.state_in ? St{p.state_in[ch], p.state_in[BC + ch], (double)p.state_in[2 * BC + ch]}
                      : St{0.f, 0.f, (double)kEmptyMaxNat};
    const float w = p.w[c], u = p.u[c];
    const IO* kg = static_cast<const IO*>(p.k);
    const IO* vg = static_cast<const IO*>(p.v);
    const IO* rg = static_cast<const IO*>(p.r);
    IO* yg = static_cast<IO*>(p.y);
    for (int64_t t = 0; t < p.T; ++t) {
        const int64_t off = (b * p.T + t) * p.C + c;
        if (!in_range(off, BC * p.T)) break;
        const float r = kGate ? Io<IO>::to_f(rg[off]) : 0.f;
        const float y = step_nat<kGate>(s, Io<IO>::to_f(kg[off]), Io<IO>::to_f(vg[off]), w, u, r);
        yg[off] = Io<IO>::from_f(y);
    }
    if (p.state_out) store_state_nat_d(p.state_out, BC, ch, s.a, s.b, s.p);
}

// The caller checks that C % V == 0 and every pointer is aligned to its
// vector width.
template <typename IO, int V, bool kSlots = false, bool kGate = false>
__global__ void __launch_bounds__(256) wkv4_decode_kernel(const StepParams p) {
    allow_dependents();
    grid_dependency_wait();
    const int64_t BC = p.B * p.C;
    const int64_t ch = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * V;
    if (ch >= BC) return;
    const int64_t c = ch % p.C;
    if (!in_range(ch + V - 1, BC) || !in_range(c + V - 1, p.C)) return;
    float kk[V], vv[V], rr[V], yy[V], a[V], bb[V], pp[V], w[V], u[V];
    load_vec<IO, V>(static_cast<const IO*>(p.k) + ch, kk);
    load_vec<IO, V>(static_cast<const IO*>(p.v) + ch, vv);
    if constexpr (kGate) load_vec<IO, V>(static_cast<const IO*>(p.r) + ch, rr);
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
    if (!in_range(sch + V - 1, SC)) return;
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
        yy[j] = step_nat<kGate>(s, kk[j], vv[j], w[j], u[j], kGate ? rr[j] : 0.f);
        const float pf = (float)s.p;
        const float d = fold_factor((float)(s.p - (double)pf));  // fold the max's rounding into a, b
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

// State x (NULL: the empty state) followed by a segment of n steps whose
// state from the empty state is y: per channel, in natural units with the
// max in fp64,
//   px = p_x + n w,  p = max(px, p_y),
//   a = a_x e^{px - p} + a_y e^{p_y - p},  b likewise,
// the larger of the two factors exactly 1 (one exponential a channel); the
// max is rounded to fp32 on the way out with its rounding folded into a, b.
// out may be x or y itself (each thread reads its channel before writing it).
__global__ void __launch_bounds__(256)
    wkv4_state_combine_kernel(const float* __restrict__ w, int64_t n, const float* x,
                              const float* y, float* out, int64_t B, int64_t C) {
    allow_dependents();
    grid_dependency_wait();
    const int64_t BC = B * C;
    const int64_t ch = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (ch >= BC) return;
    const int64_t c = ch % C;
    if (!in_range(c, C)) return;
    const float xa = x ? x[ch] : 0.f, xb = x ? x[BC + ch] : 0.f;
    const double xp = x ? (double)x[2 * BC + ch] : (double)kEmptyMaxNat;
    const float ya = y[ch], yb = y[BC + ch];
    const double yp = y[2 * BC + ch];
    const double px = xp + (double)n * (double)w[c];
    const double d = px - yp;
    const float f = exp2f((float)-fabs(d) * kLog2e);
    const float fx = d >= 0.0 ? 1.f : f, fy = d >= 0.0 ? f : 1.f;
    store_state_nat_d(out, BC, ch, fmaf(xa, fx, ya * fy), fmaf(xb, fx, yb * fy), d >= 0.0 ? px : yp);
}

__global__ void __launch_bounds__(256) wkv4_copy_state_kernel(const float* in, float* out, int64_t BC) {
    allow_dependents();
    grid_dependency_wait();
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
