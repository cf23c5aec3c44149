// Device-side building blocks of the RWKV-4 WKV kernels (sm_100a).
//
// Inside the kernels the state triple is kept in log2 units: A = a 2^p,
// D = b 2^p, and k is scaled by log2(e) on load, so every exponential is one
// ex2.approx.  The per-channel numerator / denominator / max state in fp32
// with the max-trick is the one of "RWKV in a self-built engine: a second
// non-attention paradigm (WKV/RNN)" (Methods table, "Precision").
//
// Chunk arithmetic.  A stretch of n <= L steps is processed against one
// fixed reference r = max_i k_i (log2 units) instead of a per-step running
// max: with e_i = 2^{k_i - r} <= 1 the stretch needs one ex2 per step for its
// summary and reuses e_i for its outputs (plus one reciprocal), instead of
// two ex2 and a reciprocal for the per-step max-trick.  This is exact
// algebra; it is taken only when the stretch's exponents stay well inside
// fp32 range (kmax - kmin <= kFastRange + min(0, u), u <= kFastMaxU,
// w <= kFastMaxW, and a carried state at most kFastStateLift above r), so
// every denominator is >= 2^-80 and anything that underflows is below 2^-126.
// Otherwise the stretch falls back to the per-step max-trick.
//
// Stretches are joined with an associative combine on (a, b, p) over a
// stretch length n: X then Y = (a_x 2^{p_x + n w - p} + a_y 2^{p_y - p}, ...,
// p = max(p_x + n w, p_y)).  Decay across stretches is applied through the
// exponent (2^{n w}), not by n repeated multiplications, so fp32 rounding of
// e^w does not accumulate over long T.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace wkv4 {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kEmptyMaxNat = -1e38f;               // max of the empty state (natural units)
constexpr float kEmptyMax2 = -1e38f * 1.4426950408889634f;
constexpr float kFastRange = 80.f;                   // log2 units
constexpr float kFastStateLift = 64.f;               // log2 units
constexpr float kFastMaxU = 64.f;                    // log2 units
constexpr float kFastMaxW = 0.5f;                    // log2 units per step

// device error word bits
constexpr unsigned kErrLookback = 1u;
constexpr unsigned kErrTmaWait = 2u;

// bounded waits: polls before a wait gives up (each poll sleeps ~100 ns or more)
constexpr uint32_t kMaxPolls = 1u << 22;

struct St {
    float a, b, p;
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ St empty_state() { return {0.f, 0.f, kEmptyMax2}; }

// X followed by a stretch summarised (from the empty state) as Y, the stretch
// spanning n steps; nw2 = n * w (log2 units).  The larger of the two scale
// factors is exactly 1, so one ex2 serves.
__device__ __forceinline__ St combine(St x, St y, float nw2) {
    const float px = x.p + nw2;
    const float d = px - y.p;
    const float f = ex2(-fabsf(d));
    const bool xbig = d >= 0.f;
    const float fx = xbig ? 1.f : f, fy = xbig ? f : 1.f;
    return {fmaf(x.a, fx, y.a * fy), fmaf(x.b, fx, y.b * fy), xbig ? px : y.p};
}

// (A, D) at reference r with D a normal positive float -> triple with b in [1, 2),
// by an exact power-of-two rescale.
__device__ __forceinline__ St normalized(float A, float D, float r) {
    const int e = ((__float_as_int(D) >> 23) & 0xff) - 127;
    const float s = __int_as_float((127 - e) << 23);
    return {A * s, D * s, r + (float)e};
}

// One exact max-trick step in log2 units on state s with input
// (x = k log2e, v): returns the output and advances the state.
__device__ __forceinline__ float exact_step(St& s, float x, float v, float w2, float u2) {
    const float q = fmaxf(s.p, u2 + x);
    const float f1 = ex2(s.p - q), f2 = ex2(u2 + x - q);
    const float y = __fdividef(fmaf(f1, s.a, f2 * v), fmaf(f1, s.b, f2));
    const float q2 = fmaxf(s.p + w2, x);
    const float g1 = ex2(s.p + w2 - q2), g2 = ex2(x - q2);
    s.a = fmaf(g1, s.a, g2 * v);
    s.b = fmaf(g1, s.b, g2);
    s.p = q2;
    return y;
}

// The same step with the state, k, w and u in natural units (the units of
// the state buffers), so a state carried over many single-step calls is
// never converted: used by the decode step and the exact per-step kernel.
__device__ __forceinline__ float exp_nat(float x) { return ex2(x * kLog2e); }

__device__ __forceinline__ float exact_step_nat(St& s, float k, float v, float w, float u) {
    const float q = fmaxf(s.p, u + k);
    const float f1 = exp_nat(s.p - q), f2 = exp_nat(u + k - q);
    const float y = __fdividef(fmaf(f1, s.a, f2 * v), fmaf(f1, s.b, f2));
    const float q2 = fmaxf(s.p + w, k);
    const float g1 = exp_nat(s.p + w - q2), g2 = exp_nat(k - q2);
    s.a = fmaf(g1, s.a, g2 * v);
    s.b = fmaf(g1, s.b, g2);
    s.p = q2;
    return y;
}

// State advance only (no output), exact max-trick, log2 units.
__device__ __forceinline__ void exact_update(St& s, float x, float v, float w2) {
    const float q2 = fmaxf(s.p + w2, x);
    const float g1 = ex2(s.p + w2 - q2), g2 = ex2(x - q2);
    s.a = fmaf(g1, s.a, g2 * v);
    s.b = fmaf(g1, s.b, g2);
    s.p = q2;
}

__device__ __forceinline__ bool fast_ok(float kmax, float kmin, float u2, float w2) {
    return (kmax - kmin <= kFastRange + fminf(0.f, u2)) && (u2 <= kFastMaxU) && (w2 <= kFastMaxW);
}

// ---------------------------------------------------------------- I/O dtypes

template <typename IO> struct Io;

template <> struct Io<float> {
    __device__ __forceinline__ static float to_f(float x) { return x; }
    __device__ __forceinline__ static float from_f(float x) { return x; }
};
template <> struct Io<__half> {
    __device__ __forceinline__ static float to_f(__half x) { return __half2float(x); }
    __device__ __forceinline__ static __half from_f(float x) { return __float2half_rn(x); }
};
template <> struct Io<__nv_bfloat16> {
    __device__ __forceinline__ static float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    __device__ __forceinline__ static __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// V consecutive elements <-> floats, as one vector access when V * sizeof(IO)
// is 4, 8 or 16 bytes (caller guarantees alignment).
template <typename IO, int V>
__device__ __forceinline__ void load_vec(const IO* p, float (&o)[V]) {
    constexpr int kBytes = V * (int)sizeof(IO);
    if constexpr (kBytes == 2 || kBytes == 4) {
        if constexpr (V == 1) {
            o[0] = Io<IO>::to_f(*p);
        } else {
            IO t[2];
            *reinterpret_cast<uint32_t*>(t) = *reinterpret_cast<const uint32_t*>(p);
            o[0] = Io<IO>::to_f(t[0]);
            o[1] = Io<IO>::to_f(t[1]);
        }
    } else if constexpr (kBytes == 8) {
        IO t[V];
        *reinterpret_cast<uint2*>(t) = *reinterpret_cast<const uint2*>(p);
#pragma unroll
        for (int j = 0; j < V; ++j) o[j] = Io<IO>::to_f(t[j]);
    } else {
        static_assert(kBytes == 16, "vector width");
        IO t[V];
        *reinterpret_cast<uint4*>(t) = *reinterpret_cast<const uint4*>(p);
#pragma unroll
        for (int j = 0; j < V; ++j) o[j] = Io<IO>::to_f(t[j]);
    }
}

template <typename IO, int V>
__device__ __forceinline__ void store_vec(IO* p, const float (&x)[V]) {
    constexpr int kBytes = V * (int)sizeof(IO);
    IO t[V];
#pragma unroll
    for (int j = 0; j < V; ++j) t[j] = Io<IO>::from_f(x[j]);
    if constexpr (V == 1) {
        *p = t[0];
    } else if constexpr (kBytes == 4) {
        *reinterpret_cast<uint32_t*>(p) = *reinterpret_cast<const uint32_t*>(t);
    } else if constexpr (kBytes == 8) {
        *reinterpret_cast<uint2*>(p) = *reinterpret_cast<const uint2*>(t);
    } else {
        static_assert(kBytes == 16, "vector width");
        *reinterpret_cast<uint4*>(p) = *reinterpret_cast<const uint4*>(t);
    }
}

// ------------------------------------------------------- TMA / mbarrier PTX

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, P;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait on an mbarrier phase; false when it ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
    for (uint32_t i = 0; i < kMaxPolls; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if (i > 64) __nanosleep(128);
    }
    return false;
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y,
                                             int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------ cross-CTA flags (look-back)

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

}  // namespace wkv4
