// Device-side building blocks of the RWKV-4 WKV kernels (sm_100a).
//
// Inside the chunked kernels the state triple is kept in log2 units:
// A = a 2^p, D = b 2^p, with the max p in fp64, and every exponential is one
// ex2.approx of an fp32 difference k log2(e) - r formed by one FMA.  The per-channel numerator / denominator / max state in fp32
// with the max-trick is the one of "RWKV in a self-built engine: a second
// non-attention paradigm (WKV/RNN)" (Methods table, "Precision").
//
// Chunk arithmetic.  A stretch of n <= L steps is processed against one
// fixed reference r = max_i k_i (log2 units) instead of a per-step running
// max: with e_i = 2^{k_i - r} <= 1 the stretch needs one ex2 per step for its
// summary and reuses e_i for its outputs (plus one reciprocal), instead of
// two ex2 and a reciprocal for the per-step max-trick.  This is exact
// algebra; it is taken only when the stretch's exponents stay well inside
// fp32 range (in nats: kmax - kmin <= kFastRange + min(0, u), u <= kFastMaxU,
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

#include "wkv4_internal.h"  // device error word bits

namespace wkv4 {

// The device error word (per device; wkv4_device_error reads and clears it):
// the bits of wkv4_internal.h, set by the kernels with atomicOr.
__device__ unsigned int g_device_error = 0;

// Checked builds (WKV4_CHECKED): every global index is checked against the
// extent of its buffer before the access; one outside it sets kErrBounds in
// the error word and the access is skipped.  Other builds compile the check
// to `true`.
#ifdef WKV4_CHECKED
__device__ __forceinline__ bool in_range(int64_t i, int64_t n) {
    if (i >= 0 && i < n) return true;
    atomicOr(&g_device_error, kErrBounds);
    return false;
}
#else
__device__ __forceinline__ constexpr bool in_range(int64_t, int64_t) { return true; }
#endif

// Programmatic dependent launch.  Every kernel of the library is launched so
// that it may start while the kernel before it in the stream is finishing
// (its CTAs become resident and set up as the earlier grid's CTAs leave); it
// lets the next one do the same as soon as it starts, and touches no global
// memory before grid_dependency_wait(), which returns once the earlier grid
// has completed and its memory is visible (at once for a normal launch).
__device__ __forceinline__ void allow_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr double kLog2eD = 1.4426950408889634;
constexpr double kLn2D = 0.6931471805599453;
constexpr float kEmptyMaxNat = -1e38f;               // max of the empty state (natural units)
constexpr double kEmptyMax2 = -1e38 * 1.4426950408889634;
// fixed-reference chunk path limits (natural units)
constexpr float kFastRange = 55.f;       // max k - min k (+ min(0, u)) within a chunk
constexpr float kFastStateLift = 44.f;   // carried state's max above the chunk's max k
constexpr float kFastMaxU = 44.f;
constexpr float kFastMaxW = 0.35f;



// A = a 2^p, D = b 2^p.  The max p is carried in fp64 inside the kernels, so
// that adding n*w to a large max loses nothing; it is rounded to fp32 only at
// the state buffers, with the rounding folded back into a and b.
struct St {
    float a, b;
    double p;
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
__device__ __forceinline__ St combine(St x, St y, double nw2) {
    const double px = x.p + nw2;
    const double d = px - y.p;
    const float f = ex2((float)-fabs(d));
    const bool xbig = d >= 0.0;
    const float fx = xbig ? 1.f : f, fy = xbig ? f : 1.f;
    return {fmaf(x.a, fx, y.a * fy), fmaf(x.b, fx, y.b * fy), xbig ? px : y.p};
}

// (A, D) at reference r with D a normal positive float -> triple with b in [1, 2),
// by an exact power-of-two rescale.
__device__ __forceinline__ St normalized(float A, float D, double r) {
    const int e = ((__float_as_int(D) >> 23) & 0xff) - 127;
    const float s = __int_as_float((127 - e) << 23);
    return {A * s, D * s, r + (double)e};
}

// One exact max-trick step (log2 units, fp64 max) with input k (natural), v:
// returns the output and advances the state.  w2, u2 = w, u in log2 units.
__device__ __forceinline__ float exact_step(St& s, float k, float v, double w2, double u2) {
    const double x = (double)k * kLog2eD;
    const double q = fmax(s.p, u2 + x);
    const float f1 = ex2((float)(s.p - q)), f2 = ex2((float)(u2 + x - q));
    const float y = __fdividef(fmaf(f1, s.a, f2 * v), fmaf(f1, s.b, f2));
    const double q2 = fmax(s.p + w2, x);
    const float g1 = ex2((float)(s.p + w2 - q2)), g2 = ex2((float)(x - q2));
    s.a = fmaf(g1, s.a, g2 * v);
    s.b = fmaf(g1, s.b, g2);
    s.p = q2;
    return y;
}

// State advance only (no output).
__device__ __forceinline__ void exact_update(St& s, float k, float v, double w2) {
    const double x = (double)k * kLog2eD;
    const double q2 = fmax(s.p + w2, x);
    const float g1 = ex2((float)(s.p + w2 - q2)), g2 = ex2((float)(x - q2));
    s.a = fmaf(g1, s.a, g2 * v);
    s.b = fmaf(g1, s.b, g2);
    s.p = q2;
}

// The per-step max-trick with the state in natural units (the units of the
// state buffers), fp64 max and accurate exp2f: the decode step and the
// per-step kernel, where one step's rounding is carried to the next call.
// Of the two scale factors of each half step the one at the max is exactly
// 1 (exp2f(0)), so only the other one is evaluated: the same bits as taking
// both, with half the exponentials.  kGate: the output gated by the
// receptance r, sigmoid(r) y = num / (den (1 + e^{-r})) (e^{-r} = inf below
// r = -88 gives 0, the gate's limit).
template <bool kGate = false>
__device__ __forceinline__ float step_nat(St& s, float k, float v, float w, float u, float r = 0.f) {
    const double kd = k;
    // output: q = max(p, u + k)
    const double d1 = s.p - ((double)u + kd);
    const float f = exp2f((float)-fabs(d1) * kLog2e);
    const float f1 = d1 >= 0.0 ? 1.f : f, f2 = d1 >= 0.0 ? f : 1.f;
    float den = fmaf(f1, s.b, f2);
    if constexpr (kGate) den = fmaf(den, exp2f(-r * kLog2e), den);
    const float y = __fdividef(fmaf(f1, s.a, f2 * v), den);
    // state: q2 = max(p + w, k)
    const double pw = s.p + (double)w;
    const double d2 = pw - kd;
    const float g = exp2f((float)-fabs(d2) * kLog2e);
    const float g1 = d2 >= 0.0 ? 1.f : g, g2 = d2 >= 0.0 ? g : 1.f;
    s.a = fmaf(g1, s.a, g2 * v);
    s.b = fmaf(g1, s.b, g2);
    s.p = d2 >= 0.0 ? pw : kd;
    return y;
}

__device__ __forceinline__ bool fast_ok(float kmax, float kmin, float u, float w) {
    return (kmax - kmin <= kFastRange + fminf(0.f, u)) && (u <= kFastMaxU) && (w <= kFastMaxW);
}

// fp32 state buffers <-> kernel state.  On the way out the max is rounded to
// fp32 and the rounding error d (natural units, |d| <= half an ulp of the
// max) is folded into a and b as a e^d = a + a (e^d - 1), b likewise.  While
// |d| < 2^-12 (a max below 4096 nats in magnitude, the usual case) e^d - 1
// is d to within its last bit, and d is used as it is; beyond (a max of 10^5
// nats after a long decay with nothing new has |d| up to 2^-5, where d alone
// would be off by d^2 / 2) e^d - 1 comes from expm1f.
__device__ __forceinline__ float fold_factor(float d) {
    return fabsf(d) < 0x1p-12f ? d : expm1f(d);
}
__device__ __forceinline__ St load_state_log2(const float* __restrict__ s, int64_t BC, int64_t ch) {
    return {s[ch], s[BC + ch], (double)s[2 * BC + ch] * kLog2eD};
}

__device__ __forceinline__ void store_state_nat_d(float* __restrict__ s, int64_t BC, int64_t ch,
                                                  float a, float b, double p_nat) {
    const float pf = (float)p_nat;
    const float d = fold_factor((float)(p_nat - (double)pf));
    s[ch] = fmaf(a, d, a);
    s[BC + ch] = fmaf(b, d, b);
    s[2 * BC + ch] = pf;
}

__device__ __forceinline__ void store_state_log2(float* __restrict__ s, int64_t BC, int64_t ch, St x) {
    store_state_nat_d(s, BC, ch, x.a, x.b, x.p * kLn2D);
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

// try_wait with a suspend-time hint: the thread sleeps in hardware until the
// phase completes or about `ns` nanoseconds pass, instead of spinning (a
// spinning warp takes issue slots from the warps that compute).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, P;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// Bounded wait on an mbarrier phase (about `rounds` x 1 ms at most); false
// when it ran out.
constexpr uint32_t kWaitRounds = 1000;
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint32_t rounds = kWaitRounds) {
    for (uint32_t i = 0; i < rounds; ++i)
        if (mbar_try_wait_sleep(bar, parity, 1000000u)) return true;
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

// Untiled bulk copy global -> shared (16-byte aligned addresses, size a
// multiple of 16), completing on an mbarrier.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Prefetch of a box of a tiled tensor into L2 (no shared-memory destination,
// nothing to wait for).
__device__ __forceinline__ void tma_prefetch_3d_l2(const CUtensorMap* map, int x, int y, int z) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(z)
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

// ------------------------------------------------ distributed shared memory

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_u32(uint32_t local_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
    return r;
}

// Asynchronous stores into (possibly another CTA's) shared memory whose bytes
// complete a transaction on the mbarrier at `mbar` in the target CTA.
__device__ __forceinline__ void st_async_v2f32(uint32_t addr, float x, float y, uint32_t mbar) {
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(addr),
        "f"(x), "f"(y), "r"(mbar)
        : "memory");
}
__device__ __forceinline__ void st_async_v2f64(uint32_t addr, double x, double y, uint32_t mbar) {
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f64 [%0], {%1, %2}, [%3];" ::"r"(addr),
        "d"(x), "d"(y), "r"(mbar)
        : "memory");
}

// try_wait acquiring at cluster scope (writes by other CTAs' st.async).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 P, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, P;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t* bar, uint32_t parity,
                                                          uint32_t rounds = kWaitRounds) {
    for (uint32_t i = 0; i < rounds; ++i)
        if (mbar_try_wait_cluster(bar, parity, 1000000u)) return true;
    return false;
}

// ------------------------------------------------ tensor memory (tcgen05)
//
// The scan kernel keeps per-step values of a chunk in tensor memory between
// its two passes over the chunk: 128 lanes x 512 columns of 32 bits per SM.
// A warp reaches only the 32 lanes of its quarter (warp index mod 4); with
// the .32x32b shape each thread reads / writes its own lane, the address
// carrying lane (bits 31..16) and column (bits 15..0).

// Warp-wide: allocate ncols columns (a power of two, 32..512); the base
// address is written to *slot in shared memory.
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// Around a thread barrier that orders tensor-memory accesses of different warps.
__device__ __forceinline__ void tmem_fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Warp-wide: 16 consecutive columns of this thread's lane <- r.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// Warp-wide: this thread's stores to tensor memory have completed.
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Warp-wide: r <- 16 consecutive columns of this thread's lane.  The wait is
// tied to the destination registers, so no use of them is scheduled before it.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
}

}  // namespace wkv4
