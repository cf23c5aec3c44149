// Per-chunk routines shared by the chunked-scan and sequential kernels.
//
// One lane owns a PAIR of adjacent channels of one chunk of n <= L
// consecutive steps whose rows sit in shared memory (row stride `stride`
// elements, the pair at column `col`).  The pair's fp32 arithmetic runs as
// packed f32x2 operations (one FFMA2 / FMUL2 / FADD2 for both channels).
//
// chunk_phase1 computes the chunk's summary from the empty state (its A, D
// and max) and keeps e_i = 2^{k_i log2e - r} (r = the chunk's max k in log2
// units, rounded to fp32) for chunk_phase3, which produces the outputs from
// the state at the chunk's start.
#pragma once

#include "wkv4_device.cuh"

namespace wkv4 {

// ------------------------------------------------------------ packed f32x2

typedef unsigned long long f2;  // lo = first channel, hi = second channel

__device__ __forceinline__ f2 pk(float lo, float hi) {
    f2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ f2 pku(uint32_t lo, uint32_t hi) { return ((f2)hi << 32) | lo; }
__device__ __forceinline__ float lo(f2 r) { return __uint_as_float((unsigned)(r & 0xffffffffull)); }
__device__ __forceinline__ float hi(f2 r) { return __uint_as_float((unsigned)(r >> 32)); }
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
    f2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
    f2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f2 add2(f2 a, f2 b) {
    f2 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ f2 ex2_2(f2 x) { return pk(ex2(lo(x)), ex2(hi(x))); }
__device__ __forceinline__ f2 rcp2(f2 x) { return pk(rcp_approx(lo(x)), rcp_approx(hi(x))); }

// ------------------------------------------------------ receptance gate
//
// The time mix's output is gated by the receptance: y = sigmoid(r) wkv
// ("RWKV in a self-built engine: a second non-attention paradigm
// (WKV/RNN)", abstract and Reproducibility / Provenance, "Implementation":
// time-mix gating; "RWKV-4 14B", "Every architecture field": the time mix's
// receptance matrix), with sigmoid(r) = 1 / (1 + e^{-r}).  On the outputs'
// fast paths it is folded into the one reciprocal they already take:
//   y = num / (den (1 + e^{-r})),  den (1 + g) = fma(den, g, den),  g = e^{-r},
// one more exponential and one FMA a channel-step.  e^{-r} overflows to
// +inf below r = -88, where the quotient is 0: the gate's limit.

// g = e^{-r} for a channel pair
__device__ __forceinline__ f2 gate_g2(f2 r) { return ex2_2(mul2(r, pk(-kLog2e, -kLog2e))); }

// sigmoid(r) y for one channel (the per-step paths)
__device__ __forceinline__ float gate_one(float y, float r) {
    return y * rcp_approx(1.f + ex2(-r * kLog2e));
}

// No gate: the outputs' paths compile without it.
struct NoGate {
    static constexpr bool kOn = false;
    __device__ __forceinline__ f2 operator()(int) const { return 0ull; }
};

// A gate of the outputs' fast paths: f(i) gives g = e^{-r} of step i's pair.
template <typename F>
struct FnGate {
    static constexpr bool kOn = true;
    F f;
    __device__ __forceinline__ f2 operator()(int i) const { return f(i); }
};
template <typename F>
__device__ __forceinline__ FnGate<F> fn_gate(F f) {
    return FnGate<F>{f};
}

// ------------------------------------------------------- pair I/O by dtype

template <typename IO> struct Pair;

template <> struct Pair<float> {
    typedef f2 Raw;  // the pair as stored
    __device__ __forceinline__ static Raw raw(const float* p) { return *reinterpret_cast<const f2*>(p); }
    __device__ __forceinline__ static f2 cvt(Raw r) { return r; }
    __device__ __forceinline__ static void minmax(Raw r, Raw& mx, Raw& mn) {
        mx = pk(fmaxf(lo(mx), lo(r)), fmaxf(hi(mx), hi(r)));
        mn = pk(fminf(lo(mn), lo(r)), fminf(hi(mn), hi(r)));
    }
    __device__ __forceinline__ static void bounds(Raw mx, Raw mn, float (&x)[2], float (&n)[2]) {
        x[0] = lo(mx), x[1] = hi(mx), n[0] = lo(mn), n[1] = hi(mn);
    }
    __device__ __forceinline__ static f2 load(const float* p) {
        return *reinterpret_cast<const f2*>(p);
    }
    __device__ __forceinline__ static void store(float* p, f2 y) { *reinterpret_cast<f2*>(p) = y; }
    // running max / min over raw elements
    struct MinMax {
        float mx0, mx1, mn0, mn1;
        __device__ __forceinline__ void init(const float* p) {
            mx0 = mn0 = p[0];
            mx1 = mn1 = p[1];
        }
        __device__ __forceinline__ void add(const float* p) {
            const float a = p[0], b = p[1];
            mx0 = fmaxf(mx0, a);
            mn0 = fminf(mn0, a);
            mx1 = fmaxf(mx1, b);
            mn1 = fminf(mn1, b);
        }
        __device__ __forceinline__ void get(float (&mx)[2], float (&mn)[2]) const {
            mx[0] = mx0, mx[1] = mx1, mn[0] = mn0, mn[1] = mn1;
        }
    };
};

template <> struct Pair<__half> {
    typedef __half2 Raw;
    __device__ __forceinline__ static Raw raw(const __half* p) { return *reinterpret_cast<const __half2*>(p); }
    __device__ __forceinline__ static f2 cvt(Raw r) {
        const float2 f = __half22float2(r);
        return pk(f.x, f.y);
    }
    __device__ __forceinline__ static void minmax(Raw r, Raw& mx, Raw& mn) {
        mx = __hmax2(mx, r);
        mn = __hmin2(mn, r);
    }
    __device__ __forceinline__ static void bounds(Raw mx, Raw mn, float (&x)[2], float (&n)[2]) {
        const float2 a = __half22float2(mx), b = __half22float2(mn);
        x[0] = a.x, x[1] = a.y, n[0] = b.x, n[1] = b.y;
    }
    __device__ __forceinline__ static f2 load(const __half* p) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(p));
        return pk(f.x, f.y);
    }
    __device__ __forceinline__ static void store(__half* p, f2 y) {
        *reinterpret_cast<__half2*>(p) = __floats2half2_rn(lo(y), hi(y));
    }
    struct MinMax {
        __half2 mx, mn;
        __device__ __forceinline__ void init(const __half* p) {
            mx = mn = *reinterpret_cast<const __half2*>(p);
        }
        __device__ __forceinline__ void add(const __half* p) {
            const __half2 h = *reinterpret_cast<const __half2*>(p);
            mx = __hmax2(mx, h);
            mn = __hmin2(mn, h);
        }
        __device__ __forceinline__ void get(float (&x)[2], float (&n)[2]) const {
            const float2 a = __half22float2(mx), b = __half22float2(mn);
            x[0] = a.x, x[1] = a.y, n[0] = b.x, n[1] = b.y;
        }
    };
};

template <> struct Pair<__nv_bfloat16> {
    typedef __nv_bfloat162 Raw;
    __device__ __forceinline__ static Raw raw(const __nv_bfloat16* p) {
        return *reinterpret_cast<const __nv_bfloat162*>(p);
    }
    __device__ __forceinline__ static f2 cvt(Raw r) {
        const float2 f = __bfloat1622float2(r);
        return pk(f.x, f.y);
    }
    __device__ __forceinline__ static void minmax(Raw r, Raw& mx, Raw& mn) {
        mx = __hmax2(mx, r);
        mn = __hmin2(mn, r);
    }
    __device__ __forceinline__ static void bounds(Raw mx, Raw mn, float (&x)[2], float (&n)[2]) {
        const float2 a = __bfloat1622float2(mx), b = __bfloat1622float2(mn);
        x[0] = a.x, x[1] = a.y, n[0] = b.x, n[1] = b.y;
    }
    __device__ __forceinline__ static f2 load(const __nv_bfloat16* p) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
        return pk(f.x, f.y);
    }
    __device__ __forceinline__ static void store(__nv_bfloat16* p, f2 y) {
        *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(lo(y), hi(y));
    }
    struct MinMax {
        __nv_bfloat162 mx, mn;
        __device__ __forceinline__ void init(const __nv_bfloat16* p) {
            mx = mn = *reinterpret_cast<const __nv_bfloat162*>(p);
        }
        __device__ __forceinline__ void add(const __nv_bfloat16* p) {
            const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(p);
            mx = __hmax2(mx, h);
            mn = __hmin2(mn, h);
        }
        __device__ __forceinline__ void get(float (&x)[2], float (&n)[2]) const {
            const float2 a = __bfloat1622float2(mx), b = __bfloat1622float2(mn);
            x[0] = a.x, x[1] = a.y, n[0] = b.x, n[1] = b.y;
        }
    };
};

// --------------------------------------------------------- per-pair state

struct PairConsts {
    f2 ew, eu;       // e^w, e^u
    float w[2], u[2];  // natural units
    double w2[2];    // w in log2 units
};

// Loads of a pair's w and u (issued early: kernels fetch them before their
// bulk tensor copies so that they do not queue behind them).
__device__ __forceinline__ void pair_wu(const float* __restrict__ w, const float* __restrict__ u,
                                        int64_t c, int64_t C, PairConsts& cc) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const bool ok = c + j < C;
        cc.w[j] = ok ? __ldg(w + c + j) : 0.f;
        cc.u[j] = ok ? __ldg(u + c + j) : 0.f;
    }
}

// The derived constants, once w and u are loaded.
__device__ __forceinline__ void pair_derive(PairConsts& cc) {
    float ew[2], eu[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        ew[j] = expf(cc.w[j]);
        eu[j] = expf(cc.u[j]);
        cc.w2[j] = (double)cc.w[j] * kLog2eD;
    }
    cc.ew = pk(ew[0], ew[1]);
    cc.eu = pk(eu[0], eu[1]);
}

__device__ __forceinline__ void pair_consts(const float* __restrict__ w, const float* __restrict__ u,
                                            int64_t c, int64_t C, PairConsts& cc) {
    pair_wu(w, u, c, C, cc);
    pair_derive(cc);
}

// The per-step max-trick for a chunk's summary, kept out of line: it runs
// only for chunks whose exponents leave the fixed-reference range.
template <typename IO>
__device__ __noinline__ St slow_summary(const IO* sk, const IO* sv, int stride, int m, double w2) {
    St s = empty_state();
    for (int i = 0; i < m; ++i)
        exact_update(s, Io<IO>::to_f(sk[i * stride]), Io<IO>::to_f(sv[i * stride]), w2);
    return s;
}

// Per-lane result of chunk_phase1 that chunk_phase3 needs: the chunk's
// reference (max k in log2 units, rounded to fp32) and whether each channel
// takes the fixed-reference path.  The e_i themselves are recomputed in
// phase 3 from k (one ex2 per step) instead of being held in registers.
struct PairRef {
    float kref[2];
    bool fast[2];
};

// Summary of the chunk from the empty state: max/min pass, then e_i and the
// two Horner chains.  kFull (n == L) is a separate instantiation so that the
// full chunk's loops carry no per-step guard and consecutive steps overlap.
//
// With kStash the pass also leaves, for the output pass,
// each step's chunk-local numerator and denominator of y_i at the reference,
//   N_i = A_i + e^u e_i v_i,   Dn_i = D_i + e^u e_i
// (A_i, D_i: the chunk's state before step i, from the empty state), in
// tensor memory at taddr: 4 columns a step (N lo, N hi, Dn lo, Dn hi), so
// that the output pass needs neither k, v nor an exponential.
template <typename IO, int L, bool kFull, bool kStash>
__device__ __forceinline__ void chunk_phase1_t(PairRef& r, const IO* sk, const IO* sv, int stride,
                                               int col, int n, const PairConsts& cc, St (&sum)[2],
                                               uint32_t taddr) {
    static_assert(!kStash || L % 4 == 0, "stash: whole column groups");
    typename Pair<IO>::Raw mx = Pair<IO>::raw(sk + col), mn = mx;
#pragma unroll
    for (int i = 1; i < L; ++i)
        if (kFull || i < n) Pair<IO>::minmax(Pair<IO>::raw(sk + i * stride + col), mx, mn);
    float kmax[2], kmin[2];
    Pair<IO>::bounds(mx, mn, kmax, kmin);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        r.fast[j] = fast_ok(kmax[j], kmin[j], cc.u[j], cc.w[j]);
        r.kref[j] = kmax[j] * kLog2e;
    }
    const f2 l2e = pk(kLog2e, kLog2e);
    const f2 nref = pk(-r.kref[0], -r.kref[1]);
    f2 A = 0ull, D = 0ull;
    uint32_t st[16];
    if constexpr (kStash) __syncwarp();  // tensor-memory stores are warp-collective
#pragma unroll
    for (int i = 0; i < L; ++i) {
        if (kFull || i < n) {
            const f2 e = ex2_2(fma2(Pair<IO>::load(sk + i * stride + col), l2e, nref));
            const f2 ev = mul2(e, Pair<IO>::load(sv + i * stride + col));
            if constexpr (kStash) {
                const f2 N = fma2(cc.eu, ev, A), Dn = fma2(cc.eu, e, D);
                const int s = (i & 3) * 4;
                st[s] = (uint32_t)N;
                st[s + 1] = (uint32_t)(N >> 32);
                st[s + 2] = (uint32_t)Dn;
                st[s + 3] = (uint32_t)(Dn >> 32);
                // a group of 4 steps at a time (n is the same on every lane)
                if ((i & 3) == 3 || (!kFull && i == n - 1)) tmem_st16(taddr + (uint32_t)(i >> 2) * 16u, st);
            }
            A = fma2(cc.ew, A, ev);
            D = fma2(cc.ew, D, e);
        }
    }
    if constexpr (kStash) tmem_wait_st();
    const float Aj[2] = {lo(A), hi(A)}, Dj[2] = {lo(D), hi(D)};
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        if (r.fast[j]) {
            sum[j] = normalized(Aj[j], Dj[j], (double)r.kref[j]);
        } else {
            sum[j] = slow_summary<IO>(sk + col + j, sv + col + j, stride, n, cc.w2[j]);
        }
    }
}

template <typename IO, int L, bool kStash = false>
__device__ __forceinline__ void chunk_phase1(PairRef& r, const IO* sk, const IO* sv, int stride,
                                             int col, int n, const PairConsts& cc, St (&sum)[2],
                                             uint32_t taddr = 0) {
    if (n >= L) {
        chunk_phase1_t<IO, L, true, kStash>(r, sk, sv, stride, col, L, cc, sum, taddr);
    } else if (n > 0) {
        chunk_phase1_t<IO, L, false, kStash>(r, sk, sv, stride, col, n, cc, sum, taddr);
    } else {
        sum[0] = sum[1] = empty_state();
        r.fast[0] = r.fast[1] = false;
        r.kref[0] = r.kref[1] = 0.f;
    }
}

// Outputs of the chunk from the state S at its start, through
// out_pair(i, y) or out_one(i, j, value).  Step i reads k_i and v_i before
// writing y_i, so y may be staged in place of k.  The common case (both
// channels on the fixed-reference path, a full chunk) is one branch-free
// unrolled loop; anything else goes through chunk_phase3_general, where the
// per-step channels read k again, so a fast channel's y is then written one
// element at a time and the slow channel's k stays intact.
template <typename IO, int L, typename OutOne>
__device__ __noinline__ void chunk_phase3_general(const PairRef& r, const IO* sk, const IO* sv,
                                                  int stride, int col, int m, bool f30, bool f31,
                                                  f2 Ah, f2 Dh, St S0, St S1, const PairConsts& cc,
                                                  OutOne out_one) {
    const bool f3[2] = {f30, f31};
    const St S[2] = {S0, S1};
    const f2 l2e = pk(kLog2e, kLog2e);
    const f2 nref = pk(-r.kref[0], -r.kref[1]);
    for (int i = 0; i < m; ++i) {
        const f2 e = ex2_2(fma2(Pair<IO>::load(sk + i * stride + col), l2e, nref));
        const f2 ev = mul2(e, Pair<IO>::load(sv + i * stride + col));
        const f2 y = mul2(fma2(cc.eu, ev, Ah), rcp2(fma2(cc.eu, e, Dh)));
        Ah = fma2(cc.ew, Ah, ev);
        Dh = fma2(cc.ew, Dh, e);
        if (f3[0]) out_one(i, 0, lo(y));
        if (f3[1]) out_one(i, 1, hi(y));
    }
    for (int j = 0; j < 2; ++j) {
        if (f3[j]) continue;
        St s = S[j];
        const double u2 = (double)cc.u[j] * kLog2eD;
        for (int i = 0; i < m; ++i) {
            const float k = Io<IO>::to_f(sk[i * stride + col + j]);
            const float v = Io<IO>::to_f(sv[i * stride + col + j]);
            out_one(i, j, exact_step(s, k, v, cc.w2[j], u2));
        }
    }
}

// With a gate (Gate::kOn), gate(i) gives g = e^{-r_i} of step i's pair and
// the fast loop divides by den (1 + g); the general path's out_one applies
// the gate itself.
template <typename IO, int L, typename OutPair, typename OutOne, typename Gate = NoGate>
__device__ __forceinline__ void chunk_phase3(const PairRef& r, const IO* sk, const IO* sv, int stride,
                                             int col, int n, const St (&S)[2], const PairConsts& cc,
                                             OutPair out_pair, OutOne out_one, Gate gate = Gate()) {
    if (n <= 0) return;
    bool f3[2];
    float a0[2], b0[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const double lift = S[j].p - (double)r.kref[j];
        f3[j] = r.fast[j] && (lift <= (double)(kFastStateLift * kLog2e));
        const float sc = ex2((float)lift);
        a0[j] = S[j].a * sc;
        b0[j] = S[j].b * sc;
    }
    f2 Ah = pk(a0[0], a0[1]), Dh = pk(b0[0], b0[1]);
    if (n == L && f3[0] && f3[1]) {
        const f2 l2e = pk(kLog2e, kLog2e);
        const f2 nref = pk(-r.kref[0], -r.kref[1]);
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const f2 e = ex2_2(fma2(Pair<IO>::load(sk + i * stride + col), l2e, nref));
            const f2 ev = mul2(e, Pair<IO>::load(sv + i * stride + col));
            // (A + e^u e v) / (D + e^u e), then A <- e^w A + e v, D <- e^w D + e
            f2 den = fma2(cc.eu, e, Dh);
            if constexpr (Gate::kOn) den = fma2(den, gate(i), den);
            const f2 y = mul2(fma2(cc.eu, ev, Ah), rcp2(den));
            Ah = fma2(cc.ew, Ah, ev);
            Dh = fma2(cc.ew, Dh, e);
            out_pair(i, y);
        }
    } else {
        chunk_phase3_general<IO, L, OutOne>(r, sk, sv, stride, col, n, f3[0], f3[1], Ah, Dh, S[0],
                                            S[1], cc, out_one);
    }
}

// Outputs of a chunk of n steps from the state S at its start by the exact
// per-step max-trick, reading k and v of channel j at gk[i * stride + j],
// gv[...] (global memory; only channels with ok[j]).  The fallback of the
// stash path: it runs for a warp only where some lane's chunk leaves the
// fixed-reference range.
template <typename IO, typename OutOne>
__device__ __noinline__ void chunk_exact_global(const IO* gk, const IO* gv, int64_t stride, int n,
                                                bool ok0, bool ok1, St S0, St S1,
                                                const PairConsts& cc, OutOne out_one) {
    const bool ok[2] = {ok0, ok1};
    const St S[2] = {S0, S1};
    for (int j = 0; j < 2; ++j) {
        if (!ok[j]) continue;
        St s = S[j];
        const double u2 = (double)cc.u[j] * kLog2eD;
        for (int i = 0; i < n; ++i) {
            const float k = Io<IO>::to_f(gk[(int64_t)i * stride + j]);
            const float v = Io<IO>::to_f(gv[(int64_t)i * stride + j]);
            out_one(i, j, exact_step(s, k, v, cc.w2[j], u2));
        }
    }
}

// Outputs of a chunk of n steps whose summary pass left its stash in tensor
// memory at taddr (chunk_phase1 with kStash).  When every lane of the warp
// has both channels on the fixed-reference path (the decision is warp-wide:
// tensor-memory loads are warp-collective), from the state S = (a, b, p) at
// the chunk start, whose weight at step i relative to the reference r is
// f_i = 2^{p - r} e^{i w},
//   y_i = (f_i a + N_i) / (f_i b + Dn_i),
// one reciprocal a step, through out_pair(i, y).  f_i is carried as one
// factor (f_0 = 2^{p - r}, times e^w a step), so it leaves the float range
// only where the state's share of y_i does: a separate e^{i w} would
// underflow under a fast decay while the state, lifted up to 2^63 above the
// reference, still outweighs Dn_i.  Otherwise the exact per-step
// path from k, v in global memory (gk, gv: the pair's first channel at the
// chunk's first step, row stride `stride`; ok[j]: channel j exists) through
// out_one(i, j, y).
// With a gate (Gate::kOn), gate(i) gives g = e^{-r_i} of step i's pair and
// y_i = num / (den (1 + g)); the exact path's out_one applies the gate itself.
template <typename IO, int L, typename OutPair, typename OutOne, typename Gate = NoGate>
__device__ __forceinline__ void chunk_phase3_stash(const PairRef& r, int n, const St (&S)[2],
                                                   const PairConsts& cc, uint32_t taddr,
                                                   const IO* gk, const IO* gv, int64_t stride,
                                                   bool ok0, bool ok1, OutPair out_pair,
                                                   OutOne out_one, Gate gate = Gate()) {
    static_assert(L % 4 == 0, "stash: whole column groups");
    if (n <= 0) return;
    bool f3[2];
    float sc[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const double lift = S[j].p - (double)r.kref[j];
        f3[j] = r.fast[j] && (lift <= (double)(kFastStateLift * kLog2e));
        sc[j] = ex2((float)lift);
    }
    if (__all_sync(0xffffffffu, f3[0] && f3[1])) {
        const f2 al = pk(S[0].a, S[1].a), be = pk(S[0].b, S[1].b);
        f2 f = pk(sc[0], sc[1]);  // 2^{p - r} e^{i w}
        if (n == L) {
#pragma unroll
            for (int q = 0; q < L / 4; ++q) {
                uint32_t st[16];
                tmem_ld16(taddr + (uint32_t)q * 16u, st);
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const f2 N = pku(st[4 * s], st[4 * s + 1]), Dn = pku(st[4 * s + 2], st[4 * s + 3]);
                    f2 den = fma2(f, be, Dn);
                    if constexpr (Gate::kOn) den = fma2(den, gate(4 * q + s), den);
                    out_pair(4 * q + s, mul2(fma2(f, al, N), rcp2(den)));
                    f = mul2(f, cc.ew);
                }
            }
        } else {
#pragma unroll 1
            for (int q = 0; 4 * q < n; ++q) {
                uint32_t st[16];
                tmem_ld16(taddr + (uint32_t)q * 16u, st);
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    if (4 * q + s < n) {
                        const f2 N = pku(st[4 * s], st[4 * s + 1]);
                        const f2 Dn = pku(st[4 * s + 2], st[4 * s + 3]);
                        f2 den = fma2(f, be, Dn);
                        if constexpr (Gate::kOn) den = fma2(den, gate(4 * q + s), den);
                        out_pair(4 * q + s, mul2(fma2(f, al, N), rcp2(den)));
                        f = mul2(f, cc.ew);
                    }
                }
            }
        }
    } else {
        chunk_exact_global<IO>(gk, gv, stride, n, ok0, ok1, S[0], S[1], cc, out_one);
    }
}

}  // namespace wkv4
