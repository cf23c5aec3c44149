// RWKV-4 WKV forward and decode kernels for B200 (sm_100a).
//
// The recurrence (per batch row and channel, decay w, bonus u):
//   wkv_t = (A_t + e^{u+k_t} v_t) / (D_t + e^{u+k_t}),
//   A_{t+1} = e^w A_t + e^{k_t} v_t,  D_{t+1} = e^w D_t + e^{k_t},
// with A, D carried as an fp32 (num, den, max) triple under the max-trick
// ("RWKV in a self-built engine: a second non-attention paradigm (WKV/RNN)",
// Methods table "Precision"; Reproducibility / Provenance "Implementation").
//
// Kernels
//   wkv4_scan_kernel    chunked scan over (channel tile x time segment) tiles.
//                       k, v tiles arrive by TMA into shared memory; each warp
//                       owns one chunk of L steps, each lane V channels.
//                       Chunk summaries are combined inside the CTA; segments
//                       of the same channels are chained across CTAs with a
//                       decoupled look-back on per-tile flags (bounded waits).
//                       y leaves through shared memory by a TMA store.
//   wkv4_seq_kernel     channel-parallel, sequential over T: each thread walks
//                       its channels' whole sequence through a multi-stage
//                       TMA ring of time tiles, chunk by chunk.
//   wkv4_step_kernel    one thread per channel, the per-step max-trick
//                       verbatim in natural units (any T).
//   wkv4_decode_kernel  T = 1 step, state updated in place, vectorised.
//
// No tensor cores: nothing here is a dense contraction; the work is bound by
// HBM bandwidth (k, v read once, y written once).
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstring>

#include "../../include/wkv4.h"
#include "wkv4_device.cuh"
#include "wkv4_internal.h"

namespace wkv4 {

__device__ unsigned int g_device_error = 0;

__device__ __forceinline__ void raise_error(unsigned bits) { atomicOr(&g_device_error, bits); }

// ============================================================ chunk routines
//
// One lane, V channels, one chunk of n <= L steps whose rows sit in shared
// memory at row stride `stride` elements (the lane's channels at column
// `col`).  phase1 computes the chunk's summary from the empty state and
// leaves e[j][i] = 2^{x_i - kmax_j} (fast channels) for phase3.

template <int V, int L>
struct ChunkRegs {
    float e[V][L];
    float kmax[V];
    bool fast[V];
};

template <typename IO, int V, int L>
__device__ __forceinline__ void chunk_phase1(ChunkRegs<V, L>& r, const IO* sk, const IO* sv,
                                             int stride, int col, int n, const float (&w2)[V],
                                             const float (&u2)[V], const float (&ew)[V],
                                             St (&sum)[V]) {
    float kmin[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        r.kmax[j] = -3.0e38f;
        kmin[j] = 3.0e38f;
    }
#pragma unroll
    for (int i = 0; i < L; ++i) {
        if (i < n) {
            float kk[V];
            load_vec<IO, V>(sk + i * stride + col, kk);
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const float x = kk[j] * kLog2e;
                r.e[j][i] = x;
                r.kmax[j] = fmaxf(r.kmax[j], x);
                kmin[j] = fminf(kmin[j], x);
            }
        }
    }
    float A[V], D[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        r.fast[j] = (n > 0) && fast_ok(r.kmax[j], kmin[j], u2[j], w2[j]);
        A[j] = 0.f;
        D[j] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < L; ++i) {
        if (i < n) {
            float vv[V];
            load_vec<IO, V>(sv + i * stride + col, vv);
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const float ee = ex2(r.e[j][i] - r.kmax[j]);
                r.e[j][i] = ee;
                A[j] = fmaf(ew[j], A[j], ee * vv[j]);
                D[j] = fmaf(ew[j], D[j], ee);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < V; ++j) {
        if (n <= 0) {
            sum[j] = empty_state();
        } else if (r.fast[j]) {
            sum[j] = normalized(A[j], D[j], r.kmax[j]);
        } else {
            // per-step max-trick from the empty state
            St s = empty_state();
            for (int i = 0; i < n; ++i) {
                const float x = Io<IO>::to_f(sk[i * stride + col + j]) * kLog2e;
                const float vv = Io<IO>::to_f(sv[i * stride + col + j]);
                exact_update(s, x, vv, w2[j]);
            }
            sum[j] = s;
        }
    }
}

// Outputs of the chunk given the state S at its start.  Writes y through
// `out(i, j, value)` / `out_vec(i, values)`; for channels that take the
// per-step path, k is read again from shared memory (a fast channel's slot
// may already hold its y when y is staged in place of k).
template <typename IO, int V, int L, typename OutVec, typename OutOne>
__device__ __forceinline__ void chunk_phase3(const ChunkRegs<V, L>& r, const IO* sk, const IO* sv,
                                             int stride, int col, int n, const St (&S)[V],
                                             const float (&w2)[V], const float (&u2)[V],
                                             const float (&ew)[V], const float (&eu)[V],
                                             OutVec out_vec, OutOne out_one) {
    bool f3[V];
    bool all_fast = true;
    float Ah[V], Dh[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        f3[j] = r.fast[j] && (S[j].p - r.kmax[j] <= kFastStateLift);
        all_fast = all_fast && f3[j];
        const float sc = ex2(S[j].p - r.kmax[j]);
        Ah[j] = S[j].a * sc;
        Dh[j] = S[j].b * sc;
    }
#pragma unroll
    for (int i = 0; i < L; ++i) {
        if (i < n) {
            float vv[V];
            load_vec<IO, V>(sv + i * stride + col, vv);
            float yv[V];
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const float ee = r.e[j][i];
                const float eb = eu[j] * ee;
                yv[j] = __fdividef(fmaf(eb, vv[j], Ah[j]), Dh[j] + eb);
                Ah[j] = fmaf(ew[j], Ah[j], ee * vv[j]);
                Dh[j] = fmaf(ew[j], Dh[j], ee);
            }
            if (all_fast) {
                out_vec(i, yv);
            } else {
#pragma unroll
                for (int j = 0; j < V; ++j)
                    if (f3[j]) out_one(i, j, yv[j]);
            }
        }
    }
    if (!all_fast) {
#pragma unroll
        for (int j = 0; j < V; ++j) {
            if (f3[j] || n <= 0) continue;
            St s = S[j];
            for (int i = 0; i < n; ++i) {
                const float x = Io<IO>::to_f(sk[i * stride + col + j]) * kLog2e;
                const float vv = Io<IO>::to_f(sv[i * stride + col + j]);
                out_one(i, j, exact_step(s, x, vv, w2[j], u2[j]));
            }
        }
    }
}

template <int V>
__device__ __forceinline__ void channel_consts(const float* __restrict__ w,
                                               const float* __restrict__ u, int64_t c, int64_t C,
                                               float (&w2)[V], float (&u2)[V], float (&ew)[V],
                                               float (&eu)[V]) {
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const bool ok = c + j < C;
        const float wn = ok ? __ldg(w + c + j) : 0.f;
        const float un = ok ? __ldg(u + c + j) : 0.f;
        w2[j] = wn * kLog2e;
        u2[j] = un * kLog2e;
        ew[j] = expf(wn);
        eu[j] = expf(un);
    }
}

__device__ __forceinline__ St load_state_log2(const float* __restrict__ s, int64_t BC, int64_t ch) {
    return {s[ch], s[BC + ch], s[2 * BC + ch] * kLog2e};
}

__device__ __forceinline__ void store_state_nat(float* __restrict__ s, int64_t BC, int64_t ch, St x) {
    s[ch] = x.a;
    s[BC + ch] = x.b;
    s[2 * BC + ch] = x.p * kLn2;
}

// ============================================================ chunked scan

template <typename IO, int V, int L, int NW>
struct ScanShape {
    static constexpr int kCg = 32 * V;    // channels per tile
    static constexpr int kTs = L * NW;    // steps per tile
    static constexpr int kThreads = 32 * NW;
    static constexpr int kTileBytes = kTs * kCg * (int)sizeof(IO);
    static constexpr int kSumFloats = 3 * NW * kCg;
    static constexpr int kPreFloats = 3 * kCg;
    static constexpr size_t kSmem =
        1024 + 2 * (size_t)kTileBytes + (size_t)(kSumFloats + kPreFloats) * 4 + 16;
    static_assert(kTs <= 256 && kCg <= 256, "TMA box dims");
    static_assert((kCg * sizeof(IO)) % 16 == 0, "TMA inner box bytes");
};

struct ScanParams {
    int64_t T, C;
    int G;      // channel tiles over all batch rows
    int CGB;    // channel tiles per batch row
    int nseg;   // time segments
    const float* w;
    const float* u;
    const void* k;
    const void* v;
    const float* state_in;
    void* y;
    float* state_out;
    unsigned long long* flags;  // [tiles]
    float* agg;                 // [tiles][3][Cg]
    float* pre;                 // [tiles][3][Cg]
    unsigned long long epoch;
};

template <typename IO, int V, int L, int NW, bool kTMA>
__global__ void __launch_bounds__(32 * NW)
    wkv4_scan_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                     const __grid_constant__ CUtensorMap tmy, const ScanParams p) {
    using Sh = ScanShape<IO, V, L, NW>;
    constexpr int Cg = Sh::kCg, Ts = Sh::kTs;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* base = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    IO* sk = reinterpret_cast<IO*>(base);
    IO* sv = reinterpret_cast<IO*>(base + Sh::kTileBytes);
    float* sa = reinterpret_cast<float*>(base + 2 * Sh::kTileBytes);
    float* sb = sa + NW * Cg;
    float* sp = sb + NW * Cg;
    float* pa = sp + NW * Cg;
    float* pb = pa + Cg;
    float* pp = pb + Cg;
    uint64_t* mbar = reinterpret_cast<uint64_t*>(pp + Cg);

    const int tile = blockIdx.x;
    const int s = tile / p.G;
    const int g = tile - s * p.G;
    const int b = g / p.CGB;
    const int64_t c0 = (int64_t)(g - b * p.CGB) * Cg;
    const int64_t t0 = (int64_t)s * Ts;
    const int64_t T = p.T, C = p.C, BC = (int64_t)(p.G / p.CGB) * C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int col = lane * V;

    if constexpr (kTMA) {
        if (threadIdx.x == 0) {
            prefetch_tmap(&tmk);
            prefetch_tmap(&tmv);
            mbar_init(mbar, 1);
            fence_mbar_init();
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            mbar_arrive_expect_tx(mbar, 2u * Sh::kTileBytes);
            tma_load_3d(sk, &tmk, (int)c0, (int)t0, b, mbar);
            tma_load_3d(sv, &tmv, (int)c0, (int)t0, b, mbar);
        }
    } else {
        const IO* kg = static_cast<const IO*>(p.k);
        const IO* vg = static_cast<const IO*>(p.v);
        for (int idx = threadIdx.x; idx < Ts * Cg; idx += 32 * NW) {
            const int rr = idx / Cg, cc = idx - rr * Cg;
            const int64_t t = t0 + rr, c = c0 + cc;
            IO kx = Io<IO>::from_f(0.f), vx = Io<IO>::from_f(0.f);
            if (t < T && c < C) {
                const int64_t off = ((int64_t)b * T + t) * C + c;
                kx = kg[off];
                vx = vg[off];
            }
            sk[idx] = kx;
            sv[idx] = vx;
        }
    }

    float w2[V], u2[V], ew[V], eu[V];
    channel_consts<V>(p.w, p.u, c0 + col, C, w2, u2, ew, eu);
    const int row0 = warp * L;
    const int64_t tc = t0 + row0;
    const int n = (int)max((int64_t)0, min((int64_t)L, T - tc));
    const int n_tile = (int)min((int64_t)Ts, T - t0);

    if constexpr (kTMA) {
        const bool ok = mbar_wait_bounded(mbar, 0);
        if (__syncthreads_or(!ok)) {
            if (threadIdx.x == 0) raise_error(kErrTmaWait);
            mbar_wait_bounded(mbar, 0);  // let copies in flight land before the CTA leaves
            return;
        }
    } else {
        __syncthreads();
    }

    // ---- phase 1: chunk summaries
    ChunkRegs<V, L> r;
    St sum[V];
    chunk_phase1<IO, V, L>(r, sk + row0 * Cg, sv + row0 * Cg, Cg, col, n, w2, u2, ew, sum);
#pragma unroll
    for (int j = 0; j < V; ++j) {
        sa[warp * Cg + col + j] = sum[j].a;
        sb[warp * Cg + col + j] = sum[j].b;
        sp[warp * Cg + col + j] = sum[j].p;
    }
    __syncthreads();

    // ---- exclusive prefix of the chunks before this warp's chunk
    St E[V];
#pragma unroll
    for (int j = 0; j < V; ++j) E[j] = empty_state();
    for (int q = 0; q < warp; ++q) {
        const int nq = (int)max((int64_t)0, min((int64_t)L, T - (t0 + q * L)));
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const St Sq = {sa[q * Cg + col + j], sb[q * Cg + col + j], sp[q * Cg + col + j]};
            E[j] = combine(E[j], Sq, (float)nq * w2[j]);
        }
    }

    // ---- segment chaining (last warp): state at the tile start
    if (warp == NW - 1) {
        St agg[V], P[V];
#pragma unroll
        for (int j = 0; j < V; ++j) agg[j] = combine(E[j], sum[j], (float)n * w2[j]);
        if (s == 0) {
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const int64_t c = c0 + col + j;
                P[j] = (p.state_in && c < C) ? load_state_log2(p.state_in, BC, (int64_t)b * C + c)
                                             : empty_state();
            }
        } else {
            // publish this tile's aggregate, then walk back over earlier segments
            float* ag = p.agg + (int64_t)tile * 3 * Cg;
#pragma unroll
            for (int j = 0; j < V; ++j) {
                ag[col + j] = agg[j].a;
                ag[Cg + col + j] = agg[j].b;
                ag[2 * Cg + col + j] = agg[j].p;
            }
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release_u64(p.flags + tile, (p.epoch << 2) | 1ull);

            bool have = false;
            St suf[V];
            int64_t nsuf = 0;
            for (int sj = s - 1; sj >= 0; --sj) {
                const int64_t pid = (int64_t)sj * p.G + g;
                unsigned long long f = 0;
                bool ok = false;
                for (uint32_t it = 0; it < kMaxPolls; ++it) {
                    f = ld_acquire_u64(p.flags + pid);
                    if ((f >> 2) == p.epoch && (f & 3ull) != 0) {
                        ok = true;
                        break;
                    }
                    __nanosleep(64);
                }
                if (__any_sync(0xffffffffu, !ok)) {
                    if (lane == 0) raise_error(kErrLookback);
#pragma unroll
                    for (int j = 0; j < V; ++j) P[j] = empty_state();
                    break;
                }
                const unsigned st = __reduce_min_sync(0xffffffffu, (unsigned)(f & 3ull));
                const float* src = (st == 2 ? p.pre : p.agg) + pid * 3 * Cg;
                St X[V];
#pragma unroll
                for (int j = 0; j < V; ++j)
                    X[j] = {__ldcg(src + col + j), __ldcg(src + Cg + col + j),
                            __ldcg(src + 2 * Cg + col + j)};
                if (st == 2) {
#pragma unroll
                    for (int j = 0; j < V; ++j)
                        P[j] = have ? combine(X[j], suf[j], (float)nsuf * w2[j]) : X[j];
                    break;
                }
#pragma unroll
                for (int j = 0; j < V; ++j)
                    suf[j] = have ? combine(X[j], suf[j], (float)nsuf * w2[j]) : X[j];
                have = true;
                nsuf += Ts;
            }
        }
        St Ps[V];
#pragma unroll
        for (int j = 0; j < V; ++j) Ps[j] = combine(P[j], agg[j], (float)n_tile * w2[j]);
        if (s + 1 < p.nseg) {
            float* pr = p.pre + (int64_t)tile * 3 * Cg;
#pragma unroll
            for (int j = 0; j < V; ++j) {
                pr[col + j] = Ps[j].a;
                pr[Cg + col + j] = Ps[j].b;
                pr[2 * Cg + col + j] = Ps[j].p;
            }
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release_u64(p.flags + tile, (p.epoch << 2) | 2ull);
        } else if (p.state_out) {
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const int64_t c = c0 + col + j;
                if (c < C) store_state_nat(p.state_out, BC, (int64_t)b * C + c, Ps[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < V; ++j) {
            pa[col + j] = P[j].a;
            pb[col + j] = P[j].b;
            pp[col + j] = P[j].p;
        }
    }
    __syncthreads();

    // ---- phase 3: outputs from the state at the chunk start
    St S[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const St P0 = {pa[col + j], pb[col + j], pp[col + j]};
        S[j] = combine(P0, E[j], (float)row0 * w2[j]);
    }
    IO* krow = sk + row0 * Cg;
    if constexpr (kTMA) {
        // y is staged in place of k (each slot is read by its own lane only)
        auto out_vec = [&](int i, const float (&yv)[V]) { store_vec<IO, V>(krow + i * Cg + col, yv); };
        auto out_one = [&](int i, int j, float yv) { krow[i * Cg + col + j] = Io<IO>::from_f(yv); };
        chunk_phase3<IO, V, L>(r, krow, sv + row0 * Cg, Cg, col, n, S, w2, u2, ew, eu, out_vec,
                               out_one);
        fence_proxy_async_smem();
        __syncthreads();
        if (threadIdx.x == 0) {
            tma_store_3d(&tmy, sk, (int)c0, (int)t0, b);
            bulk_commit();
            bulk_wait_read_all();
        }
    } else {
        IO* yg = static_cast<IO*>(p.y);
        const int64_t ybase = ((int64_t)b * T + tc) * C + c0 + col;
        auto out_one = [&](int i, int j, float yv) {
            if (c0 + col + j < C) yg[ybase + (int64_t)i * C + j] = Io<IO>::from_f(yv);
        };
        auto out_vec = [&](int i, const float (&yv)[V]) {
#pragma unroll
            for (int j = 0; j < V; ++j) out_one(i, j, yv[j]);
        };
        chunk_phase3<IO, V, L>(r, krow, sv + row0 * Cg, Cg, col, n, S, w2, u2, ew, eu, out_vec,
                               out_one);
    }
}

// ============================================================ sequential kernel

template <typename IO, int V, int L, int NW, int NS>
struct SeqShape {
    static constexpr int kCw = 32 * V * NW;  // channels per CTA
    static constexpr int kThreads = 32 * NW;
    static constexpr int kStageBytes = L * kCw * (int)sizeof(IO);  // one tensor, one stage
    static constexpr size_t kSmem = 1024 + 2 * (size_t)NS * kStageBytes + NS * 8;
    static_assert(kCw <= 256 && L <= 256, "TMA box dims");
};

struct SeqParams {
    int64_t T, C;
    int CGB;  // channel groups per batch row
    const float* w;
    const float* u;
    const float* state_in;
    void* y;
    float* state_out;
    int64_t BC;
};

template <typename IO, int V, int L, int NW, int NS>
__global__ void __launch_bounds__(32 * NW)
    wkv4_seq_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                    const SeqParams p) {
    using Sh = SeqShape<IO, V, L, NW, NS>;
    constexpr int Cw = Sh::kCw;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* base = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    IO* sk = reinterpret_cast<IO*>(base);                       // [NS][L][Cw]
    IO* sv = reinterpret_cast<IO*>(base + NS * Sh::kStageBytes);  // [NS][L][Cw]
    uint64_t* mbar = reinterpret_cast<uint64_t*>(base + 2 * NS * Sh::kStageBytes);

    const int b = blockIdx.x / p.CGB;
    const int64_t c0 = (int64_t)(blockIdx.x - b * p.CGB) * Cw;
    const int64_t T = p.T, C = p.C;
    const int col = threadIdx.x * V;
    const int64_t c = c0 + col;
    const int64_t nchunks = (T + L - 1) / L;

    if (threadIdx.x == 0) {
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
        for (int st = 0; st < NS; ++st) mbar_init(mbar + st, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int st = 0; st < NS && st < nchunks; ++st) {
            mbar_arrive_expect_tx(mbar + st, 2u * Sh::kStageBytes);
            tma_load_3d(sk + st * L * Cw, &tmk, (int)c0, st * L, b, mbar + st);
            tma_load_3d(sv + st * L * Cw, &tmv, (int)c0, st * L, b, mbar + st);
        }
    }

    float w2[V], u2[V], ew[V], eu[V];
    channel_consts<V>(p.w, p.u, c, C, w2, u2, ew, eu);
    St S[V];
#pragma unroll
    for (int j = 0; j < V; ++j)
        S[j] = (p.state_in && c + j < C) ? load_state_log2(p.state_in, p.BC, (int64_t)b * C + c + j)
                                         : empty_state();
    IO* yg = static_cast<IO*>(p.y);
    const bool vec_ok = c + V <= C;

    for (int64_t q = 0; q < nchunks; ++q) {
        const int st = (int)(q % NS);
        const uint32_t parity = (uint32_t)((q / NS) & 1);
        const bool ok = mbar_wait_bounded(mbar + st, parity);
        if (__syncthreads_or(!ok)) {
            if (threadIdx.x == 0) raise_error(kErrTmaWait);
            for (int s2 = 0; s2 < NS; ++s2) mbar_wait_bounded(mbar + s2, parity);
            return;
        }
        const int64_t tq = q * L;
        const int n = (int)min((int64_t)L, T - tq);
        const IO* kr = sk + st * L * Cw;
        const IO* vr = sv + st * L * Cw;
        ChunkRegs<V, L> r;
        St sum[V];
        chunk_phase1<IO, V, L>(r, kr, vr, Cw, col, n, w2, u2, ew, sum);
        const int64_t ybase = ((int64_t)b * T + tq) * C + c;
        auto out_one = [&](int i, int j, float yv) {
            if (c + j < C) yg[ybase + (int64_t)i * C + j] = Io<IO>::from_f(yv);
        };
        auto out_vec = [&](int i, const float (&yv)[V]) {
            if (vec_ok) {
                store_vec<IO, V>(yg + ybase + (int64_t)i * C, yv);
            } else {
#pragma unroll
                for (int j = 0; j < V; ++j) out_one(i, j, yv[j]);
            }
        };
        chunk_phase3<IO, V, L>(r, kr, vr, Cw, col, n, S, w2, u2, ew, eu, out_vec, out_one);
#pragma unroll
        for (int j = 0; j < V; ++j) S[j] = combine(S[j], sum[j], (float)n * w2[j]);
        __syncthreads();  // stage st fully consumed
        if (threadIdx.x == 0 && q + NS < nchunks) {
            mbar_arrive_expect_tx(mbar + st, 2u * Sh::kStageBytes);
            tma_load_3d(sk + st * L * Cw, &tmk, (int)c0, (int)((q + NS) * L), b, mbar + st);
            tma_load_3d(sv + st * L * Cw, &tmv, (int)c0, (int)((q + NS) * L), b, mbar + st);
        }
    }
    if (p.state_out) {
#pragma unroll
        for (int j = 0; j < V; ++j)
            if (c + j < C) store_state_nat(p.state_out, p.BC, (int64_t)b * C + c + j, S[j]);
    }
}

// ============================================================ per-step kernels

struct StepParams {
    int64_t B, T, C;
    const float* w;
    const float* u;
    const void* k;
    const void* v;
    const float* state_in;
    void* y;
    float* state_out;
};

// One thread per channel; the per-step max-trick in natural units, any T.
template <typename IO>
__global__ void __launch_bounds__(256) wkv4_step_kernel(const StepParams p) {
    const int64_t BC = p.B * p.C;
    const int64_t ch = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (ch >= BC) return;
    const int64_t b = ch / p.C, c = ch - b * p.C;
    St s = p.state_in ? St{p.state_in[ch], p.state_in[BC + ch], p.state_in[2 * BC + ch]}
                      : St{0.f, 0.f, kEmptyMaxNat};
    const float w = p.w[c], u = p.u[c];
    const IO* kg = static_cast<const IO*>(p.k);
    const IO* vg = static_cast<const IO*>(p.v);
    IO* yg = static_cast<IO*>(p.y);
    for (int64_t t = 0; t < p.T; ++t) {
        const int64_t off = (b * p.T + t) * p.C + c;
        const float y = exact_step_nat(s, Io<IO>::to_f(kg[off]), Io<IO>::to_f(vg[off]), w, u);
        yg[off] = Io<IO>::from_f(y);
    }
    if (p.state_out) {
        p.state_out[ch] = s.a;
        p.state_out[BC + ch] = s.b;
        p.state_out[2 * BC + ch] = s.p;
    }
}

// T = 1, V channels per thread with vector accesses; the caller checks that
// C % V == 0 and every pointer is aligned to its vector width.
template <typename IO, int V>
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
    if (p.state_in) {
        load_vec<float, V>(p.state_in + ch, a);
        load_vec<float, V>(p.state_in + BC + ch, bb);
        load_vec<float, V>(p.state_in + 2 * BC + ch, pp);
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
        St s = {a[j], bb[j], pp[j]};
        yy[j] = exact_step_nat(s, kk[j], vv[j], w[j], u[j]);
        a[j] = s.a;
        bb[j] = s.b;
        pp[j] = s.p;
    }
    store_vec<IO, V>(static_cast<IO*>(p.y) + ch, yy);
    if (p.state_out) {
        store_vec<float, V>(p.state_out + ch, a);
        store_vec<float, V>(p.state_out + BC + ch, bb);
        store_vec<float, V>(p.state_out + 2 * BC + ch, pp);
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

// ============================================================ launchers

// Kernel configurations.  fp32: 32 channels x 256 steps per scan tile
// (128-byte rows); 16-bit: 64 channels x 128 steps.
#define WKV4_SCAN_F32 float, 1, 32, 8
#define WKV4_SCAN_F16 __half, 2, 16, 8
#define WKV4_SCAN_BF16 __nv_bfloat16, 2, 16, 8
#define WKV4_SEQ_F32 float, 1, 16, 4, 4
#define WKV4_SEQ_F16 __half, 2, 16, 4, 4
#define WKV4_SEQ_BF16 __nv_bfloat16, 2, 16, 4, 4

size_t dtype_size(int dtype) { return dtype == WKV4_F32 ? 4 : 2; }

// The dynamic shared memory limit is a per-device function attribute: set it
// once per device for each kernel instantiation.
struct DeviceFlags {
    std::atomic<bool> done[64];
};

template <typename Kern>
static cudaError_t ensure_smem_attr(DeviceFlags& f, Kern kern, size_t smem) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && f.done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess && dev >= 0 && dev < 64) f.done[dev].store(true, std::memory_order_release);
    return e;
}

template <typename IO, int V, int L, int NW>
static Geom scan_geom_t() {
    using Sh = ScanShape<IO, V, L, NW>;
    return {Sh::kCg, Sh::kTs, Sh::kThreads, Sh::kSmem};
}
template <typename IO, int V, int L, int NW, int NS>
static Geom seq_geom_t() {
    using Sh = SeqShape<IO, V, L, NW, NS>;
    return {Sh::kCw, L, Sh::kThreads, Sh::kSmem};
}

Geom scan_geom(int dtype) {
    if (dtype == WKV4_F32) return scan_geom_t<WKV4_SCAN_F32>();
    if (dtype == WKV4_F16) return scan_geom_t<WKV4_SCAN_F16>();
    return scan_geom_t<WKV4_SCAN_BF16>();
}

Geom seq_geom(int dtype) {
    if (dtype == WKV4_F32) return seq_geom_t<WKV4_SEQ_F32>();
    if (dtype == WKV4_F16) return seq_geom_t<WKV4_SEQ_F16>();
    return seq_geom_t<WKV4_SEQ_BF16>();
}

size_t scan_scratch_bytes(int64_t B, int64_t T, int64_t C, int dtype) {
    const Geom g = scan_geom(dtype);
    const int64_t nseg = (T + g.box_t - 1) / g.box_t;
    if (nseg <= 1) return 0;
    const int64_t tiles = B * ((C + g.box_c - 1) / g.box_c) * nseg;
    // flags, then aggregates, then prefixes (each 256-byte aligned)
    const size_t flags = ((size_t)tiles * 8 + 255) & ~(size_t)255;
    const size_t tri = ((size_t)tiles * 3 * g.box_c * 4 + 255) & ~(size_t)255;
    return flags + 2 * tri;
}

template <typename IO, int V, int L, int NW, bool kTMA>
static cudaError_t launch_scan_t(const FwdArgs& a, const CUtensorMap* tk, const CUtensorMap* tv,
                                 const CUtensorMap* ty, void* scratch, unsigned long long epoch) {
    using Sh = ScanShape<IO, V, L, NW>;
    auto kern = wkv4_scan_kernel<IO, V, L, NW, kTMA>;
    static DeviceFlags attr_set;
    cudaError_t e = ensure_smem_attr(attr_set, kern, Sh::kSmem);
    if (e != cudaSuccess) return e;
    ScanParams p;
    p.T = a.T;
    p.C = a.C;
    p.CGB = (int)((a.C + Sh::kCg - 1) / Sh::kCg);
    p.G = (int)(a.B * p.CGB);
    p.nseg = (int)((a.T + Sh::kTs - 1) / Sh::kTs);
    p.w = a.w;
    p.u = a.u;
    p.k = a.k;
    p.v = a.v;
    p.state_in = a.state_in;
    p.y = a.y;
    p.state_out = a.state_out;
    p.epoch = epoch;
    p.flags = nullptr;
    p.agg = p.pre = nullptr;
    if (p.nseg > 1) {
        const int64_t tiles = (int64_t)p.G * p.nseg;
        const size_t flags = ((size_t)tiles * 8 + 255) & ~(size_t)255;
        const size_t tri = ((size_t)tiles * 3 * Sh::kCg * 4 + 255) & ~(size_t)255;
        p.flags = static_cast<unsigned long long*>(scratch);
        p.agg = reinterpret_cast<float*>(static_cast<char*>(scratch) + flags);
        p.pre = reinterpret_cast<float*>(static_cast<char*>(scratch) + flags + tri);
    }
    CUtensorMap dummy;
    memset(&dummy, 0, sizeof(dummy));
    const int64_t grid = (int64_t)p.G * p.nseg;
    kern<<<(unsigned)grid, Sh::kThreads, Sh::kSmem, a.stream>>>(tk ? *tk : dummy, tv ? *tv : dummy,
                                                                ty ? *ty : dummy, p);
    return cudaGetLastError();
}

cudaError_t launch_scan(const FwdArgs& a, const CUtensorMap* tk, const CUtensorMap* tv,
                        const CUtensorMap* ty, void* scratch, unsigned long long epoch) {
    const bool tma = tk != nullptr;
    switch (a.dtype) {
        case WKV4_F32:
            return tma ? launch_scan_t<WKV4_SCAN_F32, true>(a, tk, tv, ty, scratch, epoch)
                       : launch_scan_t<WKV4_SCAN_F32, false>(a, tk, tv, ty, scratch, epoch);
        case WKV4_F16:
            return tma ? launch_scan_t<WKV4_SCAN_F16, true>(a, tk, tv, ty, scratch, epoch)
                       : launch_scan_t<WKV4_SCAN_F16, false>(a, tk, tv, ty, scratch, epoch);
        default:
            return tma ? launch_scan_t<WKV4_SCAN_BF16, true>(a, tk, tv, ty, scratch, epoch)
                       : launch_scan_t<WKV4_SCAN_BF16, false>(a, tk, tv, ty, scratch, epoch);
    }
}

template <typename IO, int V, int L, int NW, int NS>
static cudaError_t launch_seq_t(const FwdArgs& a, const CUtensorMap* tk, const CUtensorMap* tv) {
    using Sh = SeqShape<IO, V, L, NW, NS>;
    auto kern = wkv4_seq_kernel<IO, V, L, NW, NS>;
    static DeviceFlags attr_set;
    cudaError_t e = ensure_smem_attr(attr_set, kern, Sh::kSmem);
    if (e != cudaSuccess) return e;
    SeqParams p;
    p.T = a.T;
    p.C = a.C;
    p.CGB = (int)((a.C + Sh::kCw - 1) / Sh::kCw);
    p.w = a.w;
    p.u = a.u;
    p.state_in = a.state_in;
    p.y = a.y;
    p.state_out = a.state_out;
    p.BC = a.B * a.C;
    const int64_t grid = a.B * p.CGB;
    kern<<<(unsigned)grid, Sh::kThreads, Sh::kSmem, a.stream>>>(*tk, *tv, p);
    return cudaGetLastError();
}

cudaError_t launch_seq(const FwdArgs& a, const CUtensorMap* tk, const CUtensorMap* tv) {
    switch (a.dtype) {
        case WKV4_F32: return launch_seq_t<WKV4_SEQ_F32>(a, tk, tv);
        case WKV4_F16: return launch_seq_t<WKV4_SEQ_F16>(a, tk, tv);
        default: return launch_seq_t<WKV4_SEQ_BF16>(a, tk, tv);
    }
}

static StepParams step_params(const FwdArgs& a) {
    StepParams p;
    p.B = a.B;
    p.T = a.T;
    p.C = a.C;
    p.w = a.w;
    p.u = a.u;
    p.k = a.k;
    p.v = a.v;
    p.state_in = a.state_in;
    p.y = a.y;
    p.state_out = a.state_out;
    return p;
}

cudaError_t launch_step(const FwdArgs& a) {
    const StepParams p = step_params(a);
    const int64_t BC = a.B * a.C;
    const unsigned grid = (unsigned)((BC + 255) / 256);
    switch (a.dtype) {
        case WKV4_F32: wkv4_step_kernel<float><<<grid, 256, 0, a.stream>>>(p); break;
        case WKV4_F16: wkv4_step_kernel<__half><<<grid, 256, 0, a.stream>>>(p); break;
        default: wkv4_step_kernel<__nv_bfloat16><<<grid, 256, 0, a.stream>>>(p); break;
    }
    return cudaGetLastError();
}

static bool aligned(const void* ptr, size_t bytes) {
    return ptr == nullptr || ((uintptr_t)ptr % bytes) == 0;
}

cudaError_t launch_decode(const FwdArgs& a) {
    constexpr int V = 4;
    const size_t es = dtype_size(a.dtype);
    const bool vec = (a.C % V == 0) && aligned(a.k, V * es) && aligned(a.v, V * es) &&
                     aligned(a.y, V * es) && aligned(a.w, 16) && aligned(a.u, 16) &&
                     aligned(a.state_in, 16) && aligned(a.state_out, 16);
    if (!vec) return launch_step(a);
    const StepParams p = step_params(a);
    const int64_t threads = a.B * a.C / V;
    const unsigned grid = (unsigned)((threads + 255) / 256);
    switch (a.dtype) {
        case WKV4_F32: wkv4_decode_kernel<float, V><<<grid, 256, 0, a.stream>>>(p); break;
        case WKV4_F16: wkv4_decode_kernel<__half, V><<<grid, 256, 0, a.stream>>>(p); break;
        default: wkv4_decode_kernel<__nv_bfloat16, V><<<grid, 256, 0, a.stream>>>(p); break;
    }
    return cudaGetLastError();
}

cudaError_t launch_copy_state(const FwdArgs& a) {
    const int64_t BC = a.B * a.C;
    if (!a.state_out || BC == 0) return cudaSuccess;
    wkv4_copy_state_kernel<<<(unsigned)((BC + 255) / 256), 256, 0, a.stream>>>(a.state_in,
                                                                               a.state_out, BC);
    return cudaGetLastError();
}

cudaError_t read_device_error(unsigned* bits, bool reset) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(bits, g_device_error, sizeof(unsigned));
    if (e != cudaSuccess) return e;
    if (reset) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned));
    }
    return e;
}

}  // namespace wkv4
