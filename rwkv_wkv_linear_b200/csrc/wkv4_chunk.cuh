// Per-chunk routines shared by the chunked-scan and sequential kernels.
//
// One lane owns V channels of one chunk of n <= L consecutive steps whose
// rows sit in shared memory (row stride `stride` elements, the lane's
// channels at column `col`).  chunk_phase1 computes the chunk's summary from
// the empty state (its A, D and max) and keeps e[j][i] = 2^{k_i log2e - r_j}
// (r_j = the chunk's max k in log2 units, rounded to fp32) for chunk_phase3,
// which produces the outputs from the state at the chunk's start.
#pragma once

#include "wkv4_device.cuh"

namespace wkv4 {

template <int V, int L>
struct ChunkRegs {
    float e[V][L];
    float kref[V];  // chunk reference: max k * log2e, rounded to fp32
    bool fast[V];
};

struct ChanConsts {
    float w, u;     // natural units
    float ew, eu;   // e^w, e^u
    double w2, u2;  // log2 units
};

template <int V>
__device__ __forceinline__ void channel_consts(const float* __restrict__ w,
                                               const float* __restrict__ u, int64_t c, int64_t C,
                                               ChanConsts (&cc)[V]) {
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const bool ok = c + j < C;
        const float wn = ok ? __ldg(w + c + j) : 0.f;
        const float un = ok ? __ldg(u + c + j) : 0.f;
        cc[j].w = wn;
        cc[j].u = un;
        cc[j].ew = expf(wn);
        cc[j].eu = expf(un);
        cc[j].w2 = (double)wn * kLog2eD;
        cc[j].u2 = (double)un * kLog2eD;
    }
}

template <typename IO, int V, int L>
__device__ __forceinline__ void chunk_phase1(ChunkRegs<V, L>& r, const IO* sk, const IO* sv,
                                             int stride, int col, int n,
                                             const ChanConsts (&cc)[V], St (&sum)[V]) {
    float kmax[V], kmin[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        kmax[j] = -3.0e38f;
        kmin[j] = 3.0e38f;
    }
#pragma unroll
    for (int i = 0; i < L; ++i) {
        if (i < n) {
            float kk[V];
            load_vec<IO, V>(sk + i * stride + col, kk);
#pragma unroll
            for (int j = 0; j < V; ++j) {
                r.e[j][i] = kk[j];
                kmax[j] = fmaxf(kmax[j], kk[j]);
                kmin[j] = fminf(kmin[j], kk[j]);
            }
        }
    }
    float A[V], D[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        r.fast[j] = (n > 0) && fast_ok(kmax[j], kmin[j], cc[j].u, cc[j].w);
        r.kref[j] = kmax[j] * kLog2e;
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
                const float ee = ex2(fmaf(r.e[j][i], kLog2e, -r.kref[j]));
                r.e[j][i] = ee;
                A[j] = fmaf(cc[j].ew, A[j], ee * vv[j]);
                D[j] = fmaf(cc[j].ew, D[j], ee);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < V; ++j) {
        if (n <= 0) {
            sum[j] = empty_state();
        } else if (r.fast[j]) {
            sum[j] = normalized(A[j], D[j], (double)r.kref[j]);
        } else {
            // per-step max-trick from the empty state
            St s = empty_state();
            for (int i = 0; i < n; ++i)
                exact_update(s, Io<IO>::to_f(sk[i * stride + col + j]),
                             Io<IO>::to_f(sv[i * stride + col + j]), cc[j].w2);
            sum[j] = s;
        }
    }
}

// Outputs of the chunk from the state S at its start, through
// out_vec(i, values[V]) or out_one(i, j, value).  Channels that take the
// per-step path read k again from shared memory; a fast channel's slot may
// already hold its y by then when y is staged in place of k, so fast
// channels are written one by one whenever some channel of the lane is slow.
template <typename IO, int V, int L, typename OutVec, typename OutOne>
__device__ __forceinline__ void chunk_phase3(const ChunkRegs<V, L>& r, const IO* sk, const IO* sv,
                                             int stride, int col, int n, const St (&S)[V],
                                             const ChanConsts (&cc)[V], OutVec out_vec,
                                             OutOne out_one) {
    bool f3[V];
    bool all_fast = true;
    float Ah[V], Dh[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const double lift = S[j].p - (double)r.kref[j];
        f3[j] = r.fast[j] && (lift <= (double)(kFastStateLift * kLog2e));
        all_fast = all_fast && f3[j];
        const float sc = ex2((float)lift);
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
                const float eb = cc[j].eu * ee;
                yv[j] = __fdividef(fmaf(eb, vv[j], Ah[j]), Dh[j] + eb);
                Ah[j] = fmaf(cc[j].ew, Ah[j], ee * vv[j]);
                Dh[j] = fmaf(cc[j].ew, Dh[j], ee);
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
                const float k = Io<IO>::to_f(sk[i * stride + col + j]);
                const float v = Io<IO>::to_f(sv[i * stride + col + j]);
                out_one(i, j, exact_step(s, k, v, cc[j].w2, cc[j].u2));
            }
        }
    }
}

}  // namespace wkv4
