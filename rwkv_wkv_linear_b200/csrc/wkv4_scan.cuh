// Chunked scan over (channel tile x time segment) tiles, chained through a
// thread-block cluster.
//
// A cluster of NC CTAs owns one channel tile (Cg = 32 V channels of one batch
// row) and walks T in rounds of NC segments of Ts = NW L steps; CTA rank r
// takes segment round * NC + r.  Inside a CTA each warp owns one chunk of L
// steps (its rows arrive by their own TMA box and mbarrier, so a warp starts
// as soon as its rows land) and each lane V channels.  Per round:
//   1. every warp summarises its chunk from the empty state (chunk_phase1);
//   2. the chunk summaries are combined inside the CTA into the segment's
//      aggregate, published in the CTA's shared memory;
//   3. one cluster barrier; every warp then reads the NC aggregates of the
//      round from its peers' shared memory (DSMEM) and folds them, from the
//      state carried into the round, into the state at its own chunk start
//      and the state carried into the next round;
//   4. every warp emits its chunk's outputs (chunk_phase3) into its k rows
//      and sends them out with its own TMA store.
// The next round's tiles are prefetched into the second buffer (NB = 2).
// There is no global scratch and no spin-wait on another CTA: all exchange is
// through cluster shared memory and hardware cluster barriers.
#pragma once

#include <cooperative_groups.h>

#include "wkv4_chunk.cuh"

namespace wkv4 {

namespace cg = cooperative_groups;

template <typename IO, int V, int L, int NW, int NB>
struct ScanShape {
    static constexpr int kCg = 32 * V;   // channels per tile
    static constexpr int kTs = L * NW;   // steps per segment
    static constexpr int kThreads = 32 * NW;
    static constexpr int kChunkBytes = L * kCg * (int)sizeof(IO);  // one warp's rows, one tensor
    static constexpr int kTileBytes = NW * kChunkBytes;
    static constexpr size_t kOffSum = (size_t)NB * 2 * kTileBytes;
    static constexpr size_t kOffAgg = kOffSum + (size_t)NW * kCg * 16;   // a, b f32 + p f64
    static constexpr size_t kOffBar = kOffAgg + (size_t)2 * kCg * 16;
    static constexpr size_t kSmem = 1024 + kOffBar + (size_t)NB * NW * 8;
    static_assert(kCg <= 256 && L <= 256, "TMA box dims");
    static_assert((kCg * sizeof(IO)) % 16 == 0, "TMA inner box bytes");
    static_assert(kChunkBytes % 128 == 0, "TMA destination alignment");
};

struct ScanParams {
    int64_t T, C;
    int CGB;     // channel tiles per batch row
    int rounds;  // ceil(nseg / NC)
    const float* w;
    const float* u;
    const void* k;  // element-wise variant only
    const void* v;
    const float* state_in;
    void* y;
    float* state_out;
    int64_t BC;
};

template <typename IO, int V, int L, int NW, int NB, bool kTMA>
__global__ void __launch_bounds__(32 * NW)
    wkv4_scan_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                     const __grid_constant__ CUtensorMap tmy, const ScanParams p) {
    using Sh = ScanShape<IO, V, L, NW, NB>;
    constexpr int Cg = Sh::kCg, Ts = Sh::kTs;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* base = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float* sum_a = reinterpret_cast<float*>(base + Sh::kOffSum);  // [NW][Cg]
    float* sum_b = sum_a + NW * Cg;
    double* sum_p = reinterpret_cast<double*>(sum_b + NW * Cg);
    float* agg_a = reinterpret_cast<float*>(base + Sh::kOffAgg);  // [2][Cg]
    float* agg_b = agg_a + 2 * Cg;
    double* agg_p = reinterpret_cast<double*>(agg_b + 2 * Cg);
    uint64_t* mbar = reinterpret_cast<uint64_t*>(base + Sh::kOffBar);  // [NB][NW]

    cg::cluster_group cluster = cg::this_cluster();
    const int NC = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int g = blockIdx.x / NC;
    const int b = g / p.CGB;
    const int64_t c0 = (int64_t)(g - b * p.CGB) * Cg;
    const int64_t T = p.T, C = p.C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int col = lane * V;
    const int64_t seg_stride = (int64_t)NC * Ts;  // steps per round

    auto tile_k = [&](int buf) { return reinterpret_cast<IO*>(base + (size_t)buf * 2 * Sh::kTileBytes); };
    auto tile_v = [&](int buf) {
        return reinterpret_cast<IO*>(base + (size_t)buf * 2 * Sh::kTileBytes + Sh::kTileBytes);
    };
    // steps of this warp's chunk in round j
    auto chunk_n = [&](int j) -> int {
        const int64_t tc = (int64_t)j * seg_stride + (int64_t)rank * Ts + (int64_t)warp * L;
        return (int)max((int64_t)0, min((int64_t)L, T - tc));
    };
    auto issue_loads = [&](int j) {  // lane 0 of each warp, own rows of round j
        const int buf = j % NB;
        if (chunk_n(j) <= 0) return;
        const int t = (int)((int64_t)j * seg_stride + (int64_t)rank * Ts + warp * L);
        uint64_t* bar = mbar + buf * NW + warp;
        if constexpr (kTMA) {
            mbar_arrive_expect_tx(bar, 2u * Sh::kChunkBytes);
            tma_load_3d(tile_k(buf) + warp * L * Cg, &tmk, (int)c0, t, b, bar);
            tma_load_3d(tile_v(buf) + warp * L * Cg, &tmv, (int)c0, t, b, bar);
        }
    };

    if constexpr (kTMA) {
        if (lane == 0) {
            if (warp == 0) {
                prefetch_tmap(&tmk);
                prefetch_tmap(&tmv);
                prefetch_tmap(&tmy);
            }
            for (int buf = 0; buf < NB; ++buf) mbar_init(mbar + buf * NW + warp, 1);
            fence_mbar_init();
            for (int j = 0; j < NB && j < p.rounds; ++j) issue_loads(j);
        }
        __syncwarp();
    }

    ChanConsts cc[V];
    channel_consts<V>(p.w, p.u, c0 + col, C, cc);
    St carry[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const int64_t c = c0 + col + j;
        carry[j] = (p.state_in && c < C) ? load_state_log2(p.state_in, p.BC, (int64_t)b * C + c)
                                         : empty_state();
    }
    bool failed = false;

    for (int round = 0; round < p.rounds; ++round) {
        const int buf = round % NB;
        const int n = chunk_n(round);
        const int64_t t0 = (int64_t)round * seg_stride + (int64_t)rank * Ts;  // segment start
        IO* kr = tile_k(buf) + warp * L * Cg;
        IO* vr = tile_v(buf) + warp * L * Cg;
        if constexpr (kTMA) {
            if (n > 0 && !failed &&
                !mbar_wait_bounded(mbar + buf * NW + warp, (uint32_t)((round / NB) & 1))) {
                failed = true;
                if (lane == 0) atomicOr(&g_device_error, kErrTmaWait);
            }
        } else {
            // element-wise loads of this warp's rows (any alignment, zero fill)
            const IO* kg = static_cast<const IO*>(p.k);
            const IO* vg = static_cast<const IO*>(p.v);
            for (int idx = lane; idx < L * Cg; idx += 32) {
                const int rr = idx / Cg, ci = idx - rr * Cg;
                const int64_t t = t0 + warp * L + rr, c = c0 + ci;
                IO kx = Io<IO>::from_f(0.f), vx = Io<IO>::from_f(0.f);
                if (t < T && c < C) {
                    const int64_t off = ((int64_t)b * T + t) * C + c;
                    kx = kg[off];
                    vx = vg[off];
                }
                kr[idx] = kx;
                vr[idx] = vx;
            }
            __syncwarp();
        }

        // ---- 1. chunk summaries
        ChunkRegs<V, L> r;
        St sum[V];
        chunk_phase1<IO, V, L>(r, kr, vr, Cg, col, n, cc, sum);
#pragma unroll
        for (int j = 0; j < V; ++j) {
            sum_a[warp * Cg + col + j] = sum[j].a;
            sum_b[warp * Cg + col + j] = sum[j].b;
            sum_p[warp * Cg + col + j] = sum[j].p;
        }
        __syncthreads();

        // ---- 2. exclusive prefix of the chunks before this warp; segment aggregate
        St E[V];
#pragma unroll
        for (int j = 0; j < V; ++j) E[j] = empty_state();
        for (int q = 0; q < warp; ++q) {
            const int64_t tq = t0 + (int64_t)q * L;
            const int nq = (int)max((int64_t)0, min((int64_t)L, T - tq));
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const St Sq = {sum_a[q * Cg + col + j], sum_b[q * Cg + col + j], sum_p[q * Cg + col + j]};
                E[j] = combine(E[j], Sq, (double)nq * cc[j].w2);
            }
        }
        const int slot = round & 1;
        if (warp == NW - 1) {
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const St A = combine(E[j], sum[j], (double)n * cc[j].w2);
                agg_a[slot * Cg + col + j] = A.a;
                agg_b[slot * Cg + col + j] = A.b;
                agg_p[slot * Cg + col + j] = A.p;
            }
        }

        // ---- 3. exchange segment aggregates across the cluster
        cluster.sync();
        St P[V], next[V];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            P[j] = carry[j];
            next[j] = carry[j];
        }
        for (int q = 0; q < NC; ++q) {
            const int64_t sq = t0 + (int64_t)(q - rank) * Ts;
            const int nq = (int)max((int64_t)0, min((int64_t)Ts, T - sq));
            const float* pa = cluster.map_shared_rank(agg_a + slot * Cg, q);
            const float* pb = cluster.map_shared_rank(agg_b + slot * Cg, q);
            const double* pp = cluster.map_shared_rank(agg_p + slot * Cg, q);
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const St Aq = {pa[col + j], pb[col + j], pp[col + j]};
                next[j] = combine(next[j], Aq, (double)nq * cc[j].w2);
                if (q + 1 == rank) P[j] = next[j];
            }
        }

        // ---- 4. outputs of this warp's chunk
        St S[V];
#pragma unroll
        for (int j = 0; j < V; ++j) S[j] = combine(P[j], E[j], (double)(warp * L) * cc[j].w2);
        if constexpr (kTMA) {
            auto out_vec = [&](int i, const float (&yv)[V]) { store_vec<IO, V>(kr + i * Cg + col, yv); };
            auto out_one = [&](int i, int j, float yv) { kr[i * Cg + col + j] = Io<IO>::from_f(yv); };
            chunk_phase3<IO, V, L>(r, kr, vr, Cg, col, n, S, cc, out_vec, out_one);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && n > 0) {
                if (!failed) tma_store_3d(&tmy, kr, (int)c0, (int)(t0 + warp * L), b);
                bulk_commit();
                bulk_wait_read_all();  // rows free for the next load into this buffer
                if (round + NB < p.rounds) issue_loads(round + NB);
            } else if (lane == 0 && round + NB < p.rounds) {
                issue_loads(round + NB);
            }
            __syncwarp();
        } else {
            IO* yg = static_cast<IO*>(p.y);
            const int64_t ybase = ((int64_t)b * T + t0 + warp * L) * C + c0 + col;
            auto out_one = [&](int i, int j, float yv) {
                if (c0 + col + j < C) yg[ybase + (int64_t)i * C + j] = Io<IO>::from_f(yv);
            };
            auto out_vec = [&](int i, const float (&yv)[V]) {
#pragma unroll
                for (int j = 0; j < V; ++j) out_one(i, j, yv[j]);
            };
            chunk_phase3<IO, V, L>(r, kr, vr, Cg, col, n, S, cc, out_vec, out_one);
            __syncwarp();
        }
#pragma unroll
        for (int j = 0; j < V; ++j) carry[j] = next[j];
    }

    if (rank == 0 && warp == 0 && p.state_out) {
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const int64_t c = c0 + col + j;
            if (c < C) store_state_log2(p.state_out, p.BC, (int64_t)b * C + c, carry[j]);
        }
    }
    // peers may still be reading this CTA's aggregates
    cluster.sync();
}

}  // namespace wkv4
