// Chunked scan over (channel tile x time segment) tiles, chained through a
// thread-block cluster.
//
// A cluster of NC CTAs owns one channel tile (Cg = 64 channels of one batch
// row, one channel pair per lane) and walks T in rounds of NC segments of
// Ts = NW L steps; CTA rank r takes segment round * NC + r.  NW (warps per
// CTA) and NC are chosen at launch so that, where the GPU can hold it, the
// whole T is one round of one wave.  Inside a CTA each warp owns one chunk of
// L steps; its rows arrive by their own TMA box and mbarrier, so a warp
// starts as soon as its rows land.  Per round:
//   1. every warp summarises its chunk from the empty state (chunk_phase1);
//   2. warp 0 scans the NW chunk summaries (the state contribution before
//      each chunk, the segment's aggregate) and pushes the aggregate into the
//      shared memory of every CTA of the cluster (DSMEM stores, posted);
//   3. one cluster barrier; every warp folds the NC aggregates of the round,
//      from the state carried into the round, into the state at the segment
//      start and the state carried into the next round;
//   4. every warp emits its chunk's outputs (chunk_phase3) into its k rows
//      and sends them out with its own TMA store.
// With several rounds the next round's rows are prefetched into a second
// buffer (NB = 2).  There is no global scratch and no spin-wait on another
// CTA: all exchange is through cluster shared memory and hardware barriers.
#pragma once

#include <cooperative_groups.h>

#include "wkv4_chunk.cuh"

namespace wkv4 {

namespace cg = cooperative_groups;

constexpr int kMaxCluster = 8;

// Register cap of the scan kernel: enough CTAs per SM for the whole grid of
// the common shapes to be resident at once.
#ifndef WKV4_SCAN_MAXNREG
#define WKV4_SCAN_MAXNREG 96
#endif

// Shared-memory layout for nw warps (offsets from a 1024-byte aligned base).
template <typename IO, int L, int NB>
struct ScanLayout {
    static constexpr int kCg = 64;  // channels per tile: 32 lanes x 2
    static constexpr int kChunkBytes = L * kCg * (int)sizeof(IO);  // one warp's rows, one tensor
    static_assert(L <= 256, "TMA box dims");
    static_assert(kChunkBytes % 128 == 0, "TMA destination alignment");
    int nw;
    __host__ __device__ size_t tile() const { return (size_t)nw * kChunkBytes; }
    __host__ __device__ size_t k(int buf) const { return (size_t)buf * 2 * tile(); }
    __host__ __device__ size_t v(int buf) const { return k(buf) + tile(); }
    int nc;
    __host__ __device__ size_t sums() const { return (size_t)NB * 2 * tile(); }        // [nw][Cg] x 16 B
    __host__ __device__ size_t params() const { return sums() + (size_t)nw * kCg * 16; }  // w, u, state [5][Cg] f32
    __host__ __device__ size_t bars() const { return params() + (size_t)5 * kCg * 4; }    // [NB][nw] + 1 x 8 B
    __host__ __device__ size_t agg() const {                                              // [2][nc][Cg] x 16 B
        return (bars() + (size_t)(NB * nw + 1) * 8 + 15) & ~(size_t)15;
    }
    __host__ __device__ size_t bytes() const { return 1024 + agg() + (size_t)2 * nc * kCg * 16; }
};

struct ScanParams {
    int64_t T, C;
    int CGB;     // channel tiles per batch row
    int rounds;  // ceil(segments / NC)
    const float* w;
    const float* u;
    const void* k;  // element-wise variant only
    const void* v;
    const float* state_in;
    void* y;
    float* state_out;
    int64_t BC;
    int bulk_params;  // w, u, state_in are 16-byte aligned: fetch them by bulk copy
};

// (a, b, p) triples in shared memory, stored as three planes of n entries.
struct TripleRef {
    float* a;
    float* b;
    double* p;
    __device__ __forceinline__ St get(int i) const { return {a[i], b[i], p[i]}; }
    __device__ __forceinline__ void put(int i, St s) const {
        a[i] = s.a;
        b[i] = s.b;
        p[i] = s.p;
    }
};

__device__ __forceinline__ TripleRef triples(unsigned char* at, int n) {
    float* a = reinterpret_cast<float*>(at);
    float* b = a + n;
    return {a, b, reinterpret_cast<double*>(b + n)};
}

template <typename IO, int L, int NB, bool kTMA>
__global__ void __maxnreg__(WKV4_SCAN_MAXNREG)
    wkv4_scan_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                     const __grid_constant__ CUtensorMap tmy, const ScanParams p) {
    constexpr int Cg = ScanLayout<IO, L, NB>::kCg;
    constexpr int kChunkBytes = ScanLayout<IO, L, NB>::kChunkBytes;
    const int NW = blockDim.x >> 5;
    cg::cluster_group cluster = cg::this_cluster();
    const int NC = (int)cluster.num_blocks();
    const ScanLayout<IO, L, NB> lay{NW, NC};
    const int Ts = NW * L;
    extern __shared__ unsigned char smem_raw[];
    // align by offsetting the shared array itself (a round trip through an
    // integer would lose the address space and turn every access generic)
    unsigned char* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const TripleRef sums = triples(base + lay.sums(), NW * Cg);      // [NW][Cg]
    uint64_t* mbar = reinterpret_cast<uint64_t*>(base + lay.bars());  // [NB][NW]

    const int rank = (int)cluster.block_rank();
    const int g = blockIdx.x / NC;
    const int b = g / p.CGB;
    const int64_t c0 = (int64_t)(g - b * p.CGB) * Cg;
    const int64_t T = p.T, C = p.C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int col = lane * 2;
    const int64_t seg_stride = (int64_t)NC * Ts;  // steps per round

    auto chunk_len = [&](int j, int q) -> int {  // steps of chunk q of this CTA in round j
        const int64_t tc = (int64_t)j * seg_stride + (int64_t)rank * Ts + (int64_t)q * L;
        return (int)max((int64_t)0, min((int64_t)L, T - tc));
    };
    auto rows_k = [&](int buf) { return reinterpret_cast<IO*>(base + lay.k(buf)) + warp * L * Cg; };
    auto rows_v = [&](int buf) { return reinterpret_cast<IO*>(base + lay.v(buf)) + warp * L * Cg; };
    auto issue_loads = [&](int j) {  // lane 0 of each warp: this warp's rows of round j
        if constexpr (kTMA) {
            if (chunk_len(j, warp) <= 0) return;
            const int buf = j % NB;
            const int t = (int)((int64_t)j * seg_stride + (int64_t)rank * Ts + warp * L);
            uint64_t* bar = mbar + buf * NW + warp;
            mbar_arrive_expect_tx(bar, 2u * kChunkBytes);
            tma_load_3d(rows_k(buf), &tmk, (int)c0, t, b, bar);
            tma_load_3d(rows_v(buf), &tmv, (int)c0, t, b, bar);
        }
    };

    // Per-channel w, u and the state for this tile: a full 64-channel slice
    // with aligned pointers comes by bulk copy on its own mbarrier, issued
    // before the tiles, so it does not queue behind other CTAs' tile traffic.
    PairConsts cc;
    St carry[2];  // every warp: the state carried into the current round
    uint64_t* pbar = mbar + NB * NW;
    float* sw = reinterpret_cast<float*>(base + lay.params());  // [5][Cg]: w, u, a, b, p
    const bool bulk = kTMA && p.bulk_params && c0 + Cg <= C;
    if (bulk) {
        if (threadIdx.x == 0) {
            mbar_init(pbar, 1);
            fence_mbar_init();
            const uint32_t nb = Cg * 4;
            const int64_t ch = (int64_t)b * C + c0;
            mbar_arrive_expect_tx(pbar, (p.state_in ? 5u : 2u) * nb);
            bulk_load(sw, p.w + c0, nb, pbar);
            bulk_load(sw + Cg, p.u + c0, nb, pbar);
            if (p.state_in) {
                bulk_load(sw + 2 * Cg, p.state_in + ch, nb, pbar);
                bulk_load(sw + 3 * Cg, p.state_in + p.BC + ch, nb, pbar);
                bulk_load(sw + 4 * Cg, p.state_in + 2 * p.BC + ch, nb, pbar);
            }
        }
    } else {
        pair_wu(p.w, p.u, c0 + col, C, cc);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int64_t c = c0 + col + j;
            carry[j] = (p.state_in && c < C) ? load_state_log2(p.state_in, p.BC, (int64_t)b * C + c)
                                             : empty_state();
        }
    }
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
    if (bulk) {
        __syncthreads();  // the params barrier is initialised
        if (!mbar_wait_bounded(pbar, 0)) {
            if (lane == 0) atomicOr(&g_device_error, kErrTmaWait);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            cc.w[j] = sw[col + j];
            cc.u[j] = sw[Cg + col + j];
            carry[j] = p.state_in ? St{sw[2 * Cg + col + j], sw[3 * Cg + col + j],
                                       (double)sw[4 * Cg + col + j] * kLog2eD}
                                  : empty_state();
        }
    }
    pair_derive(cc);
    bool failed = false;

    for (int round = 0; round < p.rounds; ++round) {
        const int buf = round % NB;
        const int n = chunk_len(round, warp);
        const int64_t t0 = (int64_t)round * seg_stride + (int64_t)rank * Ts;  // segment start
        IO* kr = rows_k(buf);
        IO* vr = rows_v(buf);
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
        PairRef ref;
        St sum[2];
        chunk_phase1<IO, L>(ref, kr, vr, Cg, col, n, cc, sum);
#pragma unroll
        for (int j = 0; j < 2; ++j) sums.put(warp * Cg + col + j, sum[j]);
        __syncthreads();

        // ---- 2. warp 0: exclusive prefix of the chunk summaries (in place); the
        //         segment aggregate is pushed into slot [round & 1][rank] of every
        //         CTA of the cluster (posted remote stores)
        const int slot = round & 1;
        const TripleRef agg = triples(base + lay.agg() + (size_t)slot * NC * Cg * 16, NC * Cg);
        if (warp == 0) {
            St acc[2] = {empty_state(), empty_state()};
#pragma unroll 1
            for (int q = 0; q < NW; ++q) {
                const double nq = (double)chunk_len(round, q);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int i = q * Cg + col + j;
                    const St Sq = sums.get(i);
                    sums.put(i, acc[j]);
                    acc[j] = combine(acc[j], Sq, nq * cc.w2[j]);
                }
            }
            const int off = rank * Cg + col;
#pragma unroll 1
            for (int q = 0; q < NC; ++q) {
                float* ra = cluster.map_shared_rank(agg.a, q);
                float* rb = cluster.map_shared_rank(agg.b, q);
                double* rp = cluster.map_shared_rank(agg.p, q);
                *reinterpret_cast<float2*>(ra + off) = make_float2(acc[0].a, acc[1].a);
                *reinterpret_cast<float2*>(rb + off) = make_float2(acc[0].b, acc[1].b);
                rp[off] = acc[0].p;
                rp[off + 1] = acc[1].p;
            }
        }

        // ---- 3. every warp folds the round's aggregates from its own shared memory
        cluster.sync();
        St P[2];
#pragma unroll 1
        for (int q = 0; q < NC; ++q) {
            const int64_t sq = t0 + (int64_t)(q - rank) * Ts;
            const double nq = (double)max((int64_t)0, min((int64_t)Ts, T - sq));
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                if (q == rank) P[j] = carry[j];
                carry[j] = combine(carry[j], agg.get(q * Cg + col + j), nq * cc.w2[j]);
            }
        }

        // ---- 4. outputs of this warp's chunk
        St S[2];
#pragma unroll
        for (int j = 0; j < 2; ++j)
            S[j] = combine(P[j], sums.get(warp * Cg + col + j), (double)(warp * L) * cc.w2[j]);
        if constexpr (kTMA) {
            // y is staged in place of k (step i reads k_i before writing y_i)
            auto out_pair = [=](int i, f2 y) { Pair<IO>::store(kr + i * Cg + col, y); };
            auto out_one = [=](int i, int j, float y) { kr[i * Cg + col + j] = Io<IO>::from_f(y); };
            chunk_phase3<IO, L>(ref, kr, vr, Cg, col, n, S, cc, out_pair, out_one);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                if (n > 0 && !failed) {
                    tma_store_3d(&tmy, kr, (int)c0, (int)(t0 + warp * L), b);
                    bulk_commit();
                }
                if (round + NB < p.rounds) {
                    bulk_wait_read_all();  // rows free for the next load into this buffer
                    issue_loads(round + NB);
                }
            }
            __syncwarp();
        } else {
            IO* yg = static_cast<IO*>(p.y);
            const int64_t ybase = ((int64_t)b * T + t0 + warp * L) * C + c0 + col;
            const int64_t cpair = c0 + col;
            auto out_one = [=](int i, int j, float y) {
                if (cpair + j < C) yg[ybase + (int64_t)i * C + j] = Io<IO>::from_f(y);
            };
            auto out_pair = [=](int i, f2 y) {
                if (cpair < C) yg[ybase + (int64_t)i * C] = Io<IO>::from_f(lo(y));
                if (cpair + 1 < C) yg[ybase + (int64_t)i * C + 1] = Io<IO>::from_f(hi(y));
            };
            chunk_phase3<IO, L>(ref, kr, vr, Cg, col, n, S, cc, out_pair, out_one);
            __syncwarp();
        }
    }

    if (rank == 0 && warp == 0 && p.state_out) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int64_t c = c0 + col + j;
            if (c < C) store_state_log2(p.state_out, p.BC, (int64_t)b * C + c, carry[j]);
        }
    }
    if constexpr (kTMA) {
        if (lane == 0) bulk_wait_read_all();  // the staged rows stay valid until read
    }
    // No barrier before leaving: peers only write into this CTA's shared
    // memory before a round's cluster barrier, and read only their own.
}

}  // namespace wkv4
