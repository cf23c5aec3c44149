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
//   1. every warp summarises its chunk from the empty state (chunk_phase1
//      with stash: the per-step numerators and denominators of its outputs
//      go to tensor memory);
//   2. warp 0 scans the NW chunk summaries (the state contribution before
//      each chunk, the segment's aggregate) and pushes the aggregate into the
//      shared memory of every CTA of the cluster by asynchronous DSMEM stores
//      that complete on the receiving CTA's barrier of that round's slot;
//   3. once all NC aggregates of the round have landed, every warp folds
//      them, from the state carried into the round, into the state at the
//      segment start and the state carried into the next round;
//   4. every warp computes its chunk's outputs from the stash into its k rows
//      and sends them out with its own TMA store.
// With several rounds the next round's rows are loaded into a second buffer
// (NB = 2).
// There is no global scratch: all exchange is through cluster shared memory.
// Aggregate slots alternate between rounds; a slot's next round's stores
// come only after every CTA's own push of the round in between, which
// follows its reads of the slot.  Every wait is bounded.
#pragma once

#include <cooperative_groups.h>

#include "wkv4_chunk.cuh"

namespace wkv4 {

namespace cg = cooperative_groups;

constexpr int kMaxCluster = 8;  // cluster sizes 1, 2, 4, 8; warps per CTA 4 or 8

// Register cap of the scan kernel: two CTAs of 8 warps per SM.
#ifndef WKV4_SCAN_MAXNREG
#define WKV4_SCAN_MAXNREG 128
#endif

// Shared-memory layout for nw warps and clusters of nc (offsets from a
// 128-byte aligned base): NB row buffers of k and v, the chunk summaries,
// the tile's w, u and state, barriers, two slots of aggregates.
template <typename IO, int L, int NB>
struct ScanLayout {
    static constexpr int kCg = 64;  // channels per tile: 32 lanes x 2
    static constexpr int kChunkBytes = L * kCg * (int)sizeof(IO);  // one warp's rows, one tensor
    static constexpr int kAlign = 128;                               // TMA destinations
    static_assert(L <= 256 && L % 4 == 0, "TMA box dims, stash column groups");
    static_assert(kChunkBytes % kAlign == 0, "TMA destination alignment");
    int nw, nc;
    __host__ __device__ size_t tile() const { return (size_t)nw * kChunkBytes; }
    __host__ __device__ size_t k(int buf) const { return (size_t)buf * 2 * tile(); }
    __host__ __device__ size_t v(int buf) const { return k(buf) + tile(); }
    // y staging: in place of k with one round, its own tile with several (so
    // that the rows take the next load as soon as the summary pass is done)
    static constexpr bool kOwnY = NB > 1;
    __host__ __device__ size_t ys() const { return kOwnY ? (size_t)NB * 2 * tile() : k(0); }
    __host__ __device__ size_t sums() const {  // [nw][Cg] x 16 B
        return (size_t)NB * 2 * tile() + (kOwnY ? tile() : 0);
    }
    __host__ __device__ size_t params() const { return sums() + (size_t)nw * kCg * 16; }  // [5][Cg] f32
    __host__ __device__ size_t agg(int slot) const {                                    // [2][nc][Cg] x 16 B
        return params() + (size_t)5 * kCg * 4 + (size_t)slot * nc * kCg * 16;
    }
    // rows [NB][nw], params, aggregate slots [2] x 8 B
    __host__ __device__ size_t bars() const { return agg(2); }
    __host__ __device__ size_t tslot() const { return bars() + (size_t)(NB * nw + 3) * 8; }
    __host__ __device__ size_t bytes() const { return kAlign + tslot() + 8; }
    // tensor-memory columns: 4 a step for each warp, warps w and w + 4
    // sharing a lane quarter
    __host__ __device__ int tmem_cols() const { return nw * L; }
};

struct ScanParams {
    int64_t T, C;
    int CGB;     // channel tiles per batch row
    int rounds;  // ceil(segments / NC)
    const float* w;
    const float* u;
    const void* k;
    const void* v;
    const float* state_in;
    void* y;
    float* state_out;
    int64_t BC;
    int bulk_params;  // w, u, state_in 16-byte aligned and C % 4 == 0: bulk copies
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

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Split cluster barrier (once, at the start): every thread of every CTA of
// the cluster arrives, then waits.
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Warp 0: exclusive prefix of the NW chunk summaries of a segment (in
// place: entry q becomes the state before chunk q) and the segment aggregate
// in acc.  All summaries are read before the chain starts; chunk q spans
// clamp(rem - q L, 0, L) steps.
template <int NW, int L>
__device__ __forceinline__ void scan_chunks(const TripleRef& sums, int col, int rem,
                                            const PairConsts& cc, St (&acc)[2]) {
    constexpr int Cg = 64;
    St x[NW][2];
#pragma unroll
    for (int q = 0; q < NW; ++q)
#pragma unroll
        for (int j = 0; j < 2; ++j) x[q][j] = sums.get(q * Cg + col + j);
    acc[0] = acc[1] = empty_state();
#pragma unroll
    for (int q = 0; q < NW; ++q) {
        const double nq = (double)max(0, min(L, rem - q * L));
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            sums.put(q * Cg + col + j, acc[j]);
            acc[j] = combine(acc[j], x[q][j], nq * cc.w2[j]);
        }
    }
}

// Every warp: fold of the NC segment aggregates of a round into the state at
// this CTA's segment start (P) and the state carried into the next round
// (carry); segment q spans clamp(rrem - q Ts, 0, Ts) steps.
template <int NC>
__device__ __forceinline__ void fold_aggs(const TripleRef& agg, int col, int rank, int64_t rrem,
                                          int Ts, const PairConsts& cc, St (&carry)[2], St (&P)[2]) {
    constexpr int Cg = 64;
    St y[NC][2];
#pragma unroll
    for (int q = 0; q < NC; ++q)
#pragma unroll
        for (int j = 0; j < 2; ++j) y[q][j] = agg.get(q * Cg + col + j);
    P[0] = carry[0];
    P[1] = carry[1];
#pragma unroll
    for (int q = 0; q < NC; ++q) {
        const double nq = (double)max((int64_t)0, min((int64_t)Ts, rrem - (int64_t)q * Ts));
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            if (q == rank) P[j] = carry[j];
            carry[j] = combine(carry[j], y[q][j], nq * cc.w2[j]);
        }
    }
}

template <typename IO, int L, int NB, bool kTMA>
__global__ void __maxnreg__(WKV4_SCAN_MAXNREG)
    wkv4_scan_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                     const __grid_constant__ CUtensorMap tmy, const ScanParams p) {
    using Lay = ScanLayout<IO, L, NB>;
    constexpr int Cg = Lay::kCg;
    constexpr int kChunkBytes = Lay::kChunkBytes;
    constexpr unsigned kAlign = Lay::kAlign;
    const int NW = blockDim.x >> 5;
    cg::cluster_group cluster = cg::this_cluster();
    const int NC = (int)cluster.num_blocks();
    const Lay lay{NW, NC};
    const int Ts = NW * L;
    extern __shared__ unsigned char smem_raw[];
    // align by offsetting the shared array itself (a round trip through an
    // integer would lose the address space and turn every access generic)
    unsigned char* base = smem_raw + ((kAlign - (smem_u32(smem_raw) & (kAlign - 1))) & (kAlign - 1));
    const TripleRef sums = triples(base + lay.sums(), NW * Cg);       // [NW][Cg]
    uint64_t* mbar = reinterpret_cast<uint64_t*>(base + lay.bars());  // rows [NB][NW], params
    uint64_t* pbar = mbar + NB * NW;
    uint64_t* abar = pbar + 1;  // [2]: the aggregates of a round have landed
    uint32_t* tslot = reinterpret_cast<uint32_t*>(base + lay.tslot());
    float* sw = reinterpret_cast<float*>(base + lay.params());  // [5][Cg]: w, u, a, b, p

    const int rank = (int)cluster.block_rank();
    const int g = blockIdx.x / NC;
    const int b = g / p.CGB;
    const int64_t c0 = (int64_t)(g - b * p.CGB) * Cg;
    const int64_t T = p.T, C = p.C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int col = lane * 2;
    const int64_t seg_stride = (int64_t)NC * Ts;  // steps per round
    const IO* kg = static_cast<const IO*>(p.k);
    const IO* vg = static_cast<const IO*>(p.v);
    IO* yg = static_cast<IO*>(p.y);

    auto chunk_len = [&](int j, int q) -> int {  // steps of chunk q of this CTA in round j
        const int64_t tc = (int64_t)j * seg_stride + (int64_t)rank * Ts + (int64_t)q * L;
        return (int)max((int64_t)0, min((int64_t)L, T - tc));
    };
    auto rows_k = [&](int buf) { return reinterpret_cast<IO*>(base + lay.k(buf)) + warp * L * Cg; };
    IO* const ystage = reinterpret_cast<IO*>(base + lay.ys()) + warp * L * Cg;  // with kOwnY
    auto rows_v = [&](int buf) { return reinterpret_cast<IO*>(base + lay.v(buf)) + warp * L * Cg; };
    // Lane 0 of each warp: this warp's rows of round j into buffer j % NB.
    // Every round completes one phase of the warp's barrier of that buffer (a
    // plain arrive where nothing is copied), so its phases stay in step.
    auto issue_rows = [&](int j) {
        if constexpr (kTMA) {
            if (j >= p.rounds) return;
            const int buf = j % NB;
            uint64_t* bar = mbar + buf * NW + warp;
            if (chunk_len(j, warp) > 0) {
                const int t = (int)((int64_t)j * seg_stride + (int64_t)rank * Ts + warp * L);
                mbar_arrive_expect_tx(bar, 2u * kChunkBytes);
                tma_load_3d(rows_k(buf), &tmk, (int)c0, t, b, bar);
                tma_load_3d(rows_v(buf), &tmv, (int)c0, t, b, bar);
            } else {
                mbar_arrive(bar);
            }
        }
    };

    // Per-channel w, u and the state for this tile: a full 64-channel slice
    // with aligned pointers comes by bulk copy on its own mbarrier, issued
    // before the rows, so it does not queue behind other CTAs' row traffic.
    const bool bulk = kTMA && p.bulk_params && c0 + Cg <= C;
    // every CTA of the cluster pushes 32 B per lane into each aggregate slot
    const uint32_t agg_bytes = (uint32_t)NC * 32u * 32u;
    if (warp == 0) tmem_alloc(tslot, (uint32_t)lay.tmem_cols());
    if (threadIdx.x == 0) {
        mbar_init(abar, 1);
        mbar_init(abar + 1, 1);
        fence_mbar_init();
        for (int r = 0; r < 2 && r < p.rounds; ++r) mbar_arrive_expect_tx(abar + r, agg_bytes);
    }
    if constexpr (kTMA) {
        if (lane == 0) {
            if (warp == 0) {
                mbar_init(pbar, 1);
                prefetch_tmap(&tmk);
                prefetch_tmap(&tmv);
                prefetch_tmap(&tmy);
            }
            for (int buf = 0; buf < NB; ++buf) mbar_init(mbar + buf * NW + warp, 1);
            fence_mbar_init();
            if (warp == 0 && bulk) {
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
            for (int j = 0; j < NB; ++j) issue_rows(j);
        }
        __syncwarp();
    }
    PairConsts cc;
    St carry[2];  // every warp: the state carried into the current round
    if (!bulk) {
        pair_wu(p.w, p.u, c0 + col, C, cc);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int64_t c = c0 + col + j;
            carry[j] = (p.state_in && c < C) ? load_state_log2(p.state_in, p.BC, (int64_t)b * C + c)
                                             : empty_state();
        }
    }
    // the tensor-memory base is in shared memory, every barrier initialised
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    // the CTAs of the cluster have all started, with their barriers
    // initialised, before the first DSMEM store (this barrier's wait comes
    // just before it)
    cluster_arrive_relaxed();
    const uint32_t tbase = *tslot;
    // this warp's stash: its lane quarter, 4 L columns for each warp of the quarter
    const uint32_t taddr = tbase + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)((warp >> 2) * 4 * L);
    bool failed = false;
    if (bulk) {
        if (!mbar_wait_bounded(pbar, 0)) {
            failed = true;
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

        // ---- 1. chunk summary and stash; then the rows are free
        PairRef ref;
        St sum[2];
        chunk_phase1<IO, L, true>(ref, kr, vr, Cg, col, n, cc, sum, taddr);
#pragma unroll
        for (int j = 0; j < 2; ++j) sums.put(warp * Cg + col + j, sum[j]);
        if constexpr (kTMA && Lay::kOwnY) {
            __syncwarp();  // every lane has read the rows: they take round + NB's
            if (lane == 0) issue_rows(round + NB);
        }
        __syncthreads();

        // ---- 2. warp 0: exclusive prefix of the chunk summaries (in place); the
        //         segment aggregate goes by asynchronous DSMEM stores into slot
        //         [round & 1][rank] of every CTA of the cluster, each store
        //         completing bytes on that CTA's barrier of the slot
        const int slot = round & 1;
        const TripleRef agg = triples(base + lay.agg(slot), NC * Cg);
        // steps of this CTA's segment (the chunks' lengths follow from it)
        const int rem = (int)max((int64_t)0, min((int64_t)Ts, T - t0));
        if (round == 0) cluster_wait();  // every CTA of the cluster has started
        if (warp == 0) {
            St acc[2];
            if (NW == 8) {
                scan_chunks<8, L>(sums, col, rem, cc, acc);
            } else {
                scan_chunks<4, L>(sums, col, rem, cc, acc);
            }
            const int off = rank * Cg + col;
            const uint32_t la = smem_u32(agg.a + off), lb = smem_u32(agg.b + off);
            const uint32_t lp = smem_u32(agg.p + off), lbar = smem_u32(abar + slot);
#pragma unroll 1
            for (int q = 0; q < NC; ++q) {
                const uint32_t rbar = mapa_u32(lbar, (uint32_t)q);
                st_async_v2f32(mapa_u32(la, (uint32_t)q), acc[0].a, acc[1].a, rbar);
                st_async_v2f32(mapa_u32(lb, (uint32_t)q), acc[0].b, acc[1].b, rbar);
                st_async_v2f64(mapa_u32(lp, (uint32_t)q), acc[0].p, acc[1].p, rbar);
            }
        }
        __syncthreads();  // the exclusive prefixes are in place

        // ---- 3. every warp folds the round's aggregates once they have landed
        if (!failed && !mbar_wait_cluster_bounded(abar + slot, (uint32_t)((round >> 1) & 1))) {
            failed = true;
            if (lane == 0) atomicOr(&g_device_error, kErrExchangeWait);
        }
        // the slot's next use is round + 2: its pushes follow this CTA's own
        // push of round + 1, so the barrier is re-armed well before them
        if (threadIdx.x == 0 && round + 2 < p.rounds) mbar_arrive_expect_tx(abar + slot, agg_bytes);
        St P[2];
        {
            const int64_t rrem = T - (t0 - (int64_t)rank * Ts);  // steps of the round from segment 0 on
            switch (NC) {
                case 1: fold_aggs<1>(agg, col, rank, rrem, Ts, cc, carry, P); break;
                case 2: fold_aggs<2>(agg, col, rank, rrem, Ts, cc, carry, P); break;
                case 4: fold_aggs<4>(agg, col, rank, rrem, Ts, cc, carry, P); break;
                default: fold_aggs<8>(agg, col, rank, rrem, Ts, cc, carry, P); break;
            }
        }

        // ---- 4. outputs of this warp's chunk
        St S[2];
#pragma unroll
        for (int j = 0; j < 2; ++j)
            S[j] = combine(P[j], sums.get(warp * Cg + col + j), (double)(warp * L) * cc.w2[j]);
        const int64_t cpair = c0 + col;
        const int64_t row0 = ((int64_t)b * T + t0 + warp * L) * C + cpair;  // k, v, y offset
        const bool ok0 = cpair < C, ok1 = cpair + 1 < C;
        if constexpr (kTMA) {
            // y staged (in place of k, or in the staging tile once the previous
            // round's store has read it), sent out by one TMA store
            IO* yr = Lay::kOwnY ? ystage : kr;
            if (Lay::kOwnY && round > 0) {
                if (lane == 0) bulk_wait_read_all();
                __syncwarp();
            }
            auto st_one = [=](int s, int j, float y) { yr[s * Cg + col + j] = Io<IO>::from_f(y); };
            auto st_pair = [=](int s, f2 y) { Pair<IO>::store(yr + s * Cg + col, y); };
            chunk_phase3_stash<IO, L>(ref, n, S, cc, taddr, kg + row0, vg + row0, C, ok0, ok1, st_pair,
                                      st_one);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                if (n > 0 && !failed) {
                    tma_store_3d(&tmy, yr, (int)c0, (int)(t0 + warp * L), b);
                    bulk_commit();
                }
            }
            __syncwarp();
        } else {
            // element-wise stores (any alignment)
            IO* yrow = yg + row0;
            auto out_one = [=](int s, int j, float y) {
                if (j == 0 ? ok0 : ok1) yrow[(int64_t)s * C + j] = Io<IO>::from_f(y);
            };
            auto out_pair = [=](int s, f2 y) {
                if (ok0) yrow[(int64_t)s * C] = Io<IO>::from_f(lo(y));
                if (ok1) yrow[(int64_t)s * C + 1] = Io<IO>::from_f(hi(y));
            };
            chunk_phase3_stash<IO, L>(ref, n, S, cc, taddr, kg + row0, vg + row0, C, ok0, ok1, out_pair,
                                      out_one);
        }
    }
    if (kTMA && lane == 0) bulk_wait_read_all();  // staged rows stay valid until read

    if (rank == 0 && warp == 0 && p.state_out) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int64_t c = c0 + col + j;
            if (c < C) store_state_log2(p.state_out, p.BC, (int64_t)b * C + c, carry[j]);
        }
    }
    // Every warp's tensor-memory accesses have completed (each load and each
    // store pass ends in its wait); release the columns.  No cluster barrier
    // is needed before leaving: peers only write into this CTA's shared
    // memory before a round's cluster barrier, and read only their own.
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, (uint32_t)lay.tmem_cols());
}

}  // namespace wkv4
