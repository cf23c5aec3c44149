// Chunked scan over (channel tile x time segment) tiles, chained through a
// thread-block cluster.
//
// A cluster of NC CTAs owns one channel tile (Cg = 64 channels of one batch
// row, one channel pair per lane) and walks T in rounds of NC segments of
// Ts = NW L steps; CTA rank r takes segment round * NC + r.  Inside a CTA
// each warp owns one chunk of L steps; its rows arrive by their own TMA box
// and mbarrier, so a warp starts as soon as its rows land.  Per round:
//   1. every warp summarises its chunk from the empty state (chunk_phase1
//      with stash: the per-step numerators and denominators of its outputs
//      go to tensor memory);
//   2. once every summary is in, warp 0 joins them into the segment's
//      aggregate and pushes it into the shared memory of every CTA of the
//      cluster by asynchronous DSMEM stores that complete on the receiving
//      CTA's barrier of that exchange's slot;
//   3. once all NC aggregates have landed, warp 1 folds them, from the state
//      carried into the round, into the state at the segment start (into
//      shared memory) and the state carried into the next round;
//   4. after a CTA barrier every warp joins the segment start state with its
//      chunk's prefix (the summaries of the chunks before it) and computes its
//      chunk's outputs from the stash.
// Only warps 0, 1 (and 2) run the scan, the fold (and the chunk prefixes):
// every warp running them would queue on the transcendental and conversion
// pipe they lean on.
// One round (kMulti false): persistent clusters, as many as the GPU holds at
// once, walk the channel tiles tile, tile + G, ...; warp 0 joins the
// summaries as a balanced tree, warp 2 scans the chunk prefixes into their
// own array; a warp's k rows (and warp 0's parameters) of the next tile load
// right after its summary pass, y is staged in its v rows and sent out by one
// TMA store, and the next tile's v rows follow once the store has read them.
// Several rounds (kMulti) are software-pipelined: a warp's rows take the next
// round's load right after its summary pass; round r + 1's steps 1 and 2 run
// before round r's step 4 (warp 0 scans the summaries in place, one chain that
// also gives the aggregate), and warp 1 folds round r + 1 after its step 4 of
// round r, so the aggregates travel while the warps work.  The chunk
// summaries, the stash and the segment start state alternate between two
// slots; y goes straight from registers to global memory.  Aggregates always
// alternate between two slots.  There is no global scratch: all exchange is
// through cluster shared memory.  Every wait is bounded.
#pragma once

#include <cooperative_groups.h>

#include "wkv4_chunk.cuh"

namespace wkv4 {

namespace cg = cooperative_groups;

constexpr int kMaxCluster = 8;  // cluster sizes 1, 2, 4, 8; warps per CTA 4 or 8

// Register cap of the scan kernel: two CTAs of 8 warps per SM, except where
// an 8-warp CTA's tensor memory (nw L columns a stash slot, two slots with
// several rounds) takes more than half of the SM's 512 columns, so one CTA
// per SM is all there is and the cap would only cost spills.
template <int L, bool kMulti>
constexpr int scan_maxnreg() {
    return (kMulti && 2 * 8 * L > 256) ? 255 : 128;
}

// Shared-memory layout for nw warps and clusters of nc (offsets from a
// 128-byte aligned base): one buffer of k and v rows, the chunk summaries,
// the state at the segment start, two aggregate slots, the tile's w, u and
// state, barriers.  kMulti (T walked in several rounds, software-pipelined):
// two slots of the chunk summaries, the stash and the segment start state.
// One round (a cluster walks several channel tiles): two slots of w, u and
// state, so that the next tile's come in while this one's are in use.
template <typename IO, int L, bool kMulti>
struct ScanLayout {
    static constexpr int kCg = 64;  // channels per tile: 32 lanes x 2
    static constexpr int kChunkBytes = L * kCg * (int)sizeof(IO);  // one warp's rows, one tensor
    static constexpr int kAlign = 128;                               // TMA destinations
    static constexpr int kSlots = kMulti ? 2 : 1;       // summaries, stash, start state
    static constexpr int kAggSlots = 2;
    static constexpr int kParamSlots = kMulti ? 1 : 2;
    static_assert(L <= 256 && L % 4 == 0, "TMA box dims, stash column groups");
    static_assert(kChunkBytes % kAlign == 0, "TMA destination alignment");
    int nw, nc;
    __host__ __device__ size_t tile() const { return (size_t)nw * kChunkBytes; }
    __host__ __device__ size_t k() const { return 0; }
    __host__ __device__ size_t v() const { return tile(); }
    __host__ __device__ size_t sums(int slot) const {  // [kSlots][nw][Cg] x 16 B
        return 2 * tile() + (size_t)slot * nw * kCg * 16;
    }
    // one round: the exclusive prefixes of the chunk summaries, [nw][Cg] x 16 B
    // (several rounds scan the summaries in place)
    __host__ __device__ size_t pre() const { return sums(kSlots); }
    __host__ __device__ size_t start(int slot) const {  // [kSlots][Cg] x 16 B
        return pre() + (kMulti ? 0 : (size_t)nw * kCg * 16) + (size_t)slot * kCg * 16;
    }
    __host__ __device__ size_t agg(int slot) const {  // [kAggSlots][nc][Cg] x 16 B
        return start(kSlots) + (size_t)slot * nc * kCg * 16;
    }
    __host__ __device__ size_t params(int slot) const {  // [kParamSlots][5][Cg] f32
        return agg(kAggSlots) + (size_t)slot * 5 * kCg * 4;
    }
    // rows [nw], params [kParamSlots], aggregate slots [kAggSlots], receptance
    // rows [nw] x 8 B
    __host__ __device__ size_t bars() const { return params(kParamSlots); }
    __host__ __device__ size_t tslot() const {
        return bars() + (size_t)(2 * nw + kParamSlots + kAggSlots) * 8;
    }
    // the CTA's failure flag (a bounded wait ran out), beside the tensor-memory base
    __host__ __device__ size_t flag() const { return tslot() + 4; }
    __host__ __device__ size_t bytes() const { return kAlign + tslot() + 8; }
    // tensor-memory columns: 4 a step for each warp and slot, warps w and
    // w + 4 sharing a lane quarter
    __host__ __device__ int tmem_cols() const { return kSlots * nw * L; }
};

struct ScanParams {
    int64_t T, C;
    int CGB;     // channel tiles per batch row
    int tiles;   // B * CGB
    int rounds;  // ceil(segments / NC)
    const float* w;
    const float* u;
    const void* k;
    const void* v;
    const void* r;        // receptance [B][T][C] of the gated forward (kGate), else NULL
    const float* state_in;
    void* y;
    float* state_out;
    int64_t BC;
    int bulk_params;      // w, u, state_in 16-byte aligned and C % 4 == 0: bulk copies
    uint32_t wait_rounds;  // limit of each bounded wait, in rounds of about 1 ms
    int no_push;           // checked builds only: no CTA pushes its aggregate (fault injection)
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

// Stretches q = 0, 1, ... of a round held in shared memory as entries
// q * 64 + col + j of t (the lane's channel pair j = 0, 1), stretch q spanning
// len(q) steps (an empty stretch is the empty state), joined as a balanced
// tree: depth log2 of their count instead of a left-to-right chain (the
// combine is associative, so the result is the same up to rounding).

// Stretches lo .. lo + S - 1 joined (lo warp-uniform): r, spanning n steps.
template <int S, typename Len>
__device__ __forceinline__ void tree_range(const TripleRef& t, int col, int lo, Len len,
                                           const PairConsts& cc, St (&r)[2], int& n) {
    if constexpr (S == 1) {
#pragma unroll
        for (int j = 0; j < 2; ++j) r[j] = t.get(lo * 64 + col + j);
        n = len(lo);
    } else {
        St x[2], y[2];
        int nx, ny;
        tree_range<S / 2>(t, col, lo, len, cc, x, nx);
        tree_range<S / 2>(t, col, lo + S / 2, len, cc, y, ny);
#pragma unroll
        for (int j = 0; j < 2; ++j) r[j] = combine(x[j], y[j], (double)ny * cc.w2[j]);
        n = nx + ny;
    }
}

// Exclusive prefix of the NW chunk summaries of a segment into `out` (entry
// q becomes the state before chunk q; `out` may be `sums` itself) and the
// segment aggregate in acc.  All summaries are read before the chain starts;
// chunk q spans clamp(rem - q L, 0, L) steps.
template <int NW, int L>
__device__ __forceinline__ void scan_chunks(const TripleRef& sums, const TripleRef& out, int col,
                                            int rem, const PairConsts& cc, St (&acc)[2]) {
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
            out.put(q * Cg + col + j, acc[j]);
            acc[j] = combine(acc[j], x[q][j], nq * cc.w2[j]);
        }
    }
}

// Warp 1: fold of the NC segment aggregates of a round into the state at this
// CTA's segment start (P) and the state carried into the next round (carry);
// segment q spans clamp(rrem - q Ts, 0, Ts) steps.
template <int NC>
__device__ __forceinline__ void fold_aggs(const TripleRef& agg, int col, int rank, int64_t rrem,
                                          int Ts, const PairConsts& cc, St (&carry)[2], St (&P)[2]) {
    St y[NC][2];
#pragma unroll
    for (int q = 0; q < NC; ++q)
#pragma unroll
        for (int j = 0; j < 2; ++j) y[q][j] = agg.get(q * 64 + col + j);
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

// kGate: the gated forward, y = sigmoid(r) wkv (the receptance gate of the
// time mix applied in the output pass).  With one round and TMA the warp's r
// rows come by their own TMA box (on their own barrier) into its v rows once
// the summary pass has read them, and y is written over them in place; with
// several rounds or element-wise loads r is read from global memory in the
// output pass (several rounds: the warp's r box is prefetched into L2 at its
// summary pass).
template <typename IO, int L, bool kMulti, bool kTMA, bool kGate>
__global__ void __maxnreg__((scan_maxnreg<L, kMulti>()))
    wkv4_scan_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                     const __grid_constant__ CUtensorMap tmy, const __grid_constant__ CUtensorMap tmr,
                     const ScanParams p) {
    allow_dependents();
    grid_dependency_wait();
    using Lay = ScanLayout<IO, L, kMulti>;
    constexpr int kAS = Lay::kAggSlots;
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
    uint64_t* mbar = reinterpret_cast<uint64_t*>(base + lay.bars());  // rows [NW]
    uint64_t* pbar = mbar + NW;                                       // params [kParamSlots]
    uint64_t* abar = pbar + Lay::kParamSlots;  // [kAS]: the aggregates of a round have landed
    uint64_t* rbar = abar + kAS;               // [NW]: a warp's receptance rows (kGate)
    uint32_t* tslot = reinterpret_cast<uint32_t*>(base + lay.tslot());

    const int rank = (int)cluster.block_rank();
    const int G = (int)(gridDim.x / NC);  // clusters
    int tile = (int)(blockIdx.x / NC);    // this cluster's channel tile (its first, with one round)
    int b = tile / p.CGB;
    int64_t c0 = (int64_t)(tile - b * p.CGB) * Cg;
    const int64_t T = p.T, C = p.C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int col = lane * 2;
    const int64_t seg_stride = (int64_t)NC * Ts;  // steps per round
    const int64_t BTC = p.BC * T, Bn = p.BC / C;  // extents of k, v, y (and r); batch rows
    // a TMA box's start inside its [B][T][C] tensor (checked builds)
    auto box_in = [&](int64_t cc0, int64_t t, int64_t bb) {
        return in_range(cc0, C) && in_range(t, T) && in_range(bb, Bn);
    };
    const IO* kg = static_cast<const IO*>(p.k);
    const IO* vg = static_cast<const IO*>(p.v);
    const IO* rg = static_cast<const IO*>(p.r);
    IO* yg = static_cast<IO*>(p.y);
    // aggregate exchanges this cluster makes: one a round, or one a tile
    const int items = kMulti ? p.rounds : (p.tiles - tile + G - 1) / G;

    auto chunk_len = [&](int j, int q) -> int {  // steps of chunk q of this CTA in round j
        const int64_t tc = (int64_t)j * seg_stride + (int64_t)rank * Ts + (int64_t)q * L;
        return (int)max((int64_t)0, min((int64_t)L, T - tc));
    };
    IO* const kr = reinterpret_cast<IO*>(base + lay.k()) + warp * L * Cg;  // this warp's rows
    IO* const vr = reinterpret_cast<IO*>(base + lay.v()) + warp * L * Cg;
    // Lane 0 of each warp: this warp's rows of round j of the tile at (bb,
    // cc0), k and v (issue_k announces both on the warp's barrier, issue_v may
    // follow later), as the barrier's phase `phase` (the tile with one round,
    // the round with several).  Every round completes one phase of the
    // barrier (a plain arrive where nothing is copied), so its phases stay in
    // step; row_pend records the phase issued and not yet waited for (-1:
    // none; a wait is always for the last phase issued), so that a CTA
    // leaving after an expired wait can let a copy in flight land.
    int row_pend = -1;
    auto issue_k = [&](int j, int bb, int64_t cc0, int phase) {
        if constexpr (kTMA) {
            row_pend = phase;
            uint64_t* bar = mbar + warp;
            const int t = (int)((int64_t)j * seg_stride + (int64_t)rank * Ts + warp * L);
            if (chunk_len(j, warp) > 0 && box_in(cc0, t, bb)) {
                mbar_arrive_expect_tx(bar, 2u * kChunkBytes);
                tma_load_3d(kr, &tmk, (int)cc0, t, bb, bar);
            } else {
                mbar_arrive(bar);
            }
        }
    };
    auto issue_v = [&](int j, int bb, int64_t cc0) {
        if constexpr (kTMA) {
            const int t = (int)((int64_t)j * seg_stride + (int64_t)rank * Ts + warp * L);
            if (chunk_len(j, warp) > 0 && box_in(cc0, t, bb))
                tma_load_3d(vr, &tmv, (int)cc0, t, bb, mbar + warp);
        }
    };
    auto issue_rows = [&](int j, int bb, int64_t cc0, int phase) {
        issue_k(j, bb, cc0, phase);
        issue_v(j, bb, cc0);
    };
    // Lane 0, one round with TMA and the gate: this warp's r rows of the tile
    // at (bb, cc0) into its v rows, as phase `phase` (the tile) of its
    // receptance barrier (a plain arrive where nothing is copied).
    int r_pend = -1;
    auto issue_r = [&](int bb, int64_t cc0, int phase) {
        if constexpr (kTMA && kGate && !kMulti) {
            r_pend = phase;
            const int t = (int)((int64_t)rank * Ts + warp * L);
            if (chunk_len(0, warp) > 0 && box_in(cc0, t, bb)) {
                mbar_arrive_expect_tx(rbar + warp, (uint32_t)kChunkBytes);
                tma_load_3d(vr, &tmr, (int)cc0, t, bb, rbar + warp);
            } else {
                mbar_arrive(rbar + warp);
            }
        }
    };
    // Per-channel w, u and the state of a tile: a full 64-channel slice with
    // aligned pointers comes by bulk copy (lane 0 of warp 0) into a parameter
    // slot, on that slot's barrier; any other tile (read from global memory
    // by take_params) completes the slot's phase by a plain arrive, so that
    // every tile takes exactly one phase of its slot and the waits' parities
    // stay in step with the tiles.  par_pend (lane 0 of warp 0): the tile
    // whose parameters were issued and not yet waited for (-1: none).
    int par_pend = -1;
    auto bulk_ok = [&](int64_t cc0) { return kTMA && p.bulk_params && cc0 + Cg <= C; };
    auto issue_params = [&](int slot, int bb, int64_t cc0, int tile_no) {
        par_pend = tile_no;
        const int64_t ch = (int64_t)bb * C + cc0;
        if (!bulk_ok(cc0) || !(in_range(cc0 + Cg - 1, C) && in_range(ch + Cg - 1, p.BC))) {
            mbar_arrive(pbar + slot);
            return;
        }
        float* sw = reinterpret_cast<float*>(base + lay.params(slot));
        const uint32_t nb = Cg * 4;
        mbar_arrive_expect_tx(pbar + slot, (p.state_in ? 5u : 2u) * nb);
        bulk_load(sw, p.w + cc0, nb, pbar + slot);
        bulk_load(sw + Cg, p.u + cc0, nb, pbar + slot);
        if (p.state_in) {
            bulk_load(sw + 2 * Cg, p.state_in + ch, nb, pbar + slot);
            bulk_load(sw + 3 * Cg, p.state_in + p.BC + ch, nb, pbar + slot);
            bulk_load(sw + 4 * Cg, p.state_in + 2 * p.BC + ch, nb, pbar + slot);
        }
    };

    // every CTA of the cluster pushes 32 B per lane into each aggregate slot;
    // agg_waited (warp 1): the exchanges whose aggregates it has seen land, in
    // order; slots are armed for exchanges agg_waited .. agg_waited + kAS - 1
    // (those below `items`)
    const uint32_t agg_bytes = (uint32_t)NC * 32u * 32u;
    int agg_waited = 0;
    // The CTA's failure flag: set by any thread whose bounded wait ran out.
    // From then on the CTA issues no copy, pushes no aggregate and waits on no
    // barrier (outputs and final state are then undefined, and the device
    // error word says so); before leaving it lets the copies it issued, and
    // the aggregates its slots were armed for, land (bounded waits).
    volatile int* s_fail = reinterpret_cast<volatile int*>(base + lay.flag());
    if (threadIdx.x == 0) {
        *s_fail = 0;
        for (int r = 0; r < kAS; ++r) mbar_init(abar + r, 1);
        fence_mbar_init();
        for (int r = 0; r < kAS && r < items; ++r) mbar_arrive_expect_tx(abar + r, agg_bytes);
    }
    if constexpr (kTMA) {
        if (lane == 0) {
            if (warp == 0) {
                for (int s = 0; s < Lay::kParamSlots; ++s) mbar_init(pbar + s, 1);
                prefetch_tmap(&tmk);
                prefetch_tmap(&tmv);
                prefetch_tmap(&tmy);
                if (kGate) prefetch_tmap(&tmr);
            }
            mbar_init(mbar + warp, 1);
            if (kGate) mbar_init(rbar + warp, 1);
            fence_mbar_init();
            if (warp == 0) issue_params(0, b, c0, 0);
            issue_rows(0, b, c0, 0);
        }
        __syncwarp();
    }
    // tensor memory after the loads are on their way
    if (warp == 0) tmem_alloc(tslot, (uint32_t)lay.tmem_cols());
    // the tensor-memory base is in shared memory, every barrier initialised
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    // the CTAs of the cluster have all started, with their barriers
    // initialised, before the first DSMEM store (this barrier's wait comes
    // just before it)
    cluster_arrive_relaxed();
    const uint32_t tbase = *tslot;
    // this warp's stash in slot s: its lane quarter, NW L columns a slot,
    // 4 L for each warp of the quarter
    auto taddr = [&](int s) -> uint32_t {
        return tbase + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(s * NW * L + (warp >> 2) * 4 * L);
    };
    // this thread has seen the CTA fail: its own wait ran out, or the flag
    // was set when it last passed a CTA barrier (other warps learn of a
    // failure there; until then their copies are tracked and their waits
    // bounded as on the normal path)
    bool failed = false;
    auto cta_failed = [&]() -> bool { return failed; };
    auto sync_fail = [&]() { failed = failed || *s_fail != 0; };
    auto fail = [&](unsigned bit) {
        failed = true;
        *s_fail = 1;
        if (lane == 0) atomicOr(&g_device_error, bit);
    };

    // w, u of the current tile (cc) and the state carried into it (carry;
    // only warp 1 folds it), from parameter slot `slot` (its phase `parity`)
    // or, for a partial or unaligned slice, from global memory
    PairConsts cc;
    St carry[2];
    auto take_params = [&](int slot, uint32_t parity, int tile_no) {
        if (bulk_ok(c0)) {
            if (!cta_failed()) {
                if (mbar_wait_bounded(pbar + slot, parity, p.wait_rounds)) {
                    if (par_pend == tile_no) par_pend = -1;
                } else {
                    fail(kErrTmaWait);
                }
            }
            const float* sw = reinterpret_cast<const float*>(base + lay.params(slot));
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                cc.w[j] = sw[col + j];
                cc.u[j] = sw[Cg + col + j];
                carry[j] = p.state_in ? St{sw[2 * Cg + col + j], sw[3 * Cg + col + j],
                                           (double)sw[4 * Cg + col + j] * kLog2eD}
                                      : empty_state();
            }
        } else {
            pair_wu(p.w, p.u, c0 + col, C, cc);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int64_t c = c0 + col + j, ch = (int64_t)b * C + c;
                carry[j] = (p.state_in && c < C && in_range(ch, p.BC))
                               ? load_state_log2(p.state_in, p.BC, ch)
                               : empty_state();
            }
        }
        pair_derive(cc);
    };
    auto put_state_out = [&]() {
        if (rank == 0 && warp == 1 && p.state_out) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int64_t c = c0 + col + j, ch = (int64_t)b * C + c;
                if (c < C && in_range(ch, p.BC)) store_state_log2(p.state_out, p.BC, ch, carry[j]);
            }
        }
    };

    // ---- 1. summary pass of a round: this warp's chunk summary into its
    //         entry of summary slot round & 1 (kMulti) and its stash into
    //         tensor-memory slot round & 1, once its rows (barrier phase
    //         `parity`) are in
    auto summary = [&](int round, int phase) -> PairRef {
        const int slot = kMulti ? (round & 1) : 0;
        const int n = chunk_len(round, warp);
        const int64_t t0 = (int64_t)round * seg_stride + (int64_t)rank * Ts;  // segment start
        if constexpr (kTMA) {
            if (n > 0 && !cta_failed()) {
                if (mbar_wait_bounded(mbar + warp, (uint32_t)(phase & 1), p.wait_rounds)) {
                    if (row_pend == phase) row_pend = -1;
                } else {
                    fail(kErrTmaWait);
                }
            }
        } else {
            // element-wise loads of this warp's rows (any alignment, zero fill)
            for (int idx = lane; idx < L * Cg; idx += 32) {
                const int rr = idx / Cg, ci = idx - rr * Cg;
                const int64_t t = t0 + warp * L + rr, c = c0 + ci;
                IO kx = Io<IO>::from_f(0.f), vx = Io<IO>::from_f(0.f);
                if (t < T && c < C) {
                    const int64_t off = ((int64_t)b * T + t) * C + c;
                    if (in_range(off, BTC)) {
                        kx = kg[off];
                        vx = vg[off];
                    }
                }
                kr[idx] = kx;
                vr[idx] = vx;
            }
            __syncwarp();
        }
        if constexpr (kTMA && kGate && kMulti) {
            // this chunk's r rows, read by its output pass a round later
            if (lane == 0 && n > 0 && box_in(c0, t0 + warp * L, b))
                tma_prefetch_3d_l2(&tmr, (int)c0, (int)(t0 + warp * L), b);
        }
        PairRef ref;
        St sum[2];
        chunk_phase1<IO, L, true>(ref, kr, vr, Cg, col, n, cc, sum, taddr(slot));
        const TripleRef sums = triples(base + lay.sums(slot), NW * Cg);
#pragma unroll
        for (int j = 0; j < 2; ++j) sums.put(warp * Cg + col + j, sum[j]);
        return ref;
    };

    // ---- 2. warp 0, once every warp's summary of exchange `it` is in: the
    //         segment aggregate (one round: the chunk summaries joined as a
    //         tree; several rounds: with their exclusive prefix, in place, by
    //         one chain) goes by asynchronous DSMEM stores into slot
    //         [it % kAS][rank] of every CTA of the cluster, each store
    //         completing bytes on that CTA's barrier of the slot
    auto scan_push = [&](int round, int it) {
        if (cta_failed()) return;
#ifdef WKV4_CHECKED
        if (p.no_push) return;
#endif
        const TripleRef sums = triples(base + lay.sums(kMulti ? (round & 1) : 0), NW * Cg);
        const TripleRef agg = triples(base + lay.agg(it % kAS), NC * Cg);
        const int64_t t0 = (int64_t)round * seg_stride + (int64_t)rank * Ts;
        // steps of this CTA's segment (the chunks' lengths follow from it)
        const int rem = (int)max((int64_t)0, min((int64_t)Ts, T - t0));
        St acc[2];
        if constexpr (kMulti) {
            if (NW == 8) {
                scan_chunks<8, L>(sums, sums, col, rem, cc, acc);
            } else {
                scan_chunks<4, L>(sums, sums, col, rem, cc, acc);
            }
        } else {
            auto clen = [=](int q) { return max(0, min(L, rem - q * L)); };
            int nacc;
            if (NW == 8) {
                tree_range<8>(sums, col, 0, clen, cc, acc, nacc);
            } else {
                tree_range<4>(sums, col, 0, clen, cc, acc, nacc);
            }
        }
        const int off = rank * Cg + col;
        const uint32_t la = smem_u32(agg.a + off), lb = smem_u32(agg.b + off);
        const uint32_t lp = smem_u32(agg.p + off), lbar = smem_u32(abar + it % kAS);
#pragma unroll 1
        for (int q = 0; q < NC; ++q) {
            const uint32_t rbar = mapa_u32(lbar, (uint32_t)q);
            st_async_v2f32(mapa_u32(la, (uint32_t)q), acc[0].a, acc[1].a, rbar);
            st_async_v2f32(mapa_u32(lb, (uint32_t)q), acc[0].b, acc[1].b, rbar);
            st_async_v2f64(mapa_u32(lp, (uint32_t)q), acc[0].p, acc[1].p, rbar);
        }
    };

    // ---- 3. warp 1, once the aggregates of exchange `it` have landed: the
    //         state at this CTA's segment start (the state carried into the
    //         round joined with the aggregates of the segments before it)
    //         into start slot round & 1, and the state carried into the next
    //         round (joined with all of them)
    auto fold = [&](int round, int it) {
        const int as = it % kAS;
        const int64_t t0 = (int64_t)round * seg_stride + (int64_t)rank * Ts;
        const TripleRef agg = triples(base + lay.agg(as), NC * Cg);
        // The slot's next use is exchange it + 2.  Every CTA pushes it + 2
        // after its CTA barrier that follows its own fold of it + 1, which
        // waited for this CTA's push of it + 1, issued after the barrier
        // that follows this fold: the slot is read before it is overwritten,
        // and re-armed (here) before it is written.  A slot whose wait ran
        // out (or was skipped after a failure) is not re-armed.
        if (!cta_failed()) {
            if (mbar_wait_cluster_bounded(abar + as, (uint32_t)((it / kAS) & 1), p.wait_rounds)) {
                agg_waited = it + 1;
                if (lane == 0 && it + kAS < items) mbar_arrive_expect_tx(abar + as, agg_bytes);
            } else {
                fail(kErrExchangeWait);
            }
        }
        const int64_t rrem = T - (t0 - (int64_t)rank * Ts);  // steps of the round from segment 0 on
        St P[2];
        switch (NC) {
            case 1: fold_aggs<1>(agg, col, rank, rrem, Ts, cc, carry, P); break;
            case 2: fold_aggs<2>(agg, col, rank, rrem, Ts, cc, carry, P); break;
            case 4: fold_aggs<4>(agg, col, rank, rrem, Ts, cc, carry, P); break;
            default: fold_aggs<8>(agg, col, rank, rrem, Ts, cc, carry, P); break;
        }
        const TripleRef st = triples(base + lay.start(kMulti ? (round & 1) : 0), Cg);
#pragma unroll
        for (int j = 0; j < 2; ++j) st.put(col + j, P[j]);
    };

    // ---- several rounds, every warp, once the segment start state and the
    //      chunk prefixes of the round are in place: the state at its chunk
    //      start
    auto chunk_start = [&](int round, St (&S)[2]) {
        const int slot = kMulti ? (round & 1) : 0;
        const TripleRef st = triples(base + lay.start(slot), Cg);
        const TripleRef sums = triples(base + lay.sums(slot), NW * Cg);
#pragma unroll
        for (int j = 0; j < 2; ++j)
            S[j] = combine(st.get(col + j), sums.get(warp * Cg + col + j), (double)(warp * L) * cc.w2[j]);
    };

    // ---- one round, warp 2, once every summary is in: the exclusive prefix
    //      of the chunk summaries (one chain) into the prefix array, while
    //      warp 0 pushes and warp 1 folds
    auto chunk_prefixes = [&]() {
        const TripleRef sums = triples(base + lay.sums(0), NW * Cg);
        const TripleRef pre = triples(base + lay.pre(), NW * Cg);
        const int rem = (int)max((int64_t)0, min((int64_t)Ts, T - (int64_t)rank * Ts));
        St acc[2];
        if (NW == 8) {
            scan_chunks<8, L>(sums, pre, col, rem, cc, acc);
        } else {
            scan_chunks<4, L>(sums, pre, col, rem, cc, acc);
        }
    };

    // ---- 4. every warp: its chunk's outputs from the stash and the state S
    //         at its start.  One round (TMA launch): y is staged in place of v
    //         and sent out by one TMA store.  Several rounds (the rows already
    //         hold the next round's): y goes straight from registers, one
    //         2-channel store a step per lane (C % 4 == 0 with TMA, so a pair
    //         in range is whole and aligned).
    auto emit = [&](int round, const PairRef& ref, const St (&S)[2], int phase) {
        const int slot = kMulti ? (round & 1) : 0;
        const int n = chunk_len(round, warp);
        const int64_t t0 = (int64_t)round * seg_stride + (int64_t)rank * Ts;
        const int64_t cpair = c0 + col;
        const int64_t row0 = ((int64_t)b * T + t0 + warp * L) * C + cpair;  // k, v, y, r offset
        const bool ok0 = cpair < C, ok1 = cpair + 1 < C;
        IO* yrow = yg + row0;
        const IO* rrow = rg + row0;  // kGate only
        // every global access of the output pass is row0 + s C + j, s < n, j <= ok1;
        // a warp with a lane outside skips the pass as a whole (its steps are
        // warp-collective)
#ifdef WKV4_CHECKED
        const bool out_ok = !(ok0 && n > 0) || (in_range(row0, BTC) &&
                                                in_range(row0 + (int64_t)(n - 1) * C + (ok1 ? 1 : 0), BTC));
        if (!__all_sync(0xffffffffu, out_ok)) return;
#endif
        auto out_one = [=](int s, int j, float y) {
            if (j == 0 ? ok0 : ok1) {
                if constexpr (kGate) y = gate_one(y, Io<IO>::to_f(rrow[(int64_t)s * C + j]));
                yrow[(int64_t)s * C + j] = Io<IO>::from_f(y);
            }
        };
        // g = e^{-r} of step s's pair from global memory (a pair whose first
        // channel is in range is whole whenever C % 4 == 0, as with TMA)
        auto gate_global = fn_gate([=](int s) -> f2 {
            const IO* rp = rrow + (int64_t)s * C;
            if (kTMA) return ok0 ? gate_g2(Pair<IO>::load(rp)) : 0ull;
            const float r0 = ok0 ? Io<IO>::to_f(rp[0]) : 0.f, r1 = ok1 ? Io<IO>::to_f(rp[1]) : 0.f;
            return gate_g2(pk(r0, r1));
        });
        if constexpr (kTMA) {
            if constexpr (!kMulti) {
                IO* yr = vr;
                if constexpr (kGate) {
                    // this warp's r rows (receptance barrier, phase `phase`)
                    if (n > 0 && !cta_failed()) {
                        if (mbar_wait_bounded(rbar + warp, (uint32_t)(phase & 1), p.wait_rounds)) {
                            if (r_pend == phase) r_pend = -1;
                        } else {
                            fail(kErrTmaWait);
                        }
                    }
                }
                auto st_one = [=](int s, int j, float y) {
                    if constexpr (kGate) y = gate_one(y, Io<IO>::to_f(yr[s * Cg + col + j]));
                    yr[s * Cg + col + j] = Io<IO>::from_f(y);
                };
                auto st_pair = [=](int s, f2 y) { Pair<IO>::store(yr + s * Cg + col, y); };
                if constexpr (kGate) {
                    auto gate_smem = fn_gate([=](int s) { return gate_g2(Pair<IO>::load(yr + s * Cg + col)); });
                    chunk_phase3_stash<IO, L>(ref, n, S, cc, taddr(slot), kg + row0, vg + row0, C, ok0,
                                              ok1, st_pair, st_one, gate_smem);
                } else {
                    chunk_phase3_stash<IO, L>(ref, n, S, cc, taddr(slot), kg + row0, vg + row0, C, ok0,
                                              ok1, st_pair, st_one);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if (n > 0 && !failed && box_in(c0, t0 + warp * L, b)) {
                        tma_store_3d(&tmy, yr, (int)c0, (int)(t0 + warp * L), b);
                        bulk_commit();
                    }
                }
                __syncwarp();
            } else {
                auto out_pair = [=](int s, f2 y) {
                    if (ok0) Pair<IO>::store(yrow + (int64_t)s * C, y);
                };
                if constexpr (kGate) {
                    chunk_phase3_stash<IO, L>(ref, n, S, cc, taddr(slot), kg + row0, vg + row0, C, ok0,
                                              ok1, out_pair, out_one, gate_global);
                } else {
                    chunk_phase3_stash<IO, L>(ref, n, S, cc, taddr(slot), kg + row0, vg + row0, C, ok0,
                                              ok1, out_pair, out_one);
                }
            }
        } else {
            // element-wise stores (any alignment)
            auto out_pair = [=](int s, f2 y) {
                if (ok0) yrow[(int64_t)s * C] = Io<IO>::from_f(lo(y));
                if (ok1) yrow[(int64_t)s * C + 1] = Io<IO>::from_f(hi(y));
            };
            if constexpr (kGate) {
                chunk_phase3_stash<IO, L>(ref, n, S, cc, taddr(slot), kg + row0, vg + row0, C, ok0, ok1,
                                          out_pair, out_one, gate_global);
            } else {
                chunk_phase3_stash<IO, L>(ref, n, S, cc, taddr(slot), kg + row0, vg + row0, C, ok0, ok1,
                                          out_pair, out_one);
            }
        }
    };

    if constexpr (!kMulti) {
        // One round per tile; the cluster walks tiles tile, tile + G, ...  A
        // warp's k rows of the next tile (and warp 0's parameters of it) are
        // loaded as soon as its summary pass is done, so they land while the
        // aggregates travel and the outputs go out; its v rows once the TMA
        // store of y, staged in them, has read them (a TMA store beats one
        // store a step from registers).  Per tile j (exchange j):
        //   summary -> barrier A -> warp 0 pushes, warp 2 scans the chunk
        //   prefixes, warp 1 folds -> barrier B -> outputs.
        // Slots in use across tiles: parameters and aggregates alternate
        // (j & 1); the summaries, the stash and the start state are rewritten
        // only after barrier B of the tile that read them.
        for (int j = 0; j < items; ++j) {
            const bool more = j + 1 < items;
            take_params(j & 1, (uint32_t)((j >> 1) & 1), j);
            const PairRef ref = summary(0, j);
            const int nt = tile + G, nb = nt / p.CGB;  // the next tile, if `more`
            const int64_t nc0 = (int64_t)(nt - nb * p.CGB) * Cg;
            bool next_rows = false;  // this warp's rows of the next tile are on their way
            if (kTMA && more) {
                __syncwarp();  // every lane has read the rows
                next_rows = __shfl_sync(0xffffffffu, lane == 0 && !cta_failed(), 0);
                if (lane == 0 && next_rows) {
                    if (warp == 0) issue_params((j + 1) & 1, nb, nc0, j + 1);
                    issue_k(0, nb, nc0, j + 1);
                }
            }
            if constexpr (kTMA && kGate) {
                // this tile's r rows into the v rows the summary pass has read
                if (!(kTMA && more)) __syncwarp();
                const bool go = __shfl_sync(0xffffffffu, lane == 0 && !cta_failed(), 0);
                if (lane == 0 && go) issue_r(b, c0, j);
            }
            __syncthreads();  // A: every summary of the tile is in
            sync_fail();
            if (j == 0) cluster_wait();  // every CTA of the cluster has started
            if (warp == 0) scan_push(0, j);
            if (warp == 2) chunk_prefixes();
            if (warp == 1) fold(0, j);
            __syncthreads();  // B: the segment start state and the chunk prefixes are in place
            sync_fail();
            const TripleRef st = triples(base + lay.start(0), Cg);
            const TripleRef pre = triples(base + lay.pre(), NW * Cg);
            St S[2];
#pragma unroll
            for (int q = 0; q < 2; ++q)
                S[q] = combine(st.get(col + q), pre.get(warp * Cg + col + q), (double)(warp * L) * cc.w2[q]);
            emit(0, ref, S, j);
            put_state_out();  // warp 1 (rank 0): the tile's final state, off the exchange's path
            if (kTMA && next_rows) {
                // issued whenever the k rows were, failure or not: the phase
                // announced both
                if (lane == 0) {
                    bulk_wait_read_all();  // the staged y has been read
                    issue_v(0, nb, nc0);
                }
                __syncwarp();
            }
            if (more) {
                tile += G;
                b = tile / p.CGB;
                c0 = (int64_t)(tile - b * p.CGB) * Cg;
            }
        }
        if (kTMA && lane == 0) bulk_wait_read_all();  // staged rows stay valid until read
    } else {
        // Round r + 1's summary pass runs while round r's aggregates are on
        // their way.  One CTA barrier a round (B_r): before it every warp has
        // summarised its chunk of round r + 1, warp 0 has scanned and pushed
        // round r, and warp 1 has folded round r; after it warp 0 scans and
        // pushes round r + 1, every warp emits round r, and warp 1 folds round
        // r + 1, whose aggregates have had a whole output pass to arrive.
        take_params(0, 0, 0);
        PairRef ref_cur = summary(0, 0);
        if (kTMA && p.rounds > 1) {
            __syncwarp();  // every lane has read the rows
            if (lane == 0 && !cta_failed()) issue_rows(1, b, c0, 1);
        }
        __syncthreads();  // every summary of round 0 is in
        sync_fail();
        cluster_wait();   // every CTA of the cluster has started
        if (warp == 0) scan_push(0, 0);
        for (int round = 0; round < p.rounds; ++round) {
            const bool more = round + 1 < p.rounds;
            PairRef ref_next = ref_cur;
            if (more) {
                ref_next = summary(round + 1, round + 1);
                if (kTMA && round + 2 < p.rounds) {
                    __syncwarp();  // every lane has read the rows
                    if (lane == 0 && !cta_failed()) issue_rows(round + 2, b, c0, round + 2);
                }
            }
            if (round == 0 && warp == 1) fold(0, 0);
            __syncthreads();
            sync_fail();
            if (more && warp == 0) scan_push(round + 1, round + 1);
            St S[2];
            chunk_start(round, S);
            emit(round, ref_cur, S, round);
            if (more && warp == 1) fold(round + 1, round + 1);
            ref_cur = ref_next;
        }
        put_state_out();
    }

    // After a failure: let the copies this CTA issued and the aggregates its
    // slots were armed for land before leaving (bounded waits; without a
    // failure nothing is pending here).
    if (kTMA && lane == 0 && row_pend >= 0)
        mbar_wait_bounded(mbar + warp, (uint32_t)(row_pend & 1), p.wait_rounds);
    if (kTMA && kGate && !kMulti && lane == 0 && r_pend >= 0)
        mbar_wait_bounded(rbar + warp, (uint32_t)(r_pend & 1), p.wait_rounds);
    if (kTMA && warp == 0 && lane == 0 && par_pend >= 0)
        mbar_wait_bounded(pbar + (par_pend & 1), (uint32_t)((par_pend >> 1) & 1), p.wait_rounds);
    if (warp == 1 && lane == 0) {
        for (int e = agg_waited; e < agg_waited + kAS && e < items; ++e)
            mbar_wait_cluster_bounded(abar + e % kAS, (uint32_t)((e / kAS) & 1), p.wait_rounds);
    }
    // Every warp's tensor-memory accesses have completed (each load and each
    // store pass ends in its wait); release the columns.  No cluster barrier
    // is needed before leaving: every aggregate pushed into this CTA has
    // landed (its fold waited for it), and peers read only their own memory.
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, (uint32_t)lay.tmem_cols());
}

}  // namespace wkv4
