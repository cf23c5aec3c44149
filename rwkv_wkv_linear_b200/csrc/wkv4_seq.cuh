// Channel-parallel kernel, sequential over T.
//
// Each thread owns a channel pair and walks its whole sequence chunk by chunk
// (chunk_phase1 -> outputs from the carried state -> carried state combined
// with the chunk summary).  The CTA's Cw = 64 NW channels are staged through
// an NS-deep ring of TMA time tiles [L steps x Cw channels] with one mbarrier
// per stage; y leaves with pair stores straight from registers.  Suited to shapes with many channels (B C large), where channel
// parallelism alone fills the GPU and no cross-CTA exchange is needed.
#pragma once

#include "wkv4_chunk.cuh"

namespace wkv4 {

template <typename IO, int L, int NW, int NS>
struct SeqShape {
    static constexpr int kCw = 64 * NW;  // channels per CTA
    static constexpr int kThreads = 32 * NW;
    static constexpr int kStageBytes = L * kCw * (int)sizeof(IO);  // one tensor, one stage
    static constexpr size_t kSmem = 1024 + 2 * (size_t)NS * kStageBytes + NS * 8 + 8;
    static_assert(kCw <= 256 && L <= 256, "TMA box dims");
};

struct SeqParams {
    int64_t T, C;
    int CGB;  // channel groups per batch row
    const float* w;
    const float* u;
    const void* r;  // receptance [B][T][C] of the gated forward (kGate), else NULL
    const float* state_in;
    void* y;
    float* state_out;
    int64_t BC;
    uint32_t wait_rounds;  // limit of each bounded wait, in rounds of about 1 ms
};

// kGate: y = sigmoid(r) wkv, r read from global memory in the output pass
// (each chunk's r box is prefetched into L2 when its k, v stage is loaded).
template <typename IO, int L, int NW, int NS, bool kGate>
__global__ void __launch_bounds__(32 * NW)
    wkv4_seq_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                    const __grid_constant__ CUtensorMap tmr, const SeqParams p) {
    allow_dependents();
    grid_dependency_wait();
    using Sh = SeqShape<IO, L, NW, NS>;
    constexpr int Cw = Sh::kCw;
    extern __shared__ unsigned char smem_raw[];
    // align by offsetting the shared array itself (a round trip through an
    // integer would lose the address space and turn every access generic)
    unsigned char* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    IO* sk = reinterpret_cast<IO*>(base);                         // [NS][L][Cw]
    IO* sv = reinterpret_cast<IO*>(base + NS * Sh::kStageBytes);  // [NS][L][Cw]
    uint64_t* mbar = reinterpret_cast<uint64_t*>(base + 2 * NS * Sh::kStageBytes);
    // the CTA's failure flag: once a bounded wait ran out no stage is loaded
    // again and no thread waits again; thread 0 lets the loads in flight land
    // before the CTA leaves
    volatile int* s_fail = reinterpret_cast<volatile int*>(mbar + NS);

    const int b = blockIdx.x / p.CGB;
    const int64_t c0 = (int64_t)(blockIdx.x - b * p.CGB) * Cw;
    const int64_t T = p.T, C = p.C;
    const int col = threadIdx.x * 2;
    const int64_t c = c0 + col;
    const int64_t nchunks = (T + L - 1) / L;

    // small per-channel loads first, so they do not queue behind the tiles
    PairConsts cc;
    pair_wu(p.w, p.u, c, C, cc);
    St S[2];
#pragma unroll
    for (int j = 0; j < 2; ++j)
        S[j] = (p.state_in && c + j < C && in_range((int64_t)b * C + c + j, p.BC))
                   ? load_state_log2(p.state_in, p.BC, (int64_t)b * C + c + j)
                   : empty_state();
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
        if (kGate) prefetch_tmap(&tmr);
        for (int st = 0; st < NS; ++st) mbar_init(mbar + st, 1);
        fence_mbar_init();
        *s_fail = 0;
    }
    __syncthreads();
    int64_t q_issued = -1, q_done = -1;  // thread 0: last chunk loaded / waited for
    if (threadIdx.x == 0) {
        // (checked builds: the boxes' starts inside the tensors; the copy engine
        // clips the boxes themselves)
        in_range(c0, C), in_range(b, p.BC / C);
        for (int st = 0; st < NS && st < nchunks; ++st) {
            q_issued = st;
            if (kGate) tma_prefetch_3d_l2(&tmr, (int)c0, st * L, b);
            mbar_arrive_expect_tx(mbar + st, 2u * Sh::kStageBytes);
            tma_load_3d(sk + st * L * Cw, &tmk, (int)c0, st * L, b, mbar + st);
            tma_load_3d(sv + st * L * Cw, &tmv, (int)c0, st * L, b, mbar + st);
        }
    }
    pair_derive(cc);
    IO* yg = static_cast<IO*>(p.y);
    const IO* rg = static_cast<const IO*>(p.r);
    const bool pair_ok = c + 2 <= C;
    bool failed = false;

    for (int64_t q = 0; q < nchunks; ++q) {
        const int st = (int)(q % NS);
        const uint32_t parity = (uint32_t)((q / NS) & 1);
        if (!failed && *s_fail != 0) failed = true;
        if (!failed) {
            if (mbar_wait_bounded(mbar + st, parity, p.wait_rounds)) {
                q_done = q;
            } else {
                failed = true;
                *s_fail = 1;
                atomicOr(&g_device_error, kErrTmaWait);
            }
        }
        const int64_t tq = q * L;
        const int n = (int)min((int64_t)L, T - tq);
        const IO* kr = sk + st * L * Cw;
        const IO* vr = sv + st * L * Cw;
        PairRef r;
        St sum[2];
        const int64_t ybase = ((int64_t)b * T + tq) * C + c;
        // every output access of the chunk is ybase + i C + j, i < n (checked builds)
        const bool out_ok = !(c < C) || (in_range(ybase, p.BC * T) &&
                                         in_range(ybase + (int64_t)(n - 1) * C + (pair_ok ? 1 : 0),
                                                  p.BC * T));
        auto out_one = [&](int i, int j, float y) {
            if (c + j < C) {
                if constexpr (kGate) y = gate_one(y, Io<IO>::to_f(rg[ybase + (int64_t)i * C + j]));
                yg[ybase + (int64_t)i * C + j] = Io<IO>::from_f(y);
            }
        };
        auto out_pair = [&](int i, f2 y) {
            if (pair_ok) {
                Pair<IO>::store(yg + ybase + (int64_t)i * C, y);
            } else {
                out_one(i, 0, lo(y));
                out_one(i, 1, hi(y));
            }
        };
        chunk_phase1<IO, L>(r, kr, vr, Cw, col, n, cc, sum);
        if (!out_ok) {
        } else if constexpr (kGate) {
            auto gate = fn_gate([&](int i) -> f2 {
                const IO* rp = rg + ybase + (int64_t)i * C;
                if (pair_ok) return gate_g2(Pair<IO>::load(rp));
                const float r0 = c < C ? Io<IO>::to_f(rp[0]) : 0.f;
                const float r1 = c + 1 < C ? Io<IO>::to_f(rp[1]) : 0.f;
                return gate_g2(pk(r0, r1));
            });
            chunk_phase3<IO, L>(r, kr, vr, Cw, col, n, S, cc, out_pair, out_one, gate);
        } else {
            chunk_phase3<IO, L>(r, kr, vr, Cw, col, n, S, cc, out_pair, out_one);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) S[j] = combine(S[j], sum[j], (double)n * cc.w2[j]);
        __syncthreads();  // stage st fully consumed
        if (threadIdx.x == 0 && q + NS < nchunks && *s_fail == 0) {
            q_issued = q + NS;
            if (kGate) tma_prefetch_3d_l2(&tmr, (int)c0, (int)((q + NS) * L), b);
            mbar_arrive_expect_tx(mbar + st, 2u * Sh::kStageBytes);
            tma_load_3d(sk + st * L * Cw, &tmk, (int)c0, (int)((q + NS) * L), b, mbar + st);
            tma_load_3d(sv + st * L * Cw, &tmv, (int)c0, (int)((q + NS) * L), b, mbar + st);
        }
    }
    if (p.state_out) {
#pragma unroll
        for (int j = 0; j < 2; ++j)
            if (c + j < C && in_range((int64_t)b * C + c + j, p.BC))
                store_state_log2(p.state_out, p.BC, (int64_t)b * C + c + j, S[j]);
    }
    // after a failure: the loads still in flight land before the CTA leaves
    if (threadIdx.x == 0)
        for (int64_t q = q_done + 1; q <= q_issued; ++q)
            mbar_wait_bounded(mbar + (int)(q % NS), (uint32_t)((q / NS) & 1), p.wait_rounds);
}

}  // namespace wkv4
