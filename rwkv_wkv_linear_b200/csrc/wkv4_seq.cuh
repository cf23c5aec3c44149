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

template <typename IO, int L, int NW, int NS>
__global__ void __launch_bounds__(32 * NW)
    wkv4_seq_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                    const SeqParams p) {
    using Sh = SeqShape<IO, L, NW, NS>;
    constexpr int Cw = Sh::kCw;
    extern __shared__ unsigned char smem_raw[];
    // align by offsetting the shared array itself (a round trip through an
    // integer would lose the address space and turn every access generic)
    unsigned char* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    IO* sk = reinterpret_cast<IO*>(base);                         // [NS][L][Cw]
    IO* sv = reinterpret_cast<IO*>(base + NS * Sh::kStageBytes);  // [NS][L][Cw]
    uint64_t* mbar = reinterpret_cast<uint64_t*>(base + 2 * NS * Sh::kStageBytes);

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
        S[j] = (p.state_in && c + j < C) ? load_state_log2(p.state_in, p.BC, (int64_t)b * C + c + j)
                                         : empty_state();
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
    pair_derive(cc);
    IO* yg = static_cast<IO*>(p.y);
    const bool pair_ok = c + 2 <= C;
    bool failed = false;

    for (int64_t q = 0; q < nchunks; ++q) {
        const int st = (int)(q % NS);
        const uint32_t parity = (uint32_t)((q / NS) & 1);
        if (!failed && !mbar_wait_bounded(mbar + st, parity)) {
            failed = true;
            atomicOr(&g_device_error, kErrTmaWait);
        }
        const int64_t tq = q * L;
        const int n = (int)min((int64_t)L, T - tq);
        const IO* kr = sk + st * L * Cw;
        const IO* vr = sv + st * L * Cw;
        PairRef r;
        St sum[2];
        const int64_t ybase = ((int64_t)b * T + tq) * C + c;
        auto out_one = [&](int i, int j, float y) {
            if (c + j < C) yg[ybase + (int64_t)i * C + j] = Io<IO>::from_f(y);
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
        chunk_phase3<IO, L>(r, kr, vr, Cw, col, n, S, cc, out_pair, out_one);
#pragma unroll
        for (int j = 0; j < 2; ++j) S[j] = combine(S[j], sum[j], (double)n * cc.w2[j]);
        __syncthreads();  // stage st fully consumed
        if (threadIdx.x == 0 && q + NS < nchunks) {
            mbar_arrive_expect_tx(mbar + st, 2u * Sh::kStageBytes);
            tma_load_3d(sk + st * L * Cw, &tmk, (int)c0, (int)((q + NS) * L), b, mbar + st);
            tma_load_3d(sv + st * L * Cw, &tmv, (int)c0, (int)((q + NS) * L), b, mbar + st);
        }
    }
    if (p.state_out) {
#pragma unroll
        for (int j = 0; j < 2; ++j)
            if (c + j < C) store_state_log2(p.state_out, p.BC, (int64_t)b * C + c + j, S[j]);
    }
}

}  // namespace wkv4
