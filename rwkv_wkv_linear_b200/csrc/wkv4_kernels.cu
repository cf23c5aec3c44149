// RWKV-4 WKV forward and decode kernels for B200 (sm_100a): launchers.
//
// The recurrence (per batch row and channel, decay w, bonus u):
//   wkv_t = (A_t + e^{u+k_t} v_t) / (D_t + e^{u+k_t}),
//   A_{t+1} = e^w A_t + e^{k_t} v_t,  D_{t+1} = e^w D_t + e^{k_t},
// with A, D carried as an fp32 (num, den, max) triple under the max-trick
// ("RWKV in a self-built engine: a second non-attention paradigm (WKV/RNN)",
// Methods table "Precision"; Reproducibility / Provenance "Implementation").
//
// Kernels (one translation unit, so they share the device error word):
//   wkv4_scan_kernel    (wkv4_scan.cuh) chunked scan, time segments chained
//                       through a thread-block cluster; TMA in, TMA out (one
//                       round) or stores from registers (several rounds).
//   wkv4_seq_kernel     (wkv4_seq.cuh) channel-parallel, sequential over T.
//   wkv4_step_kernel, wkv4_decode_kernel (plain or slot-indexed),
//   wkv4_copy_state_kernel  (wkv4_step.cuh) per-step paths.
//   wkv4_token_shift_kernel (wkv4_shift.cuh) the token shift before the
//                       k, v, r projections.
// No tensor cores: nothing here is a dense contraction; the work is bound by
// HBM bandwidth (k, v read once, y written once).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/wkv4.h"
#include "wkv4_device.cuh"
#include "wkv4_internal.h"
#include "wkv4_scan.cuh"
#include "wkv4_seq.cuh"
#include "wkv4_shift.cuh"
#include "wkv4_step.cuh"

namespace wkv4 {

// Sequential kernel configurations <IO, L, NW, NS>: 64 NW channels, NS
// stages of L steps.
#define WKV4_SEQ_F32 float, 16, 2, 4
#define WKV4_SEQ_F16 __half, 16, 4, 4
#define WKV4_SEQ_BF16 __nv_bfloat16, 16, 4, 4

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

template <typename IO, int L, int NW, int NS>
static Geom seq_geom_t() {
    using Sh = SeqShape<IO, L, NW, NS>;
    return {Sh::kCw, L, Sh::kThreads, Sh::kSmem};
}

Geom seq_geom(int dtype) {
    if (dtype == WKV4_F32) return seq_geom_t<WKV4_SEQ_F32>();
    if (dtype == WKV4_F16) return seq_geom_t<WKV4_SEQ_F16>();
    return seq_geom_t<WKV4_SEQ_BF16>();
}

static int env_int(const char* name, int dflt) {
    const char* e = std::getenv(name);
    return e ? std::atoi(e) : dflt;
}

constexpr size_t kMaxSmem = 227 * 1024;
constexpr int kTmemColumns = 512;  // tensor-memory columns per SM
constexpr int kMaxDevices = 64;

// Per-device limits the launch shapes are worked out from, queried once per
// device (the launchers run on every call; attribute queries are not free).
struct DeviceAttrs {
    int smem_per_sm = 233472, smem_reserved = 1024, reg_file = 65536, max_threads = 2048,
        max_blocks = 32, sms = 148;
};

static const DeviceAttrs& device_attrs() {
    static DeviceAttrs attrs[kMaxDevices];
    static std::once_flag once[kMaxDevices];
    static DeviceAttrs fallback;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return fallback;
    }
    std::call_once(once[dev], [dev] {
        DeviceAttrs& a = attrs[dev];
        cudaDeviceGetAttribute(&a.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
        cudaDeviceGetAttribute(&a.smem_reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
        cudaDeviceGetAttribute(&a.reg_file, cudaDevAttrMaxRegistersPerMultiprocessor, dev);
        cudaDeviceGetAttribute(&a.max_threads, cudaDevAttrMaxThreadsPerMultiProcessor, dev);
        cudaDeviceGetAttribute(&a.max_blocks, cudaDevAttrMaxBlocksPerMultiprocessor, dev);
        cudaDeviceGetAttribute(&a.sms, cudaDevAttrMultiProcessorCount, dev);
        cudaGetLastError();
    });
    return attrs[dev];
}

// A launch that may begin while the kernel before it in the stream is
// finishing (programmatic stream serialization): every kernel of the library
// waits for the earlier grid before its first global access.
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Tuning overrides of the scan's launch shape, read from the environment
// once per process: WKV4_SCAN_NW (warps per CTA), WKV4_SCAN_CLUSTER (cluster
// size), WKV4_SCAN_WAVES=1 (one cluster per channel tile with one round).
struct ScanOverrides {
    int nw, nc, waves;
};

// Limit of each bounded device-side wait, in rounds of about 1 ms.  Checked
// builds (WKV4_CHECKED) take WKV4_WAIT_ROUNDS from the environment, so that a
// test can make a wait run out quickly.
static uint32_t wait_rounds() {
#ifdef WKV4_CHECKED
    static const int r = env_int("WKV4_WAIT_ROUNDS", 0);
    if (r > 0) return (uint32_t)r;
#endif
    return kWaitRounds;
}

// Fault injection, in checked builds only (WKV4_CHECKED), read once from
// WKV4_FAULT:
//   launch:N   the N-th kernel launch of the process (1-based) is made with an
//              empty grid, which the runtime rejects (cudaErrorInvalid-
//              Configuration) without running anything: the launch error path
//              of every entry point, with no GPU fault;
//   exchange   no scan CTA pushes its segment aggregate, so every CTA's
//              bounded wait for its peers' aggregates runs out (with a short
//              limit from WKV4_WAIT_ROUNDS): the expiry path of the exchange.
// Production builds compile none of it.
struct FaultPlan {
    long launch_at = 0;  // 0: none
    bool exchange = false;
};

static const FaultPlan& fault_plan() {
    static const FaultPlan plan = [] {
        FaultPlan f;
#ifdef WKV4_CHECKED
        if (const char* e = std::getenv("WKV4_FAULT")) {
            if (std::strncmp(e, "launch:", 7) == 0) f.launch_at = std::atol(e + 7);
            if (std::strcmp(e, "exchange") == 0) f.exchange = true;
        }
#endif
        return f;
    }();
    return plan;
}

// The grid of a launch: `g`, or an empty grid for the launch fault injection
// picks (one count over every launcher of the process).
#ifdef WKV4_CHECKED
static std::atomic<long> g_launches{0};
#endif
template <typename G>
static G launch_grid(G g) {
#ifdef WKV4_CHECKED
    const long at = fault_plan().launch_at;
    if (at > 0 && g_launches.fetch_add(1) + 1 == at) return G(0);
#endif
    return g;
}

static const ScanOverrides& scan_overrides() {
    static const ScanOverrides o{env_int("WKV4_SCAN_NW", 0), env_int("WKV4_SCAN_CLUSTER", 0),
                                 env_int("WKV4_SCAN_WAVES", 0)};
    return o;
}

// Dynamic shared memory to request for a scan CTA of `cta_regs` registers
// (its warps' allocations) that holds `cols` tensor-memory columns.  A CTA
// allocates its columns at its start and holds them to its end, and an
// allocation that cannot be met waits for another CTA's release; so every
// set of scan CTAs an SM can hold at once -- of one call or of concurrent
// calls on other streams, of any dtypes and shapes -- must need at most the
// SM's 512 columns.  It does when each scan CTA takes at least its column
// share (cols / 512) of one resource the SM divides among its CTAs: its
// registers (cta_regs >= reg_file * cols / 512, true of every 8-warp scan at
// the 128-register cap and 256 columns or fewer), else shared memory, whose
// request is then raised to per_sm * cols / 512 (less the per-block
// reservation).  Either way no scan CTA's allocation waits on another's.
static size_t scan_smem_request(size_t bytes, int cols, int cta_regs) {
    const DeviceAttrs& at = device_attrs();
    if ((int64_t)cta_regs * kTmemColumns >= (int64_t)at.reg_file * cols) return bytes;
    const size_t share = ((size_t)at.smem_per_sm * (size_t)cols + kTmemColumns - 1) / kTmemColumns;
    size_t need = share > (size_t)at.smem_reserved ? share - (size_t)at.smem_reserved : 0;
    need = (need + 127) & ~(size_t)127;
    return bytes > need ? bytes : need;
}

// Scan configuration per I/O type: steps per warp chunk (a warp's rows are
// L steps x 64 channels), with one round (L) and with several (LM).  fp32
// takes 16-step chunks in one round (two CTAs of 8 warps an SM) and 32-step
// chunks over several rounds, where the round's exchange and fold are then
// spread over twice the steps (measured on the 65536-step workload: 291
// against 325 us a call).
template <typename IO> struct ScanL {
    static constexpr int L = 32;
    static constexpr int LM = 32;
};
template <> struct ScanL<float> {
    static constexpr int L = 16;
    static constexpr int LM = 32;
};

constexpr int kNwChoices[2] = {8, 4};  // warps per CTA, in order of preference

// Never launched: its occupancy under a given block size and shared-memory
// request stands in for a scan kernel's cluster placement.
__global__ void wkv4_occupancy_stand_in() {}

// Clusters of nc CTAs of nthreads threads the GPU holds at once when every
// SM holds at most bps of them (cached per device).
struct ClusterFit {
    std::atomic<int> n[64][2][4][4];  // [device][warp-count index][log2 nc][bps - 1]
};

static cudaError_t clusters_fit(int nwi, int nc, int bps, int& out) {
    static ClusterFit fit;
    static DeviceFlags attr;
    out = 0;
    if (bps <= 0) return cudaSuccess;
    bps = bps > 4 ? 4 : bps;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    const int lnc = nc == 1 ? 0 : nc == 2 ? 1 : nc == 4 ? 2 : 3;
    std::atomic<int>& slot = fit.n[dev][nwi][lnc][bps - 1];
    int v = slot.load(std::memory_order_acquire);
    if (v == 0) {
        if ((e = ensure_smem_attr(attr, wkv4_occupancy_stand_in, kMaxSmem)) != cudaSuccess) return e;
        const DeviceAttrs& da = device_attrs();
        // the request at which bps, and not bps + 1, CTAs fit on an SM
        size_t req = (size_t)da.smem_per_sm / (size_t)(bps + 1) + 1;
        req = req > (size_t)da.smem_reserved ? req - (size_t)da.smem_reserved : 0;
        if (req > kMaxSmem) req = kMaxSmem;
        cudaLaunchConfig_t cfg;
        std::memset(&cfg, 0, sizeof(cfg));
        cfg.gridDim = dim3((unsigned)nc, 1, 1);
        cfg.blockDim = dim3((unsigned)(32 * kNwChoices[nwi]), 1, 1);
        cfg.dynamicSmemBytes = req;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = (unsigned)nc;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        int n = 0;
        if ((e = cudaOccupancyMaxActiveClusters(&n, wkv4_occupancy_stand_in, &cfg)) != cudaSuccess)
            return e;
        v = n > 0 ? n : -1;
        slot.store(v, std::memory_order_release);
    }
    out = v > 0 ? v : 0;
    return cudaSuccess;
}

// CTAs of one scan instantiation an SM holds, for nw warps and clusters of nc:
// the least of its registers, shared memory (the request, which the tensor
// memory cap may have raised), threads and tensor-memory columns.  Worked out
// here rather than asked of the runtime, whose per-SM occupancy query
// reports one CTA for these kernels where the SM holds two.
// Registers a thread of one scan instantiation uses (queried once per device;
// the dynamic shared-memory limit is raised with it).
template <typename IO, int L, bool kMulti, bool kTMA, bool kGate>
static cudaError_t scan_regs(int& regs) {
    static DeviceFlags attr;
    static std::atomic<int> regs_cache[kMaxDevices];
    auto kern = wkv4_scan_kernel<IO, L, kMulti, kTMA, kGate>;
    cudaError_t e = ensure_smem_attr(attr, kern, kMaxSmem);
    if (e != cudaSuccess) return e;
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    regs = regs_cache[dev].load(std::memory_order_acquire);
    if (regs == 0) {
        cudaFuncAttributes fa;
        if ((e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess) return e;
        regs = fa.numRegs > 0 ? fa.numRegs : 1;
        regs_cache[dev].store(regs, std::memory_order_release);
    }
    return cudaSuccess;
}

static int warp_regs(int regs) { return ((regs * 32 + 255) / 256) * 256; }  // allocated in 256s

template <typename IO, int L, bool kMulti, bool kTMA, bool kGate>
static cudaError_t scan_ctas_per_sm(int nw, int nc, int& bps) {
    bps = 0;
    int regs = 0;
    cudaError_t e = scan_regs<IO, L, kMulti, kTMA, kGate>(regs);
    if (e != cudaSuccess) return e;
    const ScanLayout<IO, L, kMulti> lay{nw, nc};
    const size_t req = scan_smem_request(lay.bytes(), lay.tmem_cols(), warp_regs(regs) * nw);
    if (req > kMaxSmem || lay.tmem_cols() > kTmemColumns) return cudaSuccess;
    const DeviceAttrs& at = device_attrs();
    int n = at.reg_file / (warp_regs(regs) * nw);
    n = std::min(n, (int)((size_t)at.smem_per_sm / (req + (size_t)at.smem_reserved)));
    n = std::min(n, at.max_threads / (32 * nw));
    n = std::min(n, kTmemColumns / lay.tmem_cols());
    n = std::min(n, at.max_blocks);
    bps = n > 0 ? n : 0;
    return cudaSuccess;
}

// Launch shape of the scan: warps per CTA (NW), cluster size (NC), the
// number of clusters and the chunk length.  8 warps per CTA wherever it
// fits.  When T fits in at most 8 segments of L-step chunks, one round with
// NC = segments (rounded up to a power of two), and as many clusters as the
// GPU holds at once (at most one per channel tile), each walking its share
// of the tiles; when T needs several rounds, chunks of LM steps where T still
// spans more than 8 of their segments (else L), and NC is the largest power
// of two whose grid of one cluster per tile still fits in one wave (a second
// wave of CTAs that each walk all of T would be costly).  WKV4_SCAN_NW / WKV4_SCAN_CLUSTER override NW / NC, and
// WKV4_SCAN_WAVES=1 gives one cluster per tile with one round (tuning).
struct ScanShape {
    int nw, nc, rounds;
    int64_t clusters;
    bool long_chunks;  // several rounds with LM-step chunks
};

template <typename IO, int L, int LM, bool kTMA, bool kGate>
static cudaError_t pick_scan_shape(int64_t tiles, int64_t T, ScanShape& out) {
    const int force_nw = scan_overrides().nw, force_nc = scan_overrides().nc;
    cudaError_t e = cudaSuccess;
    for (int i = 0; i < 2; ++i) {
        const int nw = kNwChoices[i];
        if (force_nw && nw != force_nw) continue;
        const int64_t nseg1 = (T + (int64_t)nw * L - 1) / ((int64_t)nw * L);
        const int64_t nsegm = (T + (int64_t)nw * LM - 1) / ((int64_t)nw * LM);
        // several rounds of LM-step chunks where T spans more than a cluster of their segments
        const bool lm = LM != L && nseg1 > kMaxCluster && nsegm > kMaxCluster;
        const int64_t nseg = lm ? nsegm : nseg1;
        auto per_sm = [&](bool multi, int c, int& bps) {
            if (!multi) return scan_ctas_per_sm<IO, L, false, kTMA, kGate>(nw, c, bps);
            return lm ? scan_ctas_per_sm<IO, LM, true, kTMA, kGate>(nw, c, bps)
                      : scan_ctas_per_sm<IO, L, true, kTMA, kGate>(nw, c, bps);
        };
        int nc = 1;
        if (force_nc == 1 || force_nc == 2 || force_nc == 4 || force_nc == 8) {
            nc = force_nc;
        } else if (nseg <= kMaxCluster) {
            while (nc < nseg) nc *= 2;
        } else {
            for (int c = kMaxCluster; c > 1; c /= 2) {
                int bps = 0, fit = 0;
                if ((e = per_sm(true, c, bps)) != cudaSuccess) return e;
                if ((e = clusters_fit(i, c, bps, fit)) != cudaSuccess) return e;
                if ((int64_t)fit >= tiles) {
                    nc = c;
                    break;
                }
            }
        }
        const int64_t rounds = (nseg + nc - 1) / nc;
        if (rounds > (1ll << 30)) continue;
        if (lm && rounds < 2) continue;  // (a forced cluster size that covers T: not this shape)
        int bps = 0;
        if ((e = per_sm(rounds > 1, nc, bps)) != cudaSuccess) return e;
        if (bps <= 0) continue;  // does not fit on an SM
        int64_t clusters = tiles;
        if (rounds == 1 && !scan_overrides().waves) {
            int fit = 0;
            if ((e = clusters_fit(i, nc, bps, fit)) != cudaSuccess) return e;
            if (fit > 0 && fit < tiles) clusters = fit;
        }
        out = {nw, nc, (int)rounds, clusters, lm};
        return cudaSuccess;
    }
    return cudaErrorInvalidConfiguration;
}

template <typename IO, int L, bool kMulti, bool kTMA, bool kGate>
static cudaError_t launch_scan_nb(const FwdArgs& a, const ScanParams& p, const ScanShape& sh,
                                  EncodeFn encode) {
    CUtensorMap tk, tv, ty, tr;
    std::memset(&tk, 0, sizeof(tk));
    std::memset(&tv, 0, sizeof(tv));
    std::memset(&ty, 0, sizeof(ty));
    std::memset(&tr, 0, sizeof(tr));
    if (kTMA) {
        if (!encode(&tk, a.k, a.dtype, a.B, a.T, a.C, 64, L) ||
            !encode(&tv, a.v, a.dtype, a.B, a.T, a.C, 64, L) ||
            !encode(&ty, a.y, a.dtype, a.B, a.T, a.C, 64, L) ||
            (kGate && !encode(&tr, a.r, a.dtype, a.B, a.T, a.C, 64, L)))
            return cudaErrorInvalidValue;
    }
    auto kern = wkv4_scan_kernel<IO, L, kMulti, kTMA, kGate>;
    const ScanLayout<IO, L, kMulti> lay{sh.nw, sh.nc};
    int regs = 0;
    cudaError_t e = scan_regs<IO, L, kMulti, kTMA, kGate>(regs);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(launch_grid((unsigned)(sh.clusters * sh.nc)), 1, 1);
    cfg.blockDim = dim3(32 * sh.nw, 1, 1);
    cfg.dynamicSmemBytes = scan_smem_request(lay.bytes(), lay.tmem_cols(), warp_regs(regs) * sh.nw);
    cfg.stream = a.stream;
    cudaLaunchAttribute attrs[2];
    attrs[0].id = cudaLaunchAttributeClusterDimension;
    attrs[0].val.clusterDim.x = (unsigned)sh.nc;
    attrs[0].val.clusterDim.y = 1;
    attrs[0].val.clusterDim.z = 1;
    attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, tk, tv, ty, tr, p);
}

template <typename IO, bool kTMA, bool kGate>
static cudaError_t launch_scan_t(const FwdArgs& a, EncodeFn encode) {
    constexpr int L = ScanL<IO>::L, LM = ScanL<IO>::LM;
    ScanParams p{};
    p.T = a.T;
    p.C = a.C;
    p.CGB = (int)((a.C + 63) / 64);
    p.w = a.w;
    p.u = a.u;
    p.k = a.k;
    p.v = a.v;
    p.r = a.r;
    p.state_in = a.state_in;
    p.y = a.y;
    p.state_out = a.state_out;
    p.BC = a.B * a.C;
    p.wait_rounds = wait_rounds();
    p.no_push = fault_plan().exchange ? 1 : 0;
    p.bulk_params = ((uintptr_t)a.w % 16 == 0) && ((uintptr_t)a.u % 16 == 0) &&
                    ((uintptr_t)a.state_in % 16 == 0) && (a.C % 4 == 0);
    const int64_t tiles = a.B * p.CGB;
    if (tiles > (1ll << 30)) return cudaErrorInvalidConfiguration;
    ScanShape sh;
    cudaError_t e = pick_scan_shape<IO, L, LM, kTMA, kGate>(tiles, a.T, sh);
    if (e != cudaSuccess) return e;
    if (sh.clusters * sh.nc > (int64_t)INT32_MAX) return cudaErrorInvalidConfiguration;
    p.tiles = (int)tiles;
    p.rounds = sh.rounds;
    if (sh.rounds == 1) return launch_scan_nb<IO, L, false, kTMA, kGate>(a, p, sh, encode);
    if constexpr (LM != L) {
        if (sh.long_chunks) return launch_scan_nb<IO, LM, true, kTMA, kGate>(a, p, sh, encode);
    }
    return launch_scan_nb<IO, L, true, kTMA, kGate>(a, p, sh, encode);
}

template <typename IO>
static cudaError_t launch_scan_io(const FwdArgs& a, bool tma, EncodeFn encode) {
    if (a.r) return tma ? launch_scan_t<IO, true, true>(a, encode) : launch_scan_t<IO, false, true>(a, encode);
    return tma ? launch_scan_t<IO, true, false>(a, encode) : launch_scan_t<IO, false, false>(a, encode);
}

cudaError_t launch_scan(const FwdArgs& a, bool tma, EncodeFn encode) {
    switch (a.dtype) {
        case WKV4_F32: return launch_scan_io<float>(a, tma, encode);
        case WKV4_F16: return launch_scan_io<__half>(a, tma, encode);
        default: return launch_scan_io<__nv_bfloat16>(a, tma, encode);
    }
}

template <typename IO, int L, int NW, int NS, bool kGate>
static cudaError_t launch_seq_g(const FwdArgs& a, const CUtensorMap* tk, const CUtensorMap* tv,
                                const CUtensorMap* tr) {
    using Sh = SeqShape<IO, L, NW, NS>;
    auto kern = wkv4_seq_kernel<IO, L, NW, NS, kGate>;
    static DeviceFlags attr;
    cudaError_t e = ensure_smem_attr(attr, kern, Sh::kSmem);
    if (e != cudaSuccess) return e;
    SeqParams p{};
    p.T = a.T;
    p.C = a.C;
    p.CGB = (int)((a.C + Sh::kCw - 1) / Sh::kCw);
    p.w = a.w;
    p.u = a.u;
    p.r = a.r;
    p.state_in = a.state_in;
    p.y = a.y;
    p.state_out = a.state_out;
    p.BC = a.B * a.C;
    p.wait_rounds = wait_rounds();
    const int64_t grid = a.B * p.CGB;
    e = launch_pdl(kern, dim3(launch_grid((unsigned)grid)), dim3(Sh::kThreads), Sh::kSmem, a.stream, *tk, *tv,
                   *tr, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <typename IO, int L, int NW, int NS>
static cudaError_t launch_seq_t(const FwdArgs& a, const CUtensorMap* tk, const CUtensorMap* tv,
                                const CUtensorMap* tr) {
    return a.r ? launch_seq_g<IO, L, NW, NS, true>(a, tk, tv, tr)
               : launch_seq_g<IO, L, NW, NS, false>(a, tk, tv, tk);
}

cudaError_t launch_seq(const FwdArgs& a, const CUtensorMap* tk, const CUtensorMap* tv,
                       const CUtensorMap* tr) {
    switch (a.dtype) {
        case WKV4_F32: return launch_seq_t<WKV4_SEQ_F32>(a, tk, tv, tr);
        case WKV4_F16: return launch_seq_t<WKV4_SEQ_F16>(a, tk, tv, tr);
        default: return launch_seq_t<WKV4_SEQ_BF16>(a, tk, tv, tr);
    }
}

static StepParams step_params(const FwdArgs& a) {
    StepParams p{};
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
    p.r = a.r;
    return p;
}

template <typename IO>
static void launch_step_io(const FwdArgs& a, const StepParams& p, unsigned grid) {
    const dim3 g(launch_grid(grid));
    if (a.r)
        launch_pdl(wkv4_step_kernel<IO, true>, g, dim3(256), 0, a.stream, p);
    else
        launch_pdl(wkv4_step_kernel<IO, false>, g, dim3(256), 0, a.stream, p);
}

cudaError_t launch_step(const FwdArgs& a) {
    const StepParams p = step_params(a);
    const int64_t BC = a.B * a.C;
    const unsigned grid = (unsigned)((BC + 255) / 256);
    switch (a.dtype) {
        case WKV4_F32: launch_step_io<float>(a, p, grid); break;
        case WKV4_F16: launch_step_io<__half>(a, p, grid); break;
        default: launch_step_io<__nv_bfloat16>(a, p, grid); break;
    }
    return cudaGetLastError();
}

static bool aligned(const void* ptr, size_t bytes) {
    return ptr == nullptr || ((uintptr_t)ptr % bytes) == 0;
}

// (kSlots: the slot-indexed decode, which has no gate)
template <typename IO, int V, bool kSlots = false>
static void launch_decode_io(const FwdArgs& a, const StepParams& p, unsigned grid) {
    const dim3 g(launch_grid(grid));
    if (kSlots)
        launch_pdl(wkv4_decode_kernel<IO, V, true>, g, dim3(256), 0, a.stream, p);
    else if (a.r)
        launch_pdl(wkv4_decode_kernel<IO, V, false, true>, g, dim3(256), 0, a.stream, p);
    else
        launch_pdl(wkv4_decode_kernel<IO, V, false, false>, g, dim3(256), 0, a.stream, p);
}

cudaError_t launch_decode(const FwdArgs& a) {
    constexpr int V = 4;
    const size_t es = dtype_size(a.dtype);
    const bool vec = (a.C % V == 0) && aligned(a.k, V * es) && aligned(a.v, V * es) &&
                     aligned(a.r, V * es) && aligned(a.y, V * es) && aligned(a.w, 16) &&
                     aligned(a.u, 16) && aligned(a.state_in, 16) && aligned(a.state_out, 16);
    if (!vec) return launch_step(a);
    const StepParams p = step_params(a);
    const int64_t threads = a.B * a.C / V;
    const unsigned grid = (unsigned)((threads + 255) / 256);
    switch (a.dtype) {
        case WKV4_F32: launch_decode_io<float, V>(a, p, grid); break;
        case WKV4_F16: launch_decode_io<__half, V>(a, p, grid); break;
        default: launch_decode_io<__nv_bfloat16, V>(a, p, grid); break;
    }
    return cudaGetLastError();
}

cudaError_t launch_decode_slots(const FwdArgs& a, const int32_t* slots, int64_t S) {
    constexpr int V = 4;
    const size_t es = dtype_size(a.dtype);
    const bool vec = (a.C % V == 0) && aligned(a.k, V * es) && aligned(a.v, V * es) &&
                     aligned(a.y, V * es) && aligned(a.w, 16) && aligned(a.u, 16) &&
                     aligned(a.state_in, 16);
    StepParams p = step_params(a);
    p.slots = slots;
    p.S = S;
    const int64_t threads = vec ? a.B * a.C / V : a.B * a.C;
    const unsigned grid = (unsigned)((threads + 255) / 256);
    if (vec) {
        switch (a.dtype) {
            case WKV4_F32: launch_decode_io<float, V, true>(a, p, grid); break;
            case WKV4_F16: launch_decode_io<__half, V, true>(a, p, grid); break;
            default: launch_decode_io<__nv_bfloat16, V, true>(a, p, grid); break;
        }
    } else {
        switch (a.dtype) {
            case WKV4_F32: launch_decode_io<float, 1, true>(a, p, grid); break;
            case WKV4_F16: launch_decode_io<__half, 1, true>(a, p, grid); break;
            default: launch_decode_io<__nv_bfloat16, 1, true>(a, p, grid); break;
        }
    }
    return cudaGetLastError();
}

// CTAs of one token-shift instantiation an SM holds (the runtime's occupancy
// query, once per device).
template <typename IO, int V>
static int shift_ctas_per_sm() {
    static std::atomic<int> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return 1;
    }
    int n = cache[dev].load(std::memory_order_acquire);
    if (n == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, wkv4_token_shift_kernel<IO, V>,
                                                          kShiftThreads, 0) != cudaSuccess || n < 1) {
            cudaGetLastError();
            n = 1;
        }
        cache[dev].store(n, std::memory_order_release);
    }
    return n;
}

template <typename IO, int V>
static void launch_shift_t(ShiftParams& p, int64_t groups, cudaStream_t stream) {
    // one wave: runs = the CTAs the GPU holds over the CTAs a step range
    // needs (channel blocks x batch rows), at least kShiftMinRun steps a run
    // and at most 65535 runs
    const int64_t xb = (groups + kShiftThreads - 1) / kShiftThreads;
    const int64_t slots = (int64_t)device_attrs().sms * shift_ctas_per_sm<IO, V>();
    const int64_t runs = std::max<int64_t>(1, slots / std::max<int64_t>(1, xb * p.B));
    int64_t run = std::max<int64_t>((p.T + runs - 1) / runs, kShiftMinRun);
    run = std::max<int64_t>(run, (p.T + 65534) / 65535);
    p.run = run;
    const dim3 grid((unsigned)xb, (unsigned)((p.T + run - 1) / run), (unsigned)p.B);
    launch_pdl(wkv4_token_shift_kernel<IO, V>, launch_grid(grid), dim3(kShiftThreads), 0, stream, p);
}

cudaError_t launch_token_shift(const ShiftArgs& a) {
    ShiftParams p{};
    p.B = a.B;
    p.T = a.T;
    p.C = a.C;
    p.x = a.x;
    p.x_prev = a.x_prev;
    for (int i = 0; i < 3; ++i) {
        p.mix[i] = a.mix[i];
        p.out[i] = a.out[i];
    }
    p.x_last = a.x_last;
    const size_t es = dtype_size(a.dtype);
    const int V = (int)(16 / es);  // 16 bytes a thread
    bool vec = a.C % V == 0 && aligned(a.x, 16) && aligned(a.x_prev, 16) && aligned(a.x_last, 16);
    for (int i = 0; i < 3; ++i) vec = vec && aligned(a.mix[i], 16) && aligned(a.out[i], 16);
    const int64_t groups = (a.C + (vec ? V : 1) - 1) / (vec ? V : 1);
    if (vec) {
        switch (a.dtype) {
            case WKV4_F32: launch_shift_t<float, 4>(p, groups, a.stream); break;
            case WKV4_F16: launch_shift_t<__half, 8>(p, groups, a.stream); break;
            default: launch_shift_t<__nv_bfloat16, 8>(p, groups, a.stream); break;
        }
    } else {
        switch (a.dtype) {
            case WKV4_F32: launch_shift_t<float, 1>(p, groups, a.stream); break;
            case WKV4_F16: launch_shift_t<__half, 1>(p, groups, a.stream); break;
            default: launch_shift_t<__nv_bfloat16, 1>(p, groups, a.stream); break;
        }
    }
    return cudaGetLastError();
}

cudaError_t launch_copy_state(const FwdArgs& a) {
    const int64_t BC = a.B * a.C;
    if (!a.state_out || BC == 0) return cudaSuccess;
    const dim3 grid(launch_grid((unsigned)((BC + 255) / 256)));
    launch_pdl(wkv4_copy_state_kernel, grid, dim3(256), 0, a.stream, a.state_in, a.state_out, BC);
    return cudaGetLastError();
}

cudaError_t launch_state_combine(int64_t B, int64_t C, const float* w, int64_t n, const float* x,
                                 const float* y, float* out, cudaStream_t stream) {
    const int64_t BC = B * C;
    const dim3 grid(launch_grid((unsigned)((BC + 255) / 256)));
    launch_pdl(wkv4_state_combine_kernel, grid, dim3(256), 0, stream, w, n, x, y, out, B, C);
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
