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
//   wkv4_scan_kernel    (wkv4_scan.cuh) chunked scan, tiles chained through
//                       a thread-block cluster; TMA in, TMA out.
//   wkv4_seq_kernel     (wkv4_seq.cuh) channel-parallel, sequential over T.
//   wkv4_step_kernel, wkv4_decode_kernel, wkv4_copy_state_kernel
//                       (wkv4_step.cuh) per-step paths.
// No tensor cores: nothing here is a dense contraction; the work is bound by
// HBM bandwidth (k, v read once, y written once).
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdlib>
#include <cstring>

#include "../../include/wkv4.h"
#include "wkv4_device.cuh"

namespace wkv4 {
__device__ unsigned int g_device_error = 0;
}

#include "wkv4_internal.h"
#include "wkv4_scan.cuh"
#include "wkv4_seq.cuh"
#include "wkv4_step.cuh"

namespace wkv4 {

// Kernel configurations: <IO, V, L, NW> for the scan (tile 32V channels x
// L*NW steps), <IO, V, L, NW, NS> for the sequential kernel.
#define WKV4_SCAN_F32 float, 1, 32, 4
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
    using Sh = ScanShape<IO, V, L, NW, 1>;
    return {Sh::kCg, L, Sh::kThreads, Sh::kSmem};
}
template <typename IO, int V, int L, int NW, int NS>
static Geom seq_geom_t() {
    using Sh = SeqShape<IO, V, L, NW, NS>;
    return {Sh::kCw, L, Sh::kThreads, Sh::kSmem};
}

// Alternative fp16 tile shapes, selected with WKV4_SCAN_CFG=1..3 (tuning).
#define WKV4_SCAN_F16_1 __half, 1, 16, 8
#define WKV4_SCAN_F16_2 __half, 1, 32, 4
#define WKV4_SCAN_F16_3 __half, 2, 8, 8

static int scan_cfg() {
    static const int cfg = [] {
        const char* env = std::getenv("WKV4_SCAN_CFG");
        const int v = env ? std::atoi(env) : 0;
        return (v >= 0 && v <= 3) ? v : 0;
    }();
    return cfg;
}

// TMA boxes: scan boxes are one warp's rows (box_t = L); seq boxes one stage.
Geom scan_geom(int dtype) {
    if (dtype == WKV4_F32) return scan_geom_t<WKV4_SCAN_F32>();
    if (dtype == WKV4_F16) {
        switch (scan_cfg()) {
            case 1: return scan_geom_t<WKV4_SCAN_F16_1>();
            case 2: return scan_geom_t<WKV4_SCAN_F16_2>();
            case 3: return scan_geom_t<WKV4_SCAN_F16_3>();
            default: return scan_geom_t<WKV4_SCAN_F16>();
        }
    }
    return scan_geom_t<WKV4_SCAN_BF16>();
}

Geom seq_geom(int dtype) {
    if (dtype == WKV4_F32) return seq_geom_t<WKV4_SEQ_F32>();
    if (dtype == WKV4_F16) return seq_geom_t<WKV4_SEQ_F16>();
    return seq_geom_t<WKV4_SEQ_BF16>();
}

static int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

// Cluster size: the largest power of two <= min(8, segments) whose grid
// (tiles x cluster size) still fits in one wave of resident CTAs; at least 1.
// WKV4_SCAN_CLUSTER=1|2|4|8 overrides (tuning).
static int pick_cluster(int64_t tiles, int64_t nseg, int blocks_per_sm) {
    const char* env = std::getenv("WKV4_SCAN_CLUSTER");
    if (env) {
        const int v = std::atoi(env);
        if (v == 1 || v == 2 || v == 4 || v == 8) return v;
    }
    const int64_t cap = (int64_t)blocks_per_sm * sm_count();
    int nc = 1;
    while (nc < 8 && nc * 2 <= nseg && tiles * nc * 2 <= cap) nc *= 2;
    return nc;
}

template <typename IO, int V, int L, int NW, int NB, bool kTMA>
static cudaError_t launch_scan_nb(const FwdArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                                  const CUtensorMap& ty, ScanParams p, int nc, int64_t tiles) {
    using Sh = ScanShape<IO, V, L, NW, NB>;
    auto kern = wkv4_scan_kernel<IO, V, L, NW, NB, kTMA>;
    static DeviceFlags attr;
    cudaError_t e = ensure_smem_attr(attr, kern, Sh::kSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)(tiles * nc), 1, 1);
    cfg.blockDim = dim3(Sh::kThreads, 1, 1);
    cfg.dynamicSmemBytes = Sh::kSmem;
    cfg.stream = a.stream;
    cudaLaunchAttribute attrs[1];
    attrs[0].id = cudaLaunchAttributeClusterDimension;
    attrs[0].val.clusterDim.x = (unsigned)nc;
    attrs[0].val.clusterDim.y = 1;
    attrs[0].val.clusterDim.z = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tk, tv, ty, p);
}

template <typename IO, int V, int L, int NW, bool kTMA>
static cudaError_t launch_scan_t(const FwdArgs& a, const CUtensorMap* tk, const CUtensorMap* tv,
                                 const CUtensorMap* ty) {
    using Sh1 = ScanShape<IO, V, L, NW, 1>;
    ScanParams p;
    p.T = a.T;
    p.C = a.C;
    p.CGB = (int)((a.C + Sh1::kCg - 1) / Sh1::kCg);
    p.w = a.w;
    p.u = a.u;
    p.k = a.k;
    p.v = a.v;
    p.state_in = a.state_in;
    p.y = a.y;
    p.state_out = a.state_out;
    p.BC = a.B * a.C;
    const int64_t tiles = a.B * p.CGB;
    const int64_t nseg = (a.T + Sh1::kTs - 1) / Sh1::kTs;
    // resident CTAs per SM of the single-buffer kernel, cached per device
    auto k1 = wkv4_scan_kernel<IO, V, L, NW, 1, kTMA>;
    static DeviceFlags attr1;
    static std::atomic<int> bps_cache[64];
    cudaError_t e = ensure_smem_attr(attr1, k1, Sh1::kSmem);
    if (e != cudaSuccess) return e;
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    int bps = (dev >= 0 && dev < 64) ? bps_cache[dev].load(std::memory_order_relaxed) : 0;
    if (bps <= 0) {
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, k1, Sh1::kThreads,
                                                               Sh1::kSmem)) != cudaSuccess)
            return e;
        bps = bps > 0 ? bps : 1;
        if (dev >= 0 && dev < 64) bps_cache[dev].store(bps, std::memory_order_relaxed);
    }
    const int nc = pick_cluster(tiles, nseg, bps);
    p.rounds = (int)((nseg + nc - 1) / nc);
    CUtensorMap dummy;
    std::memset(&dummy, 0, sizeof(dummy));
    const CUtensorMap& mk = tk ? *tk : dummy;
    const CUtensorMap& mv = tv ? *tv : dummy;
    const CUtensorMap& my = ty ? *ty : dummy;
    if (p.rounds == 1) return launch_scan_nb<IO, V, L, NW, 1, kTMA>(a, mk, mv, my, p, nc, tiles);
    return launch_scan_nb<IO, V, L, NW, 2, kTMA>(a, mk, mv, my, p, nc, tiles);
}

cudaError_t launch_scan(const FwdArgs& a, const CUtensorMap* tk, const CUtensorMap* tv,
                        const CUtensorMap* ty) {
    const bool tma = tk != nullptr;
    switch (a.dtype) {
        case WKV4_F32:
            return tma ? launch_scan_t<WKV4_SCAN_F32, true>(a, tk, tv, ty)
                       : launch_scan_t<WKV4_SCAN_F32, false>(a, tk, tv, ty);
        case WKV4_F16:
            if (!tma) return launch_scan_t<WKV4_SCAN_F16, false>(a, tk, tv, ty);
            switch (scan_cfg()) {
                case 1: return launch_scan_t<WKV4_SCAN_F16_1, true>(a, tk, tv, ty);
                case 2: return launch_scan_t<WKV4_SCAN_F16_2, true>(a, tk, tv, ty);
                case 3: return launch_scan_t<WKV4_SCAN_F16_3, true>(a, tk, tv, ty);
                default: return launch_scan_t<WKV4_SCAN_F16, true>(a, tk, tv, ty);
            }
        default:
            return tma ? launch_scan_t<WKV4_SCAN_BF16, true>(a, tk, tv, ty)
                       : launch_scan_t<WKV4_SCAN_BF16, false>(a, tk, tv, ty);
    }
}

template <typename IO, int V, int L, int NW, int NS>
static cudaError_t launch_seq_t(const FwdArgs& a, const CUtensorMap* tk, const CUtensorMap* tv) {
    using Sh = SeqShape<IO, V, L, NW, NS>;
    auto kern = wkv4_seq_kernel<IO, V, L, NW, NS>;
    static DeviceFlags attr;
    cudaError_t e = ensure_smem_attr(attr, kern, Sh::kSmem);
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
