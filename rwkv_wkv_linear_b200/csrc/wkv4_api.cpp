// C ABI of the RWKV-4 WKV forward / decode step: argument checks, kernel
// choice and TMA descriptors.  Every step of the
// computation runs in the kernels of wkv4_kernels.cu; nothing here computes.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/wkv4.h"
#include "wkv4_internal.h"

namespace {

using wkv4::FwdArgs;

// ------------------------------------------------------------------ helpers

struct Range {
    uintptr_t lo, hi;  // [lo, hi)
};

Range range_of(const void* p, uint64_t bytes) {
    const uintptr_t lo = (uintptr_t)p;
    return {lo, lo + (uintptr_t)bytes};
}

bool overlap(Range a, Range b) {
    if (a.lo == 0 || b.lo == 0 || a.lo == a.hi || b.lo == b.hi) return false;
    return a.lo < b.hi && b.lo < a.hi;
}

bool is_aligned(const void* p, size_t n) { return p == nullptr || ((uintptr_t)p % n) == 0; }

// Driver entry point of cuTensorMapEncodeTiled, fetched once through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// 3-D map over a [B][T][C] tensor (dims innermost first: C, T, B) with a
// box of box_c channels x box_t steps x 1 batch row; out-of-range elements
// read as zero and are skipped on store.
bool encode_btc_uncached(CUtensorMap* map, const void* ptr, int dtype, int64_t B, int64_t T,
                         int64_t C, int box_c, int box_t) {
    auto fn = encode_fn();
    if (!fn) return false;
    const size_t es = wkv4::dtype_size(dtype);
    const CUtensorMapDataType dt = dtype == WKV4_F32   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                   : dtype == WKV4_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                       : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[2] = {(cuuint64_t)(C * es), (cuuint64_t)(T * C * es)};
    const cuuint32_t box[3] = {(cuuint32_t)box_c, (cuuint32_t)box_t, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, dt, 3, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// encode_btc_uncached through a small per-thread cache: a map depends only on
// its arguments, and callers run the same buffers call after call (encoding
// one costs about a microsecond of host time, three a call).
struct MapKey {
    const void* ptr;
    int64_t B, T, C;
    int dtype, box_c, box_t;
    bool operator==(const MapKey& o) const {
        return ptr == o.ptr && B == o.B && T == o.T && C == o.C && dtype == o.dtype &&
               box_c == o.box_c && box_t == o.box_t;
    }
};

bool encode_btc(CUtensorMap* map, const void* ptr, int dtype, int64_t B, int64_t T, int64_t C,
                int box_c, int box_t) {
    constexpr int kEntries = 64;
    struct Entry {
        MapKey key;
        CUtensorMap map;
        bool used;
    };
    static thread_local Entry cache[kEntries];
    static thread_local int next = 0;
    const MapKey key{ptr, B, T, C, dtype, box_c, box_t};
    for (int i = 0; i < kEntries; ++i) {
        if (cache[i].used && cache[i].key == key) {
            *map = cache[i].map;
            return true;
        }
    }
    if (!encode_btc_uncached(map, ptr, dtype, B, T, C, box_c, box_t)) return false;
    Entry& e = cache[next];
    next = (next + 1) % kEntries;
    e.key = key;
    e.map = *map;
    e.used = true;
    return true;
}

// TMA needs 16-byte aligned bases and row strides that are multiples of 16 bytes.
bool tma_eligible(const FwdArgs& a) {
    const size_t es = wkv4::dtype_size(a.dtype);
    return (a.C * (int64_t)es) % 16 == 0 && is_aligned(a.k, 16) && is_aligned(a.v, 16) &&
           is_aligned(a.y, 16) && is_aligned(a.r, 16) && a.T < (1ll << 31) &&
           a.C < (1ll << 31) && a.B < (1ll << 31);
}

int check_common(int64_t B, int64_t T, int64_t C, int dtype) {
    if (B < 0 || T < 0 || C < 0) return WKV4_ERR_ARG;
    if (dtype != WKV4_F32 && dtype != WKV4_F16 && dtype != WKV4_BF16) return WKV4_ERR_DTYPE;
    return WKV4_OK;
}

int check_alias(const FwdArgs& a) {
    const size_t es = wkv4::dtype_size(a.dtype);
    const uint64_t io = (uint64_t)a.B * a.T * a.C * es;
    const uint64_t st = (uint64_t)3 * a.B * a.C * 4;
    const Range ry = range_of(a.y, io), rk = range_of(a.k, io), rv = range_of(a.v, io);
    const Range rr = range_of(a.r, io);
    const Range rw = range_of(a.w, a.C * 4), ru = range_of(a.u, a.C * 4);
    const Range rsi = range_of(a.state_in, st), rso = range_of(a.state_out, st);
    if (overlap(ry, rk) || overlap(ry, rv) || overlap(ry, rw) || overlap(ry, ru) ||
        overlap(ry, rsi) || overlap(ry, rso) || overlap(ry, rr))
        return WKV4_ERR_ALIAS;
    if (overlap(rso, rk) || overlap(rso, rv) || overlap(rso, rw) || overlap(rso, ru) ||
        overlap(rso, rr))
        return WKV4_ERR_ALIAS;
    if (overlap(rso, rsi) && a.state_in != a.state_out) return WKV4_ERR_ALIAS;
    return WKV4_OK;
}

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return WKV4_OK;
    cudaGetLastError();
    return WKV4_ERR_CUDA;
}

int run_scan(const FwdArgs& a, bool want_tma) {
    return cuda_status(wkv4::launch_scan(a, want_tma && tma_eligible(a), encode_btc));
}

int run_seq(const FwdArgs& a) {
    if (!tma_eligible(a) || !is_aligned(a.y, 16)) return run_scan(a, false);
    const wkv4::Geom g = wkv4::seq_geom(a.dtype);
    CUtensorMap tk, tv, tr;
    if (!encode_btc(&tk, a.k, a.dtype, a.B, a.T, a.C, g.box_c, g.box_t) ||
        !encode_btc(&tv, a.v, a.dtype, a.B, a.T, a.C, g.box_c, g.box_t) ||
        (a.r && !encode_btc(&tr, a.r, a.dtype, a.B, a.T, a.C, g.box_c, g.box_t)))
        return WKV4_ERR_CUDA;
    return cuda_status(wkv4::launch_seq(a, &tk, &tv, a.r ? &tr : &tk));
}

// Kernel choice of wkv4_forward.  The sequential kernel needs enough channel
// groups to fill the SMs on its own; otherwise the chunked scan splits T.
int pick_variant(const FwdArgs& a) {
    if (!tma_eligible(a)) return WKV4_KERNEL_SCAN_LDG;
    if (a.B * a.C >= (1ll << 19) && a.T >= 64) return WKV4_KERNEL_SEQ;
    return WKV4_KERNEL_SCAN;
}

int forward_impl(const FwdArgs& a, int variant) {
    int rc = check_common(a.B, a.T, a.C, a.dtype);
    if (rc != WKV4_OK) return rc;
    if (variant < WKV4_KERNEL_AUTO || variant > WKV4_KERNEL_STEP) return WKV4_ERR_VARIANT;
    if (a.B == 0 || a.C == 0) return WKV4_OK;
    if (a.T == 0) {
        rc = check_alias(a);
        if (rc != WKV4_OK) return rc;
        return cuda_status(wkv4::launch_copy_state(a));
    }
    if (!a.w || !a.u || !a.k || !a.v || !a.y) return WKV4_ERR_ARG;
    rc = check_alias(a);
    if (rc != WKV4_OK) return rc;
    if (a.T == 1 && variant == WKV4_KERNEL_AUTO) return cuda_status(wkv4::launch_decode(a));
    if (variant == WKV4_KERNEL_AUTO) variant = pick_variant(a);
    switch (variant) {
        case WKV4_KERNEL_SEQ: return run_seq(a);
        case WKV4_KERNEL_SCAN: return run_scan(a, true);
        case WKV4_KERNEL_SCAN_LDG: return run_scan(a, false);
        default: return cuda_status(wkv4::launch_step(a));
    }
}

}  // namespace

extern "C" {

int wkv4_forward(int64_t B, int64_t T, int64_t C, const float* w, const float* u, const void* k,
                 const void* v, const float* state_in, void* y, float* state_out,
                 wkv4_stream_t stream, int dtype) {
    return wkv4_forward_variant(B, T, C, w, u, k, v, state_in, y, state_out, stream, dtype,
                                WKV4_KERNEL_AUTO);
}

int wkv4_forward_variant(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                         const void* k, const void* v, const float* state_in, void* y,
                         float* state_out, wkv4_stream_t stream, int dtype, int variant) {
    FwdArgs a{B, T, C, w, u, k, v, state_in, y, state_out, dtype, (cudaStream_t)stream};
    return forward_impl(a, variant);
}

int wkv4_forward_gated(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                       const void* k, const void* v, const void* r, const float* state_in,
                       void* y, float* state_out, wkv4_stream_t stream, int dtype) {
    return wkv4_forward_gated_variant(B, T, C, w, u, k, v, r, state_in, y, state_out, stream,
                                      dtype, WKV4_KERNEL_AUTO);
}

int wkv4_forward_gated_variant(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                               const void* k, const void* v, const void* r,
                               const float* state_in, void* y, float* state_out,
                               wkv4_stream_t stream, int dtype, int variant) {
    if (T > 0 && B > 0 && C > 0 && !r) return WKV4_ERR_ARG;
    FwdArgs a{B, T, C, w, u, k, v, state_in, y, state_out, dtype, (cudaStream_t)stream, r};
    return forward_impl(a, variant);
}

int wkv4_decode_step(int64_t B, int64_t C, const float* w, const float* u, const void* k,
                     const void* v, float* state, void* y, wkv4_stream_t stream, int dtype) {
    int rc = check_common(B, 1, C, dtype);
    if (rc != WKV4_OK) return rc;
    if (B == 0 || C == 0) return WKV4_OK;
    if (!w || !u || !k || !v || !y || !state) return WKV4_ERR_ARG;
    FwdArgs a{B, 1, C, w, u, k, v, state, y, state, dtype, (cudaStream_t)stream};
    rc = check_alias(a);
    if (rc != WKV4_OK) return rc;
    return cuda_status(wkv4::launch_decode(a));
}

int wkv4_decode_step_gated(int64_t B, int64_t C, const float* w, const float* u, const void* k,
                           const void* v, const void* r, float* state, void* y,
                           wkv4_stream_t stream, int dtype) {
    int rc = check_common(B, 1, C, dtype);
    if (rc != WKV4_OK) return rc;
    if (B == 0 || C == 0) return WKV4_OK;
    if (!w || !u || !k || !v || !r || !y || !state) return WKV4_ERR_ARG;
    FwdArgs a{B, 1, C, w, u, k, v, state, y, state, dtype, (cudaStream_t)stream, r};
    rc = check_alias(a);
    if (rc != WKV4_OK) return rc;
    return cuda_status(wkv4::launch_decode(a));
}

int wkv4_decode_step_slots(int64_t B, int64_t C, int64_t S, const float* w, const float* u,
                           const void* k, const void* v, float* state_pool,
                           const int32_t* slot_ids, void* y, wkv4_stream_t stream, int dtype) {
    int rc = check_common(B, 1, C, dtype);
    if (rc != WKV4_OK) return rc;
    if (S < 0) return WKV4_ERR_ARG;
    if (B == 0 || C == 0) return WKV4_OK;
    if (!w || !u || !k || !v || !y || !state_pool || !slot_ids) return WKV4_ERR_ARG;
    const size_t es = wkv4::dtype_size(dtype);
    const uint64_t io = (uint64_t)B * C * es;
    const Range ry = range_of(y, io), rk = range_of(k, io), rv = range_of(v, io);
    const Range rw = range_of(w, C * 4), ru = range_of(u, C * 4);
    const Range rp = range_of(state_pool, (uint64_t)3 * S * C * 4), rs = range_of(slot_ids, B * 4);
    if (overlap(ry, rk) || overlap(ry, rv) || overlap(ry, rw) || overlap(ry, ru) || overlap(ry, rp) ||
        overlap(ry, rs))
        return WKV4_ERR_ALIAS;
    if (overlap(rp, rk) || overlap(rp, rv) || overlap(rp, rw) || overlap(rp, ru) || overlap(rp, rs))
        return WKV4_ERR_ALIAS;
    FwdArgs a{B, 1, C, w, u, k, v, state_pool, y, state_pool, dtype, (cudaStream_t)stream};
    return cuda_status(wkv4::launch_decode_slots(a, slot_ids, S));
}

int wkv4_token_shift(int64_t B, int64_t T, int64_t C, const void* x, const void* x_prev,
                     const float* mix_k, const float* mix_v, const float* mix_r, void* xk,
                     void* xv, void* xr, void* x_last, wkv4_stream_t stream, int dtype) {
    int rc = check_common(B, T, C, dtype);
    if (rc != WKV4_OK) return rc;
    if (B == 0 || C == 0) return WKV4_OK;
    const size_t es = wkv4::dtype_size(dtype);
    const uint64_t io = (uint64_t)B * T * C * es, row = (uint64_t)B * C * es;
    if (T == 0) {  // x_last <- x_prev (or zeros)
        if (!x_last) return WKV4_OK;
        if (overlap(range_of(x_last, row), range_of(x_prev, row))) return WKV4_ERR_ALIAS;
        cudaError_t e = x_prev ? cudaMemcpyAsync(x_last, x_prev, row, cudaMemcpyDeviceToDevice,
                                                 (cudaStream_t)stream)
                               : cudaMemsetAsync(x_last, 0, row, (cudaStream_t)stream);
        return cuda_status(e);
    }
    if (!x || !mix_k || !mix_v || !xk || !xv || (mix_r && !xr)) return WKV4_ERR_ARG;
    if (B > 65535 || T > 65535ll * 16) return WKV4_ERR_ARG;  // grid z (rows), y (at most 65535 runs)
    if (!mix_r) xr = nullptr;
    const Range in[5] = {range_of(x, io), range_of(x_prev, row), range_of(mix_k, C * 4),
                         range_of(mix_v, C * 4), range_of(mix_r, mix_r ? C * 4 : 0)};
    const Range out[4] = {range_of(xk, io), range_of(xv, io), range_of(xr, xr ? io : 0),
                          range_of(x_last, row)};
    for (int i = 0; i < 4; ++i) {
        for (int j = 0; j < 5; ++j)
            if (overlap(out[i], in[j])) return WKV4_ERR_ALIAS;
        for (int j = i + 1; j < 4; ++j)
            if (overlap(out[i], out[j])) return WKV4_ERR_ALIAS;
    }
    wkv4::ShiftArgs a{B, T, C, x, x_prev, {mix_k, mix_v, mix_r}, {xk, xv, xr}, x_last, dtype,
                      (cudaStream_t)stream};
    return cuda_status(wkv4::launch_token_shift(a));
}

int wkv4_state_combine(int64_t B, int64_t C, const float* w, int64_t n_steps, const float* x,
                       const float* y, float* out, wkv4_stream_t stream) {
    if (B < 0 || C < 0 || n_steps < 0) return WKV4_ERR_ARG;
    if (B == 0 || C == 0) return WKV4_OK;
    if (!w || !y || !out) return WKV4_ERR_ARG;
    if (B * C > (int64_t)UINT32_MAX * 256) return WKV4_ERR_ARG;
    const uint64_t st = (uint64_t)3 * B * C * 4;
    const Range ro = range_of(out, st), rx = range_of(x, st), ry = range_of(y, st);
    if (overlap(ro, range_of(w, C * 4))) return WKV4_ERR_ALIAS;
    if (overlap(ro, rx) && out != x) return WKV4_ERR_ALIAS;
    if (overlap(ro, ry) && out != y) return WKV4_ERR_ALIAS;
    return cuda_status(wkv4::launch_state_combine(B, C, w, n_steps, x, y, out, (cudaStream_t)stream));
}

int wkv4_device_error(int reset) {
    unsigned bits = 0;
    if (wkv4::read_device_error(&bits, reset != 0) != cudaSuccess) {
        cudaGetLastError();
        return WKV4_ERR_CUDA;
    }
    if (bits & (wkv4::kErrTmaWait | wkv4::kErrExchangeWait)) return WKV4_ERR_TIMEOUT;
    return bits ? WKV4_ERR_SLOT : WKV4_OK;
}

const char* wkv4_status_string(int status) {
    switch (status) {
        case WKV4_OK: return "ok";
        case WKV4_ERR_ARG: return "invalid argument (NULL pointer or negative size)";
        case WKV4_ERR_DTYPE: return "unknown dtype";
        case WKV4_ERR_ALIAS: return "output overlaps an input";
        case WKV4_ERR_CUDA: return "CUDA runtime error";
        case WKV4_ERR_TIMEOUT: return "a bounded device-side wait ran out";
        case WKV4_ERR_VARIANT: return "unknown kernel variant";
        case WKV4_ERR_SLOT: return "a decode row named a state slot outside the pool";
        default: return "unknown status";
    }
}

int wkv4_version(void) { return 100; }

}  // extern "C"
