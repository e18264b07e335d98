// Host side of libfa.so: argument validation, TMA descriptor encoding and the
// launch of the fused forward kernel. Declarations and the contract are in
// include/fa.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <algorithm>
#include <cstring>
#include <mutex>

#include "fa.h"
#include "fa_fwd_kernel.cuh"

namespace fa {

// Per-device status word written by kernels (bit set = error seen).
__device__ uint32_t g_dev_err = 0;

// One CTA whose thread 0 waits, bounded, on a barrier nothing completes.
__global__ void watchdog_selftest_kernel(uint32_t* dev_err, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const Watchdog wd{&abort_flag, dev_err, limit_ns};
        (void)mbar_wait(&bar, 0u, wd);
    }
}

namespace {

constexpr int kMaxDevices = 64;
constexpr uint64_t kWatchdogNs = 1000000000ull;  // 1 s per bounded wait
constexpr int64_t kL2GroupBytes = 80ll << 20;     // K/V bytes of one launch-order head group

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceState {
    bool probed = false;
    bool supported = false;
    bool smem_set[3] = {false, false, false};  // d = 64, 128, 256
    uint32_t* err_ptr = nullptr;
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];
EncodeTiledFn g_encode = nullptr;

EncodeTiledFn encode_fn() {
    if (g_encode) return g_encode;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
        return nullptr;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    return g_encode;
}

// Device set-up (once per device, under the lock): capability check, the
// address of the status word, the opt-in shared-memory size.
int prepare_device(int d, int* dev_out, uint32_t** err_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_LAUNCH;
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mutex);
    DeviceState& st = g_dev[dev];
    if (!st.probed) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return FA_ERR_LAUNCH;
        st.supported = (major == 10 && minor == 0);
        if (st.supported) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_dev_err) != cudaSuccess) return FA_ERR_LAUNCH;
            st.err_ptr = static_cast<uint32_t*>(p);
        }
        st.probed = true;
    }
    if (!st.supported) return FA_ERR_UNSUPPORTED;
    const int di = (d == 256) ? 2 : (d == 128) ? 1 : 0;
    if (!st.smem_set[di]) {
        cudaError_t e =
            (d == 256) ? cudaFuncSetAttribute(fa_fwd_sm100<256>,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              Cfg<256>::kSmemBytes)
            : (d == 128) ? cudaFuncSetAttribute(fa_fwd_sm100<128>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                Cfg<128>::kSmemBytes)
                         : cudaFuncSetAttribute(fa_fwd_sm100<64>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                Cfg<64>::kSmemBytes);
        if (e != cudaSuccess) return FA_ERR_LAUNCH;
        st.smem_set[di] = true;
    }
    *dev_out = dev;
    *err_out = st.err_ptr;
    return FA_OK;
}

// 3-D view [B*H, N, d] of a contiguous bf16 tensor; box = 64 columns (128
// bytes, the swizzle width) x 128 rows x 1 head. The third dimension keeps a
// tile from ever crossing into the next head: rows past N read as zero.
int make_map(CUtensorMap* map, const void* ptr, int BH, int N, int d) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return FA_ERR_LAUNCH;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * (cuuint64_t)d * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_INVALID_ARG;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
             int H_kv, int N, int d, float scale, int causal, const int32_t* kv_len,
             void* stream) {
    // ---- arguments (synchronous, nothing launched on error)
    if (B < 0 || H < 0 || N < 0) return FA_ERR_INVALID_ARG;
    if (H > 0 && (H_kv < 1 || H_kv > H || H % H_kv != 0)) return FA_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
    if (B == 0 || H == 0 || N == 0) return FA_OK;
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    const uintptr_t a16 = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                          reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o);
    if ((a16 & 15u) != 0 || (reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
        return FA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(kv_len) & 3u) != 0) return FA_ERR_INVALID_ARG;
    const int64_t BH = (int64_t)B * H;
    const int64_t BHkv = (int64_t)B * H_kv;
    const int64_t rows_per_unit = (d == 256) ? 128 : 256;   // query tiles per unit x 128
    const int64_t n_units = ((int64_t)N + rows_per_unit - 1) / rows_per_unit;
    if (BH > INT32_MAX || BH * n_units > INT32_MAX) return FA_ERR_INVALID_ARG;
    const size_t elems = (size_t)BH * (size_t)N * (size_t)d;
    if ((double)BH * N * d > 9.0e18) return FA_ERR_INVALID_ARG;
    const size_t tbytes = elems * 2, lbytes = (size_t)BH * (size_t)N * 4;
    const size_t kvbytes = (size_t)BHkv * (size_t)N * (size_t)d * 2;
    if (overlaps(o, tbytes, q, tbytes) || overlaps(o, tbytes, k, kvbytes) ||
        overlaps(o, tbytes, v, kvbytes) || overlaps(lse, lbytes, q, tbytes) ||
        overlaps(lse, lbytes, k, kvbytes) || overlaps(lse, lbytes, v, kvbytes) ||
        overlaps(lse, lbytes, o, tbytes))
        return FA_ERR_INVALID_ARG;

    int dev = 0;
    uint32_t* err = nullptr;
    int rc = prepare_device(d, &dev, &err);
    if (rc != FA_OK) return rc;

    alignas(64) CUtensorMap mq, mk, mv;
    if ((rc = make_map(&mq, q, (int)BH, N, d)) != FA_OK) return rc;
    if ((rc = make_map(&mk, k, (int)BHkv, N, d)) != FA_OK) return rc;
    if ((rc = make_map(&mv, v, (int)BHkv, N, d)) != FA_OK) return rc;

    FwdParams p{};
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.kv_len = kv_len;
    p.dev_err = err;
    p.B = B;
    p.H = H;
    p.H_kv = H_kv;
    p.N = N;
    p.n_units = (int)n_units;
    // Launch-order head groups: as few groups as keep a group's K/V (2*N*d*2
    // bytes per K/V head, shared by H / H_kv query heads) within
    // kL2GroupBytes, with the query heads split evenly.
    const int64_t kv_head_bytes = (int64_t)N * d * 4;
    const int64_t cap = std::max<int64_t>(1, kL2GroupBytes / kv_head_bytes) * (H / H_kv);
    const int64_t groups = (BH + cap - 1) / cap;
    p.group_heads = (int)((BH + groups - 1) / groups);
    p.causal = causal;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.watchdog_ns = kWatchdogNs;

    const dim3 grid((unsigned)(BH * n_units)), block(kThreads);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (d == 256)
        fa_fwd_sm100<256><<<grid, block, Cfg<256>::kSmemBytes, s>>>(mq, mk, mv, p);
    else if (d == 128)
        fa_fwd_sm100<128><<<grid, block, Cfg<128>::kSmemBytes, s>>>(mq, mk, mv, p);
    else
        fa_fwd_sm100<64><<<grid, block, Cfg<64>::kSmemBytes, s>>>(mq, mk, mv, p);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

}  // namespace
}  // namespace fa

#define FA_EXPORT __attribute__((visibility("default")))

extern "C" {

FA_EXPORT int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
           int d, float scale, int causal, void* stream) {
    return fa::fwd_impl(q, k, v, o, lse, B, H, H, N, d, scale, causal, nullptr, stream);
}

FA_EXPORT int fa_fwd_kvlen(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int H, int N, int d, float scale, int causal,
                           const int32_t* kv_len, void* stream) {
    return fa::fwd_impl(q, k, v, o, lse, B, H, H, N, d, scale, causal, kv_len, stream);
}

FA_EXPORT int fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
                         int B, int H, int H_kv, int N, int d, float scale, int causal,
                         const int32_t* kv_len, void* stream) {
    return fa::fwd_impl(q, k, v, o, lse, B, H, H_kv, N, d, scale, causal, kv_len, stream);
}

FA_EXPORT const char* fa_status_string(int status) {
    switch (status) {
        case FA_OK: return "FA_OK";
        case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: invalid argument";
        case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: unsupported head dim or device";
        case FA_ERR_LAUNCH: return "FA_ERR_LAUNCH: CUDA launch or synchronisation failed";
        case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a kernel wait ran out of time";
        default: return "unknown fa status";
    }
}

FA_EXPORT int fa_watchdog_selftest(uint64_t limit_ns, void* stream) {
    if (limit_ns < 1000ull || limit_ns > 5000000000ull) return FA_ERR_INVALID_ARG;
    int dev = 0;
    uint32_t* err = nullptr;
    const int rc = fa::prepare_device(64, &dev, &err);
    if (rc != FA_OK) return rc;
    fa::watchdog_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, limit_ns);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

FA_EXPORT int fa_last_device_error(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return FA_ERR_LAUNCH;
    uint32_t v = 0;
    if (cudaMemcpyFromSymbol(&v, fa::g_dev_err, sizeof v) != cudaSuccess) return FA_ERR_LAUNCH;
    if (v != 0) {
        const uint32_t zero = 0;
        if (cudaMemcpyToSymbol(fa::g_dev_err, &zero, sizeof zero) != cudaSuccess)
            return FA_ERR_LAUNCH;
    }
    return (v & fa::DEVERR_TIMEOUT) ? FA_ERR_TIMEOUT : FA_OK;
}

}  // extern "C"
