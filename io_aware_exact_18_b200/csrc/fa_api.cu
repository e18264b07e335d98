// Host side of libfa.so: argument validation, TMA descriptor encoding and the
// launches of the forward (square, split-KV with its merge, e4m3), backward
// and diagnostic kernels. Declarations and the contract are in include/fa.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <algorithm>
#include <cstring>
#include <mutex>

#include "fa.h"
#include "fa_bwd_kernel.cuh"
#include "fa_combine_kernel.cuh"
#include "fa_decode_kernel.cuh"
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
constexpr int kMaxSplits = FA_MAX_SPLITS;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceState {
    bool probed = false;
    bool supported = false;
    uint32_t* err_ptr = nullptr;
};

// Opt in to the dynamic shared memory of the two backward passes.
template <int D>
bool set_bwd_smem() {
    return cudaFuncSetAttribute(fa_bwd_dkdv<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                BwdCfg<D>::kSmemBytes) == cudaSuccess &&
           cudaFuncSetAttribute(fa_bwd_dq<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                BwdCfg<D>::kSmemBytes) == cudaSuccess;
}

// Opt in to the dynamic shared memory of one kernel instantiation.
template <int D, int QT, bool kGen, int E = 2>
bool set_smem() {
    return cudaFuncSetAttribute(fa_fwd_sm100<D, QT, kGen, E>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Cfg<D, QT, E>::kSmemBytes) == cudaSuccess;
}

template <int D, int E>
bool set_decode_smem() {
    return cudaFuncSetAttribute(fa_decode_sm100<D, E>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                DecCfg<D, E>::kSmemBytes) == cudaSuccess;
}

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
// address of the status word, the opt-in shared-memory size of every kernel.
int prepare_device(int* dev_out, uint32_t** err_out) {
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
            const bool ok = set_smem<64, 2, false>() && set_smem<128, 2, false>() &&
                            set_smem<256, 1, false>() && set_smem<64, 1, true>() &&
                            set_smem<128, 1, true>() && set_smem<256, 1, true>() &&
                            set_smem<128, 2, false, 1>() && set_smem<256, 1, false, 1>() &&
                            set_smem<128, 1, true, 1>() && set_smem<256, 1, true, 1>() &&
                            set_smem<64, 2, false, 1>() && set_smem<64, 1, true, 1>() &&
                            set_decode_smem<128, 2>() && set_decode_smem<128, 1>() &&
                            set_bwd_smem<64>() &&
                            set_bwd_smem<128>();
            if (!ok) return FA_ERR_LAUNCH;
        }
        st.probed = true;
    }
    if (!st.supported) return FA_ERR_UNSUPPORTED;
    // Launch failures are read back through cudaGetLastError: clear an error
    // an earlier, unrelated runtime call may have left there (a sticky error
    // stays and fails the launch anyway).
    (void)cudaGetLastError();
    *dev_out = dev;
    *err_out = st.err_ptr;
    return FA_OK;
}

// 3-D view [B*H, N, d] of a contiguous bf16 (elem = 2) or 8-bit (elem = 1)
// tensor; box = 128 bytes of columns (the swizzle width) x box_rows rows x
// box_planes heads. The third dimension keeps a tile from ever crossing into
// the next head: rows past N read as zero.
int encode_map(CUtensorMap* map, const void* ptr, int BH, int N, int d, int box_rows,
               int box_planes, int elem) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return FA_ERR_LAUNCH;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)d * elem, (cuuint64_t)N * (cuuint64_t)d * elem};
    // one column block of a tile per box: 128-byte rows with the 128-byte
    // swizzle, or whole 64-byte rows (e4m3 at d = 64) with the 64-byte swizzle
    const int row_bytes = std::min(128, d * elem);
    cuuint32_t box[3] = {(cuuint32_t)(row_bytes / elem), (cuuint32_t)box_rows,
                         (cuuint32_t)box_planes};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                     3, const_cast<void*>(ptr), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_INVALID_ARG;
}

// Encoded maps of recent calls, keyed by everything a map encodes (device,
// address, shape, box, element size), so a loop that calls the library with
// the same tensors pays for the encoding once. A map holds no reference to
// the memory: a later tensor at the same address with the same shape gets the
// same, still correct, map. Small and replaced round-robin.
struct MapKey {
    int dev;
    const void* ptr;
    int BH, N, d, box_rows, box_planes, elem;
    bool operator==(const MapKey& o) const {
        return dev == o.dev && ptr == o.ptr && BH == o.BH && N == o.N && d == o.d &&
               box_rows == o.box_rows && box_planes == o.box_planes && elem == o.elem;
    }
};
constexpr int kMapCache = 32;
struct MapEntry {
    bool used = false;
    MapKey key{};
    alignas(64) CUtensorMap map;
};
std::mutex g_map_mutex;
MapEntry g_maps[kMapCache];
int g_map_next = 0;

int make_map(CUtensorMap* map, int dev, const void* ptr, int BH, int N, int d, int box_rows = 128,
             int box_planes = 1, int elem = 2) {
    const MapKey key{dev, ptr, BH, N, d, box_rows, box_planes, elem};
    {
        std::lock_guard<std::mutex> lk(g_map_mutex);
        for (const MapEntry& e : g_maps)
            if (e.used && e.key == key) {
                *map = e.map;
                return FA_OK;
            }
    }
    const int rc = encode_map(map, ptr, BH, N, d, box_rows, box_planes, elem);
    if (rc != FA_OK) return rc;
    std::lock_guard<std::mutex> lk(g_map_mutex);
    MapEntry& e = g_maps[g_map_next];
    g_map_next = (g_map_next + 1) % kMapCache;
    e.used = true;
    e.key = key;
    e.map = *map;
    return FA_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

// One forward call. Q [B,H,Nq,d]; K, V [B,H_kv,Nk,d]; O [B,H,Nq,d]; lse
// [B,H,Nq]. splits > 1 writes per-range partials into `ws` and merges them.
struct FwdCall {
    const void *q, *k, *v;
    void* o;
    float* lse;
    int B, H, H_kv, Nq, Nk, d;
    float scale;
    int causal;
    const int32_t* kv_len;
    int splits;          // >= 1
    bool pack;           // pack the query heads of a K/V group into one tile
    void* ws;            // split partials (splits > 1)
    size_t ws_bytes;
    int elem = 2;        // bytes per element of q, k, v: 2 (bf16) or 1 (e4m3)
    float q_descale = 1.f, k_descale = 1.f, v_descale = 1.f;   // e4m3 inputs
};

// Workspace layout for `splits` ranges: O partials fp32 [splits][B*H][Nq][d],
// then (256-byte aligned) lse partials fp32 [splits][B*H][Nq].
size_t ws_o_bytes(int64_t rows, int d, int splits) {
    const size_t b = (size_t)splits * (size_t)rows * (size_t)d * 4;
    return (b + 255) & ~size_t(255);
}
size_t ws_total_bytes(int64_t rows, int d, int splits) {
    if (splits <= 1) return 0;
    return ws_o_bytes(rows, d, splits) + (size_t)splits * (size_t)rows * 4;
}

// Query heads per tile and rows per head in a tile.
void tile_shape(int H, int H_kv, int Nq, bool pack, int* G, int* nq_blk) {
    const int grp = H / H_kv;
    if (pack && grp > 1 && grp <= kTile) {
        *G = grp;
        *nq_blk = std::min(Nq, kTile / grp);
    } else {
        *G = 1;
        *nq_blk = kTile;
    }
}

// Shapes derived from a forward call's arguments.
struct FwdPlan {
    bool empty = false;      // B, H or Nq is 0: nothing to compute
    int64_t BH = 0, BHkv = 0, BHB = 0, rows = 0, n_units = 0;
    int G = 1, nq_blk = kTile, qt = 2;
    bool general = false;
    size_t tbytes = 0, lbytes = 0, qbytes = 0, kvbytes = 0;   // o, lse, q, k (= v) bytes
};

// Every host-side check of a forward call except its split-KV workspace
// (synchronous, no CUDA call). Sizes are bounded before they are multiplied,
// so no product can overflow.
int fwd_check(const FwdCall& a, FwdPlan* pl) {
    const int B = a.B, H = a.H, H_kv = a.H_kv, Nq = a.Nq, Nk = a.Nk, d = a.d;
    if (B < 0 || H < 0 || Nq < 0 || Nk < 0 || Nq > Nk) return FA_ERR_INVALID_ARG;
    if (H > 0 && (H_kv < 1 || H_kv > H || H % H_kv != 0)) return FA_ERR_INVALID_ARG;
    if (a.causal != 0 && a.causal != 1) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(a.scale) || !(a.scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (a.splits < 1 || a.splits > kMaxSplits) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
    const int E = a.elem;
    if (E == 1) {
        for (float x : {a.q_descale, a.k_descale, a.v_descale})
            if (!std::isfinite(x) || !(x > 0.f)) return FA_ERR_INVALID_ARG;
    }
    if (B == 0 || H == 0 || Nq == 0) {
        pl->empty = true;
        return FA_OK;
    }
    if (!a.q || !a.k || !a.v || !a.o || !a.lse) return FA_ERR_INVALID_ARG;
    const uintptr_t a16 = reinterpret_cast<uintptr_t>(a.q) | reinterpret_cast<uintptr_t>(a.k) |
                          reinterpret_cast<uintptr_t>(a.v) | reinterpret_cast<uintptr_t>(a.o);
    if ((a16 & 15u) != 0 || (reinterpret_cast<uintptr_t>(a.lse) & 3u) != 0)
        return FA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(a.kv_len) & 3u) != 0) return FA_ERR_INVALID_ARG;
    // B, H, Nq < 2^31, so each product of two of them fits in int64
    pl->BH = (int64_t)B * H;
    pl->BHkv = (int64_t)B * H_kv;
    if (pl->BH > INT32_MAX) return FA_ERR_INVALID_ARG;
    pl->rows = pl->BH * Nq;
    if (pl->rows > INT32_MAX) return FA_ERR_INVALID_ARG;   // row indices are 32-bit in the kernel
    tile_shape(H, H_kv, Nq, a.pack, &pl->G, &pl->nq_blk);
    // Square attention (one key range, no packing, Nq == Nk) runs the
    // specialised kernels; everything else the general one-query-tile kernel.
    pl->general = a.splits > 1 || pl->G > 1 || Nq != Nk;
    pl->qt = (pl->general || d == 256) ? 1 : 2;              // query tiles per unit
    const int64_t n_rb = ((int64_t)Nq + pl->nq_blk - 1) / pl->nq_blk;
    pl->n_units = (n_rb + pl->qt - 1) / pl->qt * a.splits;    // <= 2^31 * 128
    pl->BHB = pl->BH / pl->G;
    if (pl->n_units > INT32_MAX || pl->BHB > INT32_MAX / pl->n_units) return FA_ERR_INVALID_ARG;
    if ((double)pl->BHkv * Nk * d > 9.0e18) return FA_ERR_INVALID_ARG;
    pl->tbytes = (size_t)pl->rows * d * 2;
    pl->lbytes = (size_t)pl->rows * 4;
    pl->qbytes = (size_t)pl->rows * d * E;
    pl->kvbytes = (size_t)pl->BHkv * (size_t)Nk * (size_t)d * E;
    if (overlaps(a.o, pl->tbytes, a.q, pl->qbytes) || overlaps(a.o, pl->tbytes, a.k, pl->kvbytes) ||
        overlaps(a.o, pl->tbytes, a.v, pl->kvbytes) ||
        overlaps(a.lse, pl->lbytes, a.q, pl->qbytes) ||
        overlaps(a.lse, pl->lbytes, a.k, pl->kvbytes) ||
        overlaps(a.lse, pl->lbytes, a.v, pl->kvbytes) || overlaps(a.lse, pl->lbytes, a.o, pl->tbytes))
        return FA_ERR_INVALID_ARG;
    return FA_OK;
}

int fwd_impl(const FwdCall& a, void* stream) {
    // ---- arguments (synchronous, nothing launched on error)
    FwdPlan pl;
    int rc = fwd_check(a, &pl);
    if (rc != FA_OK || pl.empty) return rc;
    const int B = a.B, H = a.H, H_kv = a.H_kv, Nq = a.Nq, Nk = a.Nk, d = a.d, E = a.elem;
    const int64_t BH = pl.BH, BHkv = pl.BHkv, BHB = pl.BHB, rows = pl.rows, n_units = pl.n_units;
    const int G = pl.G, nq_blk = pl.nq_blk;
    float* o_part = nullptr;
    float* lse_part = nullptr;
    if (a.splits > 1) {
        const size_t need = ws_total_bytes(rows, d, a.splits);
        if (a.ws == nullptr || a.ws_bytes < need || (reinterpret_cast<uintptr_t>(a.ws) & 15u) != 0)
            return FA_ERR_INVALID_ARG;
        if (overlaps(a.ws, need, a.q, pl.qbytes) || overlaps(a.ws, need, a.k, pl.kvbytes) ||
            overlaps(a.ws, need, a.v, pl.kvbytes) || overlaps(a.ws, need, a.o, pl.tbytes) ||
            overlaps(a.ws, need, a.lse, pl.lbytes))
            return FA_ERR_INVALID_ARG;
        o_part = static_cast<float*>(a.ws);
        lse_part = reinterpret_cast<float*>(static_cast<uint8_t*>(a.ws) +
                                            ws_o_bytes(rows, d, a.splits));
    }

    int dev = 0;
    uint32_t* err = nullptr;
    rc = prepare_device(&dev, &err);
    if (rc != FA_OK) return rc;

    alignas(64) CUtensorMap mq, mk, mv;
    if ((rc = make_map(&mq, dev, a.q, (int)BH, Nq, d, nq_blk, G, E)) != FA_OK) return rc;
    if ((rc = make_map(&mk, dev, a.k, (int)BHkv, Nk, d, 128, 1, E)) != FA_OK) return rc;
    if ((rc = make_map(&mv, dev, a.v, (int)BHkv, Nk, d, 128, 1, E)) != FA_OK) return rc;

    FwdParams p{};
    p.o = static_cast<__nv_bfloat16*>(a.o);
    p.lse = a.lse;
    p.o_part = o_part;
    p.lse_part = lse_part;
    p.kv_len = a.kv_len;
    p.dev_err = err;
    p.B = B;
    p.H = H;
    p.H_kv = H_kv;
    p.Nq = Nq;
    p.Nk = Nk;
    p.q_off = Nk - Nq;
    p.G = G;
    p.nq_blk = nq_blk;
    p.n_rb = (int)(((int64_t)Nq + nq_blk - 1) / nq_blk);
    p.splits = a.splits;
    p.n_units = (int)n_units;
    // Launch-order head groups: as few groups as keep a group's K/V (2*Nk*d*2
    // bytes per K/V head, shared by H / H_kv query heads, G of them per head
    // block) within kL2GroupBytes, with the head blocks split evenly.
    const int64_t kv_head_bytes = (int64_t)Nk * d * 4;
    const int64_t cap =
        std::max<int64_t>(1, kL2GroupBytes / kv_head_bytes) * ((H / H_kv) / G);
    const int64_t groups = (BHB + cap - 1) / cap;
    p.group_heads = (int)((BHB + groups - 1) / groups);
    p.causal = a.causal;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.o_mul = 1.f;
    if (E == 1) {
        p.scale_log2 = (float)((double)a.scale * a.q_descale * a.k_descale * 1.4426950408889634);
        p.o_mul = a.v_descale;
    }
    p.watchdog_ns = kWatchdogNs;

    const dim3 grid((unsigned)(BHB * n_units)), block(kThreads);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // Decoding shapes (d = 128, a K/V group's query heads times the query rows
    // within kDecLive columns: one row block per group) take the transposed
    // tile; the unit grid is the same (head group, range) set.
    const bool dec = d == 128 && pl.general && Nq == nq_blk && (int64_t)G * Nq <= kDecLive &&
                     G == H / H_kv;
    if (dec && E == 2) {
        fa_decode_sm100<128, 2><<<grid, dim3(kDecThreads), DecCfg<128, 2>::kSmemBytes, s>>>(mq, mk, mv, p);
    } else if (dec) {
        fa_decode_sm100<128, 1><<<grid, dim3(kDecThreads), DecCfg<128, 1>::kSmemBytes, s>>>(mq, mk, mv, p);
    } else if (E == 1) {
        if (pl.general && d == 256)
            fa_fwd_sm100<256, 1, true, 1><<<grid, block, Cfg<256, 1, 1>::kSmemBytes, s>>>(mq, mk, mv, p);
        else if (pl.general && d == 128)
            fa_fwd_sm100<128, 1, true, 1><<<grid, block, Cfg<128, 1, 1>::kSmemBytes, s>>>(mq, mk, mv, p);
        else if (pl.general)
            fa_fwd_sm100<64, 1, true, 1><<<grid, block, Cfg<64, 1, 1>::kSmemBytes, s>>>(mq, mk, mv, p);
        else if (d == 256)
            fa_fwd_sm100<256, 1, false, 1><<<grid, block, Cfg<256, 1, 1>::kSmemBytes, s>>>(mq, mk, mv, p);
        else if (d == 128)
            fa_fwd_sm100<128, 2, false, 1><<<grid, block, Cfg<128, 2, 1>::kSmemBytes, s>>>(mq, mk, mv, p);
        else
            fa_fwd_sm100<64, 2, false, 1><<<grid, block, Cfg<64, 2, 1>::kSmemBytes, s>>>(mq, mk, mv, p);
    } else if (pl.general) {
        if (d == 256)
            fa_fwd_sm100<256, 1, true><<<grid, block, Cfg<256, 1>::kSmemBytes, s>>>(mq, mk, mv, p);
        else if (d == 128)
            fa_fwd_sm100<128, 1, true><<<grid, block, Cfg<128, 1>::kSmemBytes, s>>>(mq, mk, mv, p);
        else
            fa_fwd_sm100<64, 1, true><<<grid, block, Cfg<64, 1>::kSmemBytes, s>>>(mq, mk, mv, p);
    } else {
        if (d == 256)
            fa_fwd_sm100<256, 1, false><<<grid, block, Cfg<256, 1>::kSmemBytes, s>>>(mq, mk, mv, p);
        else if (d == 128)
            fa_fwd_sm100<128, 2, false><<<grid, block, Cfg<128, 2>::kSmemBytes, s>>>(mq, mk, mv, p);
        else
            fa_fwd_sm100<64, 2, false><<<grid, block, Cfg<64, 2>::kSmemBytes, s>>>(mq, mk, mv, p);
    }
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
    if (a.splits > 1) {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3((unsigned)((rows + kCombineWarps - 1) / kCombineWarps));
        cfg.blockDim = dim3(32 * kCombineWarps);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = s;
        // After the decoding kernel (not persistent; each CTA signals once it
        // has started) the merge is a programmatic dependent: its launch
        // overlaps the decoding grid's tail and it waits for that grid's
        // completion before reading the partials.
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = dec ? 1 : 0;
        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.o);
        cudaError_t e;
        if (d == 256)
            e = cudaLaunchKernelEx(&cfg, fa_splitkv_combine<256>, (const float*)o_part,
                                   (const float*)lse_part, o, a.lse, (int64_t)rows, a.splits,
                                   (const uint32_t*)err);
        else if (d == 128)
            e = cudaLaunchKernelEx(&cfg, fa_splitkv_combine<128>, (const float*)o_part,
                                   (const float*)lse_part, o, a.lse, (int64_t)rows, a.splits,
                                   (const uint32_t*)err);
        else
            e = cudaLaunchKernelEx(&cfg, fa_splitkv_combine<64>, (const float*)o_part,
                                   (const float*)lse_part, o, a.lse, (int64_t)rows, a.splits,
                                   (const uint32_t*)err);
        if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
    }
    return FA_OK;
}

// ------------------------------------------------------------------ static scratch
// Split-KV scratch owned by the library, for fa_fwd_splitkv_static: callers
// that cannot allocate device memory at call time get the partials' space from
// this array, which the CUDA module reserves on each device when it loads.
static __device__ __align__(256) unsigned char g_splitkv_scratch[FA_STATIC_SCRATCH_BYTES];
void* g_scratch_ptr[kMaxDevices] = {};

// Address of the current device's scratch, looked up once per device (with
// that device current) and cached.
int static_scratch(void** out) {
    int dev = 0;
    uint32_t* err = nullptr;
    int rc = prepare_device(&dev, &err);   // capability check first
    if (rc != FA_OK) return rc;
    std::lock_guard<std::mutex> lk(g_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_splitkv_scratch) != cudaSuccess || p == nullptr)
            return FA_ERR_LAUNCH;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return FA_OK;
}

// ------------------------------------------------------------------ backward
// Workspace of the backward pass: lse * log2(e), then D = rowsum(dO * O), each
// fp32 [B*H][Np] with Np = N rounded up to whole 128-row tiles.
int64_t bwd_np(int N) { return ((int64_t)N + 127) / 128 * 128; }
size_t bwd_ws_bytes(int64_t BH, int N) { return 2 * (size_t)BH * (size_t)bwd_np(N) * 4; }

int bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse,
             const void* d_o, void* dq, void* dk, void* dv, int B, int H, int H_kv, int N,
             int d, float scale, int causal, const int32_t* kv_len, void* ws, size_t ws_bytes,
             void* stream) {
    if (B < 0 || H < 0 || N < 0) return FA_ERR_INVALID_ARG;
    if (H > 0 && (H_kv < 1 || H_kv > H || H % H_kv != 0)) return FA_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (B == 0 || H == 0 || N == 0) return FA_OK;
    if (!q || !k || !v || !o || !lse || !d_o || !dq || !dk || !dv || !ws)
        return FA_ERR_INVALID_ARG;
    const uintptr_t a16 =
        reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o) |
        reinterpret_cast<uintptr_t>(d_o) | reinterpret_cast<uintptr_t>(dq) |
        reinterpret_cast<uintptr_t>(dk) | reinterpret_cast<uintptr_t>(dv) |
        reinterpret_cast<uintptr_t>(ws);
    if ((a16 & 15u) != 0 || (reinterpret_cast<uintptr_t>(lse) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(kv_len) & 3u) != 0)
        return FA_ERR_INVALID_ARG;
    const int64_t BH = (int64_t)B * H, BHkv = (int64_t)B * H_kv;   // < 2^62
    const int64_t Np = bwd_np(N), n_t = Np / 128;
    if (BH > INT32_MAX || BH * Np > INT32_MAX) return FA_ERR_INVALID_ARG;
    if (ws_bytes < bwd_ws_bytes(BH, N)) return FA_ERR_INVALID_ARG;
    const size_t qb = (size_t)BH * N * d * 2, kb = (size_t)BHkv * N * d * 2;
    const size_t lb = (size_t)BH * N * 4, wb = bwd_ws_bytes(BH, N);
    struct Buf { const void* p; size_t n; };
    const Buf outs[4] = {{dq, qb}, {dk, kb}, {dv, kb}, {ws, wb}};
    const Buf all[10] = {{q, qb}, {k, kb}, {v, kb}, {o, qb}, {lse, lb}, {d_o, qb},
                         {dq, qb}, {dk, kb}, {dv, kb}, {ws, wb}};
    for (int a = 0; a < 4; ++a)       // every output against every other buffer
        for (int c = 0; c < 10; ++c)
            if (c != 6 + a && overlaps(outs[a].p, outs[a].n, all[c].p, all[c].n))
                return FA_ERR_INVALID_ARG;

    int dev = 0;
    uint32_t* err = nullptr;
    int rc = prepare_device(&dev, &err);
    if (rc != FA_OK) return rc;
    alignas(64) CUtensorMap mq, mk, mv, mdo;
    if ((rc = make_map(&mq, dev, q, (int)BH, N, d)) != FA_OK) return rc;
    if ((rc = make_map(&mk, dev, k, (int)BHkv, N, d)) != FA_OK) return rc;
    if ((rc = make_map(&mv, dev, v, (int)BHkv, N, d)) != FA_OK) return rc;
    if ((rc = make_map(&mdo, dev, d_o, (int)BH, N, d)) != FA_OK) return rc;

    float* lse2 = static_cast<float*>(ws);
    float* dvec = lse2 + BH * Np;
    BwdParams p{};
    p.dq = static_cast<__nv_bfloat16*>(dq);
    p.dk = static_cast<__nv_bfloat16*>(dk);
    p.dv = static_cast<__nv_bfloat16*>(dv);
    p.lse2 = lse2;
    p.dvec = dvec;
    p.kv_len = kv_len;
    p.dev_err = err;
    p.B = B;
    p.H = H;
    p.H_kv = H_kv;
    p.N = N;
    p.Np = (int)Np;
    p.causal = causal;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.watchdog_ns = kWatchdogNs;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const dim3 pgrid((unsigned)((BH * Np + 7) / 8)), pblock(256);
    const dim3 agrid((unsigned)(BHkv * n_t)), bgrid((unsigned)(BH * n_t)), block(kBwdThreads);
    const __nv_bfloat16* ob = static_cast<const __nv_bfloat16*>(o);
    const __nv_bfloat16* dob = static_cast<const __nv_bfloat16*>(d_o);
    if (d == 128) {
        fa_bwd_prep<128><<<pgrid, pblock, 0, s>>>(ob, dob, lse, lse2, dvec, BH, N, (int)Np);
        fa_bwd_dkdv<128><<<agrid, block, BwdCfg<128>::kSmemBytes, s>>>(mq, mk, mv, mdo, p);
        fa_bwd_dq<128><<<bgrid, block, BwdCfg<128>::kSmemBytes, s>>>(mq, mk, mv, mdo, p);
    } else {
        fa_bwd_prep<64><<<pgrid, pblock, 0, s>>>(ob, dob, lse, lse2, dvec, BH, N, (int)Np);
        fa_bwd_dkdv<64><<<agrid, block, BwdCfg<64>::kSmemBytes, s>>>(mq, mk, mv, mdo, p);
        fa_bwd_dq<64><<<bgrid, block, BwdCfg<64>::kSmemBytes, s>>>(mq, mk, mv, mdo, p);
    }
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

FwdCall square_call(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int H, int H_kv, int N, int d, float scale, int causal,
                    const int32_t* kv_len) {
    FwdCall a{};
    a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
    a.B = B; a.H = H; a.H_kv = H_kv; a.Nq = N; a.Nk = N; a.d = d;
    a.scale = scale; a.causal = causal; a.kv_len = kv_len;
    a.splits = 1; a.pack = false; a.ws = nullptr; a.ws_bytes = 0;
    return a;
}

}  // namespace
}  // namespace fa

#define FA_EXPORT __attribute__((visibility("default")))

extern "C" {

FA_EXPORT int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
           int d, float scale, int causal, void* stream) {
    return fa::fwd_impl(fa::square_call(q, k, v, o, lse, B, H, H, N, d, scale, causal, nullptr),
                        stream);
}

FA_EXPORT int fa_fwd_kvlen(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int H, int N, int d, float scale, int causal,
                           const int32_t* kv_len, void* stream) {
    return fa::fwd_impl(fa::square_call(q, k, v, o, lse, B, H, H, N, d, scale, causal, kv_len),
                        stream);
}

FA_EXPORT int fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
                         int B, int H, int H_kv, int N, int d, float scale, int causal,
                         const int32_t* kv_len, void* stream) {
    return fa::fwd_impl(
        fa::square_call(q, k, v, o, lse, B, H, H_kv, N, d, scale, causal, kv_len), stream);
}

FA_EXPORT size_t fa_splitkv_workspace_bytes(int B, int H, int Nq, int d, int num_splits) {
    if (B < 0 || H < 0 || Nq < 0 || num_splits < 1 || num_splits > fa::kMaxSplits ||
        (d != 64 && d != 128 && d != 256))
        return 0;
    const int64_t bh = (int64_t)B * H;                  // < 2^62
    if (bh > INT32_MAX || bh * Nq > INT32_MAX) return 0;
    return fa::ws_total_bytes(bh * Nq, d, num_splits);
}

FA_EXPORT int fa_splitkv_default_splits(int B, int H, int H_kv, int Nq, int Nk, int d) {
    if (B < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || Nq < 1 || Nk < 1) return 1;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms = 148;
    int G = 1, nq_blk = fa::kTile;
    fa::tile_shape(H, H_kv, Nq, true, &G, &nq_blk);
    const int64_t n_rb = ((int64_t)Nq + nq_blk - 1) / nq_blk;
    const int64_t base = (int64_t)B * (H / G) * n_rb;
    const int64_t key_tiles = ((int64_t)Nk + fa::kTile - 1) / fa::kTile;
    // Each unit pays a fixed cost (its Q tile, the first scores, the epilogue and
    // the partials the merge reads back), and a second wave of units leaves most
    // SMs idle for its last part, so the units are kept to one wave: as many
    // ranges as fit base * ranges <= the cap, each at least four key tiles long;
    // a workload with at least as many units as the cap takes one range. The cap
    // is the SM count for the general kernel (measured on one head group of
    // 131072 keys: 18 ranges, 144 units, 5493 GB/s; 16 ranges, 128 units, 5069;
    // 24 ranges, two waves, 3663). The transposed decoding tile (d = 128, G * Nq
    // <= 8 columns) streams K and V at the HBM rate and ran fastest with 128
    // units in flight on every shape measured (1, 2 or 4 sequences x 8 K/V heads,
    // one query row: 6007, 6116, 6186 GB/s at 128 units against 5655 and 5692
    // at 144), so its cap is 128.
    const bool dec = d == 128 && G == H / H_kv && nq_blk == Nq && (int64_t)G * Nq <= fa::kDecLive;
    const int64_t cap = dec ? std::min<int64_t>(sms, 128) : sms;
    const int64_t s_max = std::min<int64_t>(fa::kMaxSplits, std::max<int64_t>(1, key_tiles / 4));
    const int64_t sp = base >= cap ? 1 : cap / base;
    return (int)std::max<int64_t>(1, std::min<int64_t>(sp, s_max));
}

FA_EXPORT int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int H, int H_kv, int Nq, int Nk, int d, float scale,
                             int causal, const int32_t* kv_len, int num_splits, void* workspace,
                             size_t workspace_bytes, void* stream) {
    fa::FwdCall a{};
    a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
    a.B = B; a.H = H; a.H_kv = H_kv; a.Nq = Nq; a.Nk = Nk; a.d = d;
    a.scale = scale; a.causal = causal; a.kv_len = kv_len;
    a.splits = num_splits; a.pack = true; a.ws = workspace; a.ws_bytes = workspace_bytes;
    return fa::fwd_impl(a, stream);
}

FA_EXPORT int fa_fwd_splitkv_static(const void* q, const void* k, const void* v, void* o,
                                    float* lse, int B, int H, int H_kv, int Nq, int Nk, int d,
                                    float scale, int causal, const int32_t* kv_len,
                                    int num_splits, void* stream) {
    fa::FwdCall a{};
    a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
    a.B = B; a.H = H; a.H_kv = H_kv; a.Nq = Nq; a.Nk = Nk; a.d = d;
    a.scale = scale; a.causal = causal; a.kv_len = kv_len;
    a.splits = num_splits; a.pack = true; a.ws = nullptr; a.ws_bytes = 0;
    // The same argument checks as fa_fwd_splitkv, in the same order (so both
    // entry points return the same status), then the scratch's size, all on
    // the host before any CUDA call.
    fa::FwdPlan pl;
    const int arc = fa::fwd_check(a, &pl);
    if (arc != FA_OK || pl.empty) return arc;
    if (num_splits == 1) return fa::fwd_impl(a, stream);   // one range: no partials
    if (fa::ws_total_bytes(pl.rows, d, num_splits) > (size_t)FA_STATIC_SCRATCH_BYTES)
        return FA_ERR_INVALID_ARG;
    void* scratch = nullptr;
    const int rc = fa::static_scratch(&scratch);
    if (rc != FA_OK) return rc;
    a.ws = scratch;
    a.ws_bytes = (size_t)FA_STATIC_SCRATCH_BYTES;
    return fa::fwd_impl(a, stream);
}

FA_EXPORT int fa_fwd_fp8(const void* q, const void* k, const void* v, float q_descale,
                         float k_descale, float v_descale, void* o, float* lse, int B, int H,
                         int H_kv, int N, int d, float scale, int causal,
                         const int32_t* kv_len, void* stream) {
    fa::FwdCall a = fa::square_call(q, k, v, o, lse, B, H, H_kv, N, d, scale, causal, kv_len);
    a.elem = 1;
    a.q_descale = q_descale;
    a.k_descale = k_descale;
    a.v_descale = v_descale;
    return fa::fwd_impl(a, stream);
}

FA_EXPORT int fa_fwd_splitkv_fp8(const void* q, const void* k, const void* v, float q_descale,
                                 float k_descale, float v_descale, void* o, float* lse, int B,
                                 int H, int H_kv, int Nq, int Nk, int d, float scale, int causal,
                                 const int32_t* kv_len, int num_splits, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    fa::FwdCall a{};
    a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
    a.B = B; a.H = H; a.H_kv = H_kv; a.Nq = Nq; a.Nk = Nk; a.d = d;
    a.scale = scale; a.causal = causal; a.kv_len = kv_len;
    a.splits = num_splits; a.pack = true; a.ws = workspace; a.ws_bytes = workspace_bytes;
    a.elem = 1;
    a.q_descale = q_descale;
    a.k_descale = k_descale;
    a.v_descale = v_descale;
    return fa::fwd_impl(a, stream);
}

FA_EXPORT size_t fa_bwd_workspace_bytes(int B, int H, int N) {
    if (B < 0 || H < 0 || N < 0 || (int64_t)B * H > INT32_MAX) return 0;
    return fa::bwd_ws_bytes((int64_t)B * H, N);
}

FA_EXPORT int fa_bwd(const void* q, const void* k, const void* v, const void* o,
                     const float* lse, const void* d_o, void* dq, void* dk, void* dv, int B,
                     int H, int H_kv, int N, int d, float scale, int causal,
                     const int32_t* kv_len, void* workspace, size_t workspace_bytes,
                     void* stream) {
    return fa::bwd_impl(q, k, v, o, lse, d_o, dq, dk, dv, B, H, H_kv, N, d, scale, causal,
                        kv_len, workspace, workspace_bytes, stream);
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
    const int rc = fa::prepare_device(&dev, &err);
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
