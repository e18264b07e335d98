// Split-KV forward for decoding: few query rows per K/V head, many keys.
//
// The same attention as fa_fwd_sm100's general form ("FlashAttention (UR)",
// section "Specialised solutions": inference against a key-value cache), with
// the tile transposed. When the query heads of a K/V group times the query
// rows fit in kDecLive = 8 columns (one-token decoding with grouped heads: 4
// or 8 heads x 1 row), a
// 128-row query tile would be almost all padding, and its softmax warps would
// run a full 128-column exponential pass per key tile for a handful of live
// rows. Here the keys sit on the TMEM lanes instead:
//
//   S^T = K Q^T          M = 128 keys,  N = 16 query columns,  K = d
//   O^T += V^T P^T       M = d,         N = 16 query columns,  K = 128 keys
//
// (N = 16 is the narrowest tcgen05 product at M = 128; the columns past
// kDecLive are zero in Q and P^T) so each softmax thread owns one key and 8
// scores, and the exponential work per key tile drops 16-fold. (Sixteen live
// columns per thread would not fit the registers a thread of this CTA can
// hold: 168 in this 320-thread CTA.) The online softmax runs
// per query column
// ("FlashAttention (UR)", section "Online softmax"): a column's reference
// maximum m_ref is fixed from its first visible key tile and moves only when a
// later tile's column maximum exceeds it by more than 64 in log2 units, after
// O^T and the running sums are rescaled, so every probability is at most 2^64
// and the final O / l is exact whatever m_ref is. A tile's column maxima are
// taken across its 128 key threads (a reduce-scatter of shuffles in each warp,
// then the four warps' partial maxima through shared memory). The running sums
// stay per thread (the thread's own keys) and are reduced once, in the
// epilogue. As in the general kernel, O is divided by the sum of the
// probabilities as rounded to bf16 for the P.V product and lse takes the exact
// sum.
//
// kDecWG = 2 softmax warpgroups take the key tiles in turn (warpgroup w: tiles
// j with j % kDecWG == w), each with its own S^T and P^T buffers, O^T
// accumulator, reference maxima and sums, so the fixed latencies of one tile
// (TMEM load, shuffles, the maxima exchange, the hand-over) overlap the
// others'; the epilogue merges the parts by their log-sum-exp, as the split-KV
// merge does across ranges. (Three warpgroups, 448 threads at 128 registers,
// measured no faster: the tile period is not set by the softmax alone.)
//
// One CTA per unit (batch, K/V head group, key range); 320 threads:
//   warps 0-3, 4-7  softmax, one warpgroup each: thread t owns key t of a tile
//              (TMEM lane t) and, in warpgroup 0's epilogue, head-dim index t
//              of O^T
//   warp  8    TMA loads (one thread): Q once, then K and V tiles
//   warp  9    MMA issue (one thread) and the TMEM allocation
// TMEM (64 columns): S^T of each warpgroup (16 columns each), then O^T of
// each. Shared memory: the Q tile (16 rows x d) and one P^T buffer per
// warpgroup (16 rows x 128 keys), K-major in the 128-byte swizzled layout,
// then a ring of K/V slots in the layout the forward kernel uses.
//
// Order of the products: QK(0) | QK(1) PV(0) | QK(2) PV(1) | ... : the scores
// of the next kDecAhead = kDecWG - 1 tiles are issued before each P.V, so
// every warpgroup has a tile to work on. Every wait is bounded (Watchdog).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "fa_fwd_kernel.cuh"
#include "sm100_ptx.cuh"

namespace fa {

constexpr int kDecCols = 16;        // N of both products: query columns of the tile
constexpr int kDecLive = 8;         // live columns (G heads x Nq rows) the softmax handles
constexpr int kDecWG = 2;                    // softmax warpgroups, taking the key tiles in turn
constexpr int kDecAhead = kDecWG - 1;        // key tiles whose scores are issued ahead of a P.V
constexpr int kDecThreads = 32 * (4 * kDecWG + 2);
constexpr int kDecTmaWarp = 4 * kDecWG;
constexpr int kDecMmaWarp = 4 * kDecWG + 1;
static_assert(kDecWG >= 2 && kDecWG <= 3, "two or three softmax warpgroups");

// E: bytes per element of Q, K, V and P (2: bf16; 1: e4m3 with kind::f8f6f4
// products, P rounded to e4m3).
template <int D, int E>
struct DecCfg {
    static_assert(D == 128, "the transposed decode tile is built for d = 128");
    static_assert(E == 1 || E == 2, "bf16 or e4m3");
    static_assert(kDecLive <= kDecCols, "live columns within the product's N");
    static constexpr int kBlocks = D * E / 128;              // 128-byte column blocks per row
    static constexpr int kBlockElems = 128 / E;
    static constexpr int kBlockBytes = kTile * 128;          // 16 KB: one block of a K/V tile
    static constexpr int kTileBytes = kTile * D * E;         // 32 KB (bf16), 16 KB (e4m3)
    static constexpr int kColBlockBytes = kDecCols * 128;    // 2 KB: one block of a 16-row operand
    static constexpr int kQBytes = kBlocks * kColBlockBytes;
    static constexpr int kPBytes = (kTile * E / 128) * kColBlockBytes;   // 16 x 128 keys
    static constexpr int kSlots = E == 2 ? 6 : 12;           // K/V ring depth
    static constexpr int kSmemTiles = kQBytes + kDecWG * kPBytes + kSlots * kTileBytes;
    static constexpr int kSmemBytes = kSmemTiles + 1024 /*alignment*/ + 4096 /*barriers*/;
    static constexpr uint32_t kTmemCols = 2 * kDecWG * kDecCols <= 64 ? 64 : 128;
    static constexpr uint32_t col_s(int w) { return (uint32_t)(w * kDecCols); }
    static constexpr uint32_t col_o(int w) { return (uint32_t)((kDecWG + w) * kDecCols); }
    static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
    static_assert(kSlots <= 12, "K/V ring barriers");
};

struct DecBarriers {
    uint64_t q_full;
    uint64_t kv_full[12];
    uint64_t kv_empty[12];
    // per warpgroup w (key tiles j with j % kDecWG == w)
    uint64_t s_full[kDecWG];       // S^T of a key tile is in TMEM (MMA commit)
    uint64_t s_free[kDecWG];       // its 128 threads have read it (128 arrivals)
    uint64_t p_full[kDecWG];       // P^T in shared memory (128 arrivals)
    uint64_t p_free[kDecWG];       // P.V has read it (MMA commit)
    uint64_t pv_done[kDecWG];      // one phase per P.V product of the warpgroup
    uint64_t red_full[kDecWG][2];  // [w][tile parity within w]: column maxima (128 arrivals)
    uint64_t sum_full[kDecWG];     // column sums, epilogue (128 arrivals)
    uint64_t merge_full;           // the other warpgroups' column (m, l, lr) for warpgroup 0
    uint64_t o_final;         // every product of the unit has completed
    uint64_t teardown;
    float red[kDecWG][2][4][kDecLive];
    float sum_l[kDecWG][4][kDecLive];
    float sum_lr[kDecWG][4][kDecLive];
    float merge_m[kDecWG - 1][kDecLive], merge_l[kDecWG - 1][kDecLive],
        merge_lr[kDecWG - 1][kDecLive];
    uint32_t tmem_base;
    int abort;
    int skip;
};
static_assert(sizeof(DecBarriers) <= 4096, "barrier region");

// Reduce-scatter of kDecLive = 8 per-lane values over a warp with op:
// afterwards lane l holds op over the 32 lanes of column l >> 2 (the four
// lanes of a column agree). Three halving steps (4 + 2 + 1 shuffles) and two
// final exchanges.
template <bool kMax>
__device__ __forceinline__ float warp_reduce_scatter8(const float (&v)[kDecLive], int lane) {
    static_assert(kDecLive == 8, "three halving steps");
    auto op = [](float a, float b) { return kMax ? fmaxf(a, b) : a + b; };
    float w4[4], w2[2];
    const bool u16 = (lane & 16) != 0, u8 = (lane & 8) != 0, u4 = (lane & 4) != 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float keep = u16 ? v[4 + i] : v[i], give = u16 ? v[i] : v[4 + i];
        w4[i] = op(keep, __shfl_xor_sync(0xffffffffu, give, 16));
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float keep = u8 ? w4[2 + i] : w4[i], give = u8 ? w4[i] : w4[2 + i];
        w2[i] = op(keep, __shfl_xor_sync(0xffffffffu, give, 8));
    }
    const float keep = u4 ? w2[1] : w2[0], give = u4 ? w2[0] : w2[1];
    float w1 = op(keep, __shfl_xor_sync(0xffffffffu, give, 4));
    w1 = op(w1, __shfl_xor_sync(0xffffffffu, w1, 2));
    return op(w1, __shfl_xor_sync(0xffffffffu, w1, 1));
}

// Byte offset of element (row n, column k) of a K-major operand of 16 rows of
// E-byte elements in the 128-byte swizzled layout: 128-byte column blocks of
// 2 KB, rows of 128 bytes, the 16-byte chunk index XOR-ed with the row index
// mod 8.
template <int E>
__device__ __forceinline__ uint32_t kmajor16_offset(int n, int k) {
    const int kb = k * E;
    return (uint32_t)((kb >> 7) * (kDecCols * 128) + n * 128 +
                      ((((kb & 127) >> 4) ^ (n & 7)) << 4) + (kb & 15));
}

template <int D, int E>
__global__ void __launch_bounds__(kDecThreads, 1)
    fa_decode_sm100(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = DecCfg<D, E>;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sP = sQ + C::kQBytes;                          // one buffer per warpgroup
    uint8_t* sKV = sP + kDecWG * C::kPBytes;
    DecBarriers* bars = reinterpret_cast<DecBarriers*>(smem + C::kSmemTiles);

    // ---------------------------------------------------------- the unit
    // blockIdx.x = (b * (H / G) + head group) * splits + key range
    const int G = p.G, Nq = p.Nq;
    const int cols = G * Nq;                                // live query columns (<= 16)
    const int hpb = p.H / G;
    const int s_idx = (int)(blockIdx.x % (unsigned)p.splits);
    const int bh = (int)(blockIdx.x / (unsigned)p.splits);
    const int b = bh / hpb;
    const int h0 = (bh - b * hpb) * G;
    const int bkv = b * p.H_kv + h0 / (p.H / p.H_kv);
    int kv_lim = p.Nk;
    if (p.kv_len != nullptr) kv_lim = max(0, min(p.Nk, p.kv_len[b]));
    const int nkb = (kv_lim + kTile - 1) / kTile;
    const int kt0 = (int)((long long)s_idx * nkb / p.splits);
    const int kt1 = (int)((long long)(s_idx + 1) * nkb / p.splits);
    const int n = kt1 - kt0;                                // key tiles of this range

    // ---------------------------------------------------------- setup
    if (tid == 0) {
        mbar_init(&bars->q_full, 1);
        for (int s = 0; s < C::kSlots; ++s) {
            mbar_init(&bars->kv_full[s], 1);
            mbar_init(&bars->kv_empty[s], 1);
        }
        for (int w = 0; w < kDecWG; ++w) {
            mbar_init(&bars->s_full[w], 1);
            mbar_init(&bars->s_free[w], kTile);
            mbar_init(&bars->p_full[w], kTile);
            mbar_init(&bars->p_free[w], 1);
            mbar_init(&bars->pv_done[w], 1);
            mbar_init(&bars->red_full[w][0], kTile);
            mbar_init(&bars->red_full[w][1], kTile);
            mbar_init(&bars->sum_full[w], kTile);
        }
        mbar_init(&bars->merge_full, kTile * (kDecWG - 1));
        mbar_init(&bars->o_final, 1);
        mbar_init(&bars->teardown, 1);
        bars->abort = 0;
        bars->skip = (*reinterpret_cast<volatile uint32_t*>(p.dev_err) != 0u) ? 1 : 0;
        fence_mbarrier_init();
    }
    // Q rows past the live columns are never loaded and P^T rows past kDecLive
    // never written: zero both once, so the padding columns of S^T are finite
    // (and masked) and those of O^T stay 0.
    for (int e = tid; e < (C::kQBytes + kDecWG * C::kPBytes) / 16; e += kDecThreads)
        reinterpret_cast<uint4*>(sQ)[e] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    if (warp == kDecMmaWarp) {
        tmem_alloc(&bars->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == kDecTmaWarp && lane == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // The split-KV merge queued behind this grid may be scheduled once every
    // CTA has started (it waits for this grid's completion before any read):
    // its launch overlaps this grid's tail instead of following it.
    pdl_launch_dependents();
    const uint32_t tmem = bars->tmem_base;
    const bool skip = bars->skip != 0;
    const Watchdog wd{&bars->abort, p.dev_err, p.watchdog_ns};

    if (skip) {
        // An earlier kernel on this device timed out (the status word is
        // sticky): no attention work; the unit's O rows and lse read NaN (its
        // split-KV partials are left alone: the merge checks the same word).
        if (p.o_part == nullptr && s_idx == 0)
            for (int e = tid; e < cols; e += kDecThreads) {
                const int g = e / Nq, r = e - (e / Nq) * Nq;
                const size_t row = (size_t)(b * p.H + h0 + g) * Nq + r;
                fill_nan_bf16(p.o + row * D, D);
                p.lse[row] = __int_as_float(0x7FC00000);
            }
    } else if (warp == kDecTmaWarp) {
        // ====================================================== TMA producer
        if (lane == 0) {
            const uint64_t pol_kv = policy_evict_first();
            bool ok = true;
            mbar_arrive_expect_tx(&bars->q_full, (uint32_t)(C::kBlocks * cols * 128));
            for (int blk = 0; blk < C::kBlocks; ++blk)
                tma_load_3d(&tm_q, &bars->q_full, sQ + blk * C::kColBlockBytes, blk * C::kBlockElems, 0,
                            b * p.H + h0);
            // Loads in the order the MMAs consume them (see the MMA issuer):
            // K(0) .. K(kDecAhead - 1), then K(i + kDecAhead) and V(i) for each i.
            int issued = 0;
            auto load = [&](bool is_v, int tile) -> bool {
                const int slot = issued % C::kSlots;
                const uint32_t round = (uint32_t)(issued / C::kSlots);
                if (!mbar_wait(&bars->kv_empty[slot], (round & 1u) ^ 1u, wd)) return false;
                uint8_t* dst = sKV + slot * C::kTileBytes;
                mbar_arrive_expect_tx(&bars->kv_full[slot], C::kTileBytes);
                for (int blk = 0; blk < C::kBlocks; ++blk)
                    tma_load_3d_hint(is_v ? &tm_v : &tm_k, &bars->kv_full[slot],
                                     dst + blk * C::kBlockBytes, blk * C::kBlockElems,
                                     (kt0 + tile) * kTile, bkv, pol_kv);
                ++issued;
                return true;
            };
            for (int j = 0; ok && j < min(kDecAhead, n); ++j) ok = load(false, j);
            for (int i = 0; ok && i < n; ++i) {
                if (i + kDecAhead < n) ok = load(false, i + kDecAhead);
                if (ok) ok = load(true, i);
            }
            // Drain: every copy issued must land before the CTA exits.
            for (int c = max(0, issued - C::kSlots); c < issued; ++c)
                mbar_wait_drain(&bars->kv_full[c % C::kSlots], (uint32_t)(c / C::kSlots) & 1u, wd);
            mbar_wait_drain(&bars->q_full, 0u, wd);
        }
        __syncwarp();
    } else if (warp == kDecMmaWarp) {
        // ====================================================== MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = E == 2 ? idesc_bf16_f32(128, kDecCols, 0, 0)   // K . Q^T
                                                : idesc_e4m3_f32(128, kDecCols, 0, 0);
            constexpr uint32_t idesc_o = E == 2 ? idesc_bf16_f32(128, kDecCols, 1, 0)   // V^T . P^T
                                                : idesc_e4m3_f32(128, kDecCols, 1, 0);
            auto mma = [&](uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
                if constexpr (E == 2) umma_ss(d_tmem, a, b, idesc, acc);
                else umma_ss_f8(d_tmem, a, b, idesc, acc);
            };
            const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t dk0 = smem_desc_sw128(smem_u32(sKV), 16, 1024);          // K-major
            const uint64_t dv0 = smem_desc_sw128(smem_u32(sKV), C::kBlockBytes, 1024); // MN-major
            const uint64_t dp0 = smem_desc_sw128(smem_u32(sP), 16, 1024);
            constexpr uint64_t kTileStep = (uint64_t)(C::kTileBytes >> 4);
            constexpr uint64_t kPStep = (uint64_t)(C::kPBytes >> 4);
            bool ok = mbar_wait(&bars->q_full, 0u, wd);
            int c = 0;   // K/V loads consumed, in the producer's order
            // S^T(j) = K(j) . Q^T into warpgroup (j % kDecWG)'s buffer, once it
            // has read its previous tile there
            auto issue_qk = [&](int j) -> bool {
                const int w = j % kDecWG;
                const int slot = c % C::kSlots;
                if (!mbar_wait(&bars->kv_full[slot], (uint32_t)(c / C::kSlots) & 1u, wd)) return false;
                if (j >= kDecWG &&
                    !mbar_wait(&bars->s_free[w], (uint32_t)(j / kDecWG - 1) & 1u, wd))
                    return false;
                tc_fence_after();
                const uint64_t a = dk0 + (uint64_t)slot * kTileStep;
#pragma unroll
                for (int kk = 0; kk < D * E / 32; ++kk) {       // 32-byte K-steps
                    const uint64_t oa = (uint64_t)(((kk >> 2) * C::kBlockBytes + (kk & 3) * 32) >> 4);
                    const uint64_t ob = (uint64_t)(((kk >> 2) * C::kColBlockBytes + (kk & 3) * 32) >> 4);
                    mma(tmem + C::col_s(w), a + oa, dq + ob, idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(&bars->s_full[w]);
                umma_commit(&bars->kv_empty[slot]);
                ++c;
                return true;
            };
            // O^T(w) += V(j)^T . P^T(j), w = j % kDecWG
            auto issue_pv = [&](int j) -> bool {
                const int w = j % kDecWG;
                const int slot = c % C::kSlots;
                if (!mbar_wait(&bars->kv_full[slot], (uint32_t)(c / C::kSlots) & 1u, wd)) return false;
                if (!mbar_wait(&bars->p_full[w], (uint32_t)(j / kDecWG) & 1u, wd)) return false;
                tc_fence_after();
                const uint64_t a = dv0 + (uint64_t)slot * kTileStep;
                const uint64_t bp = dp0 + (uint64_t)w * kPStep;
#pragma unroll
                for (int kk = 0; kk < kTile * E / 32; ++kk) {   // 32 / E keys per K-step
                    const uint64_t oa = (uint64_t)((kk * (32 / E) * 128) >> 4);
                    const uint64_t ob = (uint64_t)(((kk >> 2) * C::kColBlockBytes + (kk & 3) * 32) >> 4);
                    mma(tmem + C::col_o(w), a + oa, bp + ob, idesc_o,
                        (j >= kDecWG || kk > 0) ? 1u : 0u);
                }
                umma_commit(&bars->pv_done[w]);
                umma_commit(&bars->p_free[w]);
                umma_commit(&bars->kv_empty[slot]);
                ++c;
                return true;
            };
            // QK(0) .. QK(kDecAhead - 1) | QK(i + kDecAhead) PV(i) | ...: while P.V(i)
            // waits for its probabilities, the scores of the next kDecAhead tiles are
            // in flight, one per other warpgroup.
            for (int j = 0; ok && j < min(kDecAhead, n); ++j) ok = issue_qk(j);
            for (int i = 0; ok && i < n; ++i) {
                if (i + kDecAhead < n) ok = issue_qk(i + kDecAhead);
                if (ok) ok = issue_pv(i);
            }
            umma_commit(&bars->o_final);
            // Drain: all MMAs issued by this thread complete before teardown.
            umma_commit(&bars->teardown);
            mbar_wait_drain(&bars->teardown, 0u, wd);
        }
        __syncwarp();
    } else {
        // ====================================================== softmax (warps 0 .. 4 kDecWG - 1)
        const int wg = warp >> 2;                           // warpgroup: key tiles j % kDecWG == wg
        const int wq = warp & 3;                            // warp within the warpgroup
        const int t = tid & (kTile - 1);                    // key of a tile / head-dim index
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        const float c = p.scale_log2;
        float m_ref[kDecLive], l[kDecLive], lr[kDecLive];
#pragma unroll
        for (int q = 0; q < kDecLive; ++q) {
            m_ref[q] = -INFINITY;
            l[q] = 0.f;
            lr[q] = 0.f;
        }
        bool ok = true;
        for (int j = wg; j < n; j += kDecWG) {
            const int jo = j / kDecWG;                      // index among this warpgroup's tiles
            const int rb = jo & 1;                          // maxima buffer
            ok = mbar_wait(&bars->s_full[wg], (uint32_t)jo & 1u, wd);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            uint32_t r[kDecLive];
            tmem_ld8(tmem + lane_base + C::col_s(wg), r);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bars->s_free[wg]);
            // mask: column q = g * Nq + row sees key < kv_lim, and with the causal
            // mask key <= row + Nk - Nq; padding columns (q >= G * Nq) see none
            const int key = (kt0 + j) * kTile + t;
            const bool key_in = key < kv_lim;
            const int key_rel = p.causal ? key - p.q_off : INT32_MIN;
            float s[kDecLive];
            int row = 0;
#pragma unroll
            for (int q = 0; q < kDecLive; ++q) {
                s[q] = (key_in && q < cols && key_rel <= row) ? __uint_as_float(r[q]) : -INFINITY;
                row = (row + 1 == Nq) ? 0 : row + 1;
            }

            // column maxima of the tile over its 128 keys
            const float wmax = warp_reduce_scatter8<true>(s, lane);
            if ((lane & 3) == 0) bars->red[wg][rb][wq][lane >> 2] = wmax;
            mbar_arrive(&bars->red_full[wg][rb]);   // each thread releases its own write
            ok = mbar_wait(&bars->red_full[wg][rb], (uint32_t)(jo >> 1) & 1u, wd);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            auto tile_max = [&](int q) {
                return fmaxf(fmaxf(bars->red[wg][rb][0][q], bars->red[wg][rb][1][q]),
                             fmaxf(bars->red[wg][rb][2][q], bars->red[wg][rb][3][q]));
            };
            bool rescale = false;
#pragma unroll
            for (int q = 0; q < kDecLive; ++q) {
                const float tmax = tile_max(q);
                if (m_ref[q] == -INFINITY) m_ref[q] = tmax;
                else if ((tmax - m_ref[q]) * c > rescale_log2<E>()) rescale = true;
            }
            if (rescale) {   // uniform in the warpgroup: every thread sees the same maxima
                // O^T(wg) holds the products of this warpgroup's tiles < j; the
                // last of them, P.V(j - kDecWG), was issued before Q.K^T(j), whose
                // scores are in, so pv_done is exactly at that phase. Then each
                // column that moves is scaled; thread t holds head-dim row t.
                ok = mbar_wait(&bars->pv_done[wg], (uint32_t)(jo - 1) & 1u, wd);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
                uint32_t o[kDecLive];
                tmem_ld8(tmem + lane_base + C::col_o(wg), o);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < kDecLive; ++q) {
                    const float tmax = tile_max(q);
                    if ((tmax - m_ref[q]) * c > rescale_log2<E>()) {
                        const float alpha = fast_exp2((m_ref[q] - tmax) * c);
                        m_ref[q] = tmax;
                        l[q] *= alpha;
                        lr[q] *= alpha;
                        o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
                    }
                }
                tmem_st8(tmem + lane_base + C::col_o(wg), o);
                tmem_wait_st();
            }

            // probabilities of this key, rounded to bf16 (e4m3) into the warpgroup's P^T
            if (jo >= 1) {   // P.V(j - kDecWG) has read the buffer (complete, as above)
                ok = mbar_wait(&bars->p_free[wg], (uint32_t)(jo - 1) & 1u, wd);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
            }
            uint8_t* pbuf = sP + wg * C::kPBytes;
            float pv[kDecLive];
#pragma unroll
            for (int q = 0; q < kDecLive; ++q) {
                const float mc = (m_ref[q] == -INFINITY) ? 0.f : m_ref[q] * c;
                pv[q] = fast_exp2(fmaf(s[q], c, -mc));
                l[q] += pv[q];
            }
            if constexpr (E == 2) {
#pragma unroll
                for (int q = 0; q < kDecLive; ++q) {
                    const __nv_bfloat16 pb = __float2bfloat16_rn(pv[q]);
                    lr[q] += __bfloat162float(pb);
                    *reinterpret_cast<__nv_bfloat16*>(pbuf + kmajor16_offset<E>(q, t)) = pb;
                }
            } else {
                // e4m3 P: O is divided by the exact sum, as in the e4m3 forward
#pragma unroll
                for (int q4 = 0; q4 < kDecLive; q4 += 4) {
                    const uint32_t w4 = pack_e4m3x4(pv[q4], pv[q4 + 1], pv[q4 + 2], pv[q4 + 3]);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        pbuf[kmajor16_offset<E>(q4 + e, t)] = (uint8_t)(w4 >> (8 * e));
                }
#pragma unroll
                for (int q = 0; q < kDecLive; ++q) lr[q] += pv[q];
            }
            fence_proxy_async_smem();    // the P.V product reads P^T through the async proxy
            tc_fence_before();
            mbar_arrive(&bars->p_full[wg]);
        }

        // ------------------------------------------------ epilogue
        // Each warpgroup sums its columns over its 128 key threads; the others
        // hand (m_ref, l, lr) to warpgroup 0, which merges the kDecWG parts by
        // their log-sum-exp and writes the rows (thread t: head-dim index t).
        if (ok) {
            ok = mbar_wait(&bars->o_final, 0u, wd);
            ok = __all_sync(0xffffffffu, ok);
        }
        if (ok) {
            const float wl = warp_reduce_scatter8<false>(l, lane);
            const float wlr = warp_reduce_scatter8<false>(lr, lane);
            if ((lane & 3) == 0) {
                bars->sum_l[wg][wq][lane >> 2] = wl;
                bars->sum_lr[wg][wq][lane >> 2] = wlr;
            }
            mbar_arrive(&bars->sum_full[wg]);
            ok = mbar_wait(&bars->sum_full[wg], 0u, wd);
            ok = __all_sync(0xffffffffu, ok);
        }
        // the warpgroup's column totals
        auto col_l = [&](int q) {
            return bars->sum_l[wg][0][q] + bars->sum_l[wg][1][q] + bars->sum_l[wg][2][q] +
                   bars->sum_l[wg][3][q];
        };
        auto col_lr = [&](int q) {
            return bars->sum_lr[wg][0][q] + bars->sum_lr[wg][1][q] + bars->sum_lr[wg][2][q] +
                   bars->sum_lr[wg][3][q];
        };
        if (ok) {
            if (wg > 0) {
#pragma unroll
                for (int q = 0; q < kDecLive; ++q)
                    if (q == t) {
                        bars->merge_m[wg - 1][q] = m_ref[q];
                        bars->merge_l[wg - 1][q] = col_l(q);
                        bars->merge_lr[wg - 1][q] = col_lr(q);
                    }
                mbar_arrive(&bars->merge_full);
            } else {
                ok = mbar_wait(&bars->merge_full, 0u, wd);
                ok = __all_sync(0xffffffffu, ok);
            }
        }
        if (ok && wg == 0) {
            tc_fence_after();
            uint32_t o[kDecWG][kDecLive];
#pragma unroll
            for (int w = 0; w < kDecWG; ++w)
                if (n > w) tmem_ld8(tmem + lane_base + C::col_o(w), o[w]);
            tmem_wait_ld();
            const bool part = p.o_part != nullptr;
            const size_t rows = (size_t)p.B * p.H * Nq;
#pragma unroll
            for (int q = 0; q < kDecLive; ++q) {
                if (q >= cols) break;
                float mw[kDecWG], lw[kDecWG], lrw[kDecWG];
                mw[0] = m_ref[q];
                lw[0] = col_l(q);
                lrw[0] = col_lr(q);
#pragma unroll
                for (int w = 1; w < kDecWG; ++w) {
                    mw[w] = bars->merge_m[w - 1][q];
                    lw[w] = bars->merge_l[w - 1][q];
                    lrw[w] = bars->merge_lr[w - 1][q];
                }
                // weights of the parts (a part with no visible key weighs 0 and
                // its accumulator, possibly never written, is not read)
                float mm = -INFINITY;
#pragma unroll
                for (int w = 0; w < kDecWG; ++w) mm = fmaxf(mm, lw[w] > 0.f ? mw[w] : -INFINITY);
                float lsum = 0.f, lrsum = 0.f, acc = 0.f;
#pragma unroll
                for (int w = 0; w < kDecWG; ++w) {
                    const float aw = (lw[w] > 0.f) ? fast_exp2((mw[w] - mm) * c) : 0.f;
                    lsum += lw[w] * aw;
                    lrsum += lrw[w] * aw;
                    if (aw > 0.f) acc += __uint_as_float(o[w][q]) * aw;
                }
                const int g = q / Nq, rr = q - g * Nq;
                const size_t row = (size_t)(b * p.H + h0 + g) * Nq + rr;
                // a column with no visible key: O = 0, lse = -inf
                const float val = (lrsum > 0.f) ? acc * (p.o_mul / lrsum) : 0.f;
                const float row_lse = (lsum > 0.f) ? (mm * c + log2f(lsum)) * kLn2 : -INFINITY;
                if (!part) {
                    p.o[row * D + t] = __float2bfloat16_rn(val);
                    if (t == q) p.lse[row] = row_lse;
                } else {
                    const size_t prow = (size_t)s_idx * rows + row;
                    p.o_part[prow * D + t] = val;
                    if (t == q) p.lse_part[prow] = row_lse;
                }
            }
        }
    }

    // ---------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == kDecMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace fa
