// Backward pass of exact attention for sm_100a (B200).
//
// Given Q, K, V, the forward's O and lse, and dO, computes the exact
// gradients of the forward definition (the chain rule through the row
// softmax; the pages report the training speed-ups this pass makes possible,
// "FlashAttention (UR)", section "Experimental results", but give no
// backward algorithm):
//   P = exp(scale * Q K^T - lse)          (recomputed tile by tile, never stored)
//   dV = P^T dO,  dP = dO V^T,  D_i = dO_i . O_i,  dS = P * (dP - D)
//   dQ = scale * dS K,  dK = scale * dS^T Q
// As in the forward, no N x N matrix reaches device memory: each 128 x 128
// tile of S, P, dP and dS lives in tensor memory (TMEM) and feeds the next
// tensor-core product directly ("FlashAttention (UR)", sections "Tiling and
// block processing" and "Complexity and optimality": the lse is the O(N)
// statistic that makes the recomputation possible).
//
// Three kernels, no atomics (the result is deterministic):
//   fa_bwd_prep   per row: lse * log2(e) and D_i, padded to whole tiles;
//   fa_bwd_dkdv   one CTA per (batch, K/V head, 128-key tile), keys on TMEM
//                 lanes: S^T = K Q^T, dP^T = V dO^T, then P^T and dS^T (bf16)
//                 over them in TMEM and dV += P^T dO, dK += dS^T Q, over every
//                 query tile of every query head sharing the K/V head;
//   fa_bwd_dq     one CTA per (batch, head, 128-query tile), queries on
//                 lanes: S = Q K^T, dP = dO V^T, dS into TMEM, dQ += dS K.
// The dQ pass recomputes S and dP (7 tile products per tile pair instead of
// 5) in exchange for needing no cross-CTA reduction of dQ.
//
// Roles (320 threads): warps 0-7 compute -- two warpgroups, each thread owning
// one TMEM lane (tile row) and one half of that row's 128 columns, so each
// SM sub-partition runs two compute warps and one hides the other's latency;
// warp 8 issues the tcgen05 MMAs (one thread) and owns TMEM; warp 9 issues the
// TMA loads (one thread). A warpgroup writes its packed P and dS only inside
// its own 64 columns (P of columns [64 g, 64 g + 64) goes to [64 g, 64 g + 32)),
// so neither overwrites scores the other has yet to read; the MMAs address
// the K-steps of P and dS accordingly. Every mbarrier wait is bounded (the
// forward's watchdog).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace fa {

constexpr int kBwdThreads = 320;
constexpr int kBwdMmaWarp = 8;
constexpr int kBwdTmaWarp = 9;
constexpr int kBwdComputeThreads = 256;

// TMEM column of K-step kk (16 rows of the K dimension) of a packed P or dS
// operand written by the two warpgroups (see the role description above).
__device__ __forceinline__ uint32_t packed_col(uint32_t base, int kk) {
    return base + (uint32_t)((kk & 3) * 8 + (kk >> 2) * 64);
}

template <int D>
struct BwdCfg {
    static_assert(D == 64 || D == 128, "backward head dim 64 or 128");
    static constexpr int kBlocks = D / 64;               // 128-byte column blocks per row
    static constexpr int kBlockBytes = 128 * 128;        // 16 KB
    static constexpr int kTileBytes = 128 * D * 2;       // one 128-row tile
    static constexpr int kStages = (D == 128) ? 2 : 4;   // ring of streamed tile pairs
    // two fixed tiles (K, V or Q, dO) + kStages pairs of streamed tiles,
    // then the barriers, then per stage 128 lse2 and 128 D values (pass A)
    static constexpr int kSmemTiles = (2 + 2 * kStages) * kTileBytes;
    static constexpr int kSmemColVals = kSmemTiles + 1024;
    static constexpr int kSmemBytes = kSmemColVals + kStages * 1024 + 1024 /*alignment*/;
    // TMEM columns: S (P over its first 64) | dP (dS over its first 64) | acc0 | acc1
    static constexpr uint32_t kColS = 0, kColDP = 128, kColAcc0 = 256, kColAcc1 = 256 + D;
    static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
    static_assert(kStages <= 4, "barrier arrays");
};

struct BwdParams {
    __nv_bfloat16* dq;         // [B,H,N,d]
    __nv_bfloat16* dk;         // [B,H_kv,N,d]
    __nv_bfloat16* dv;         // [B,H_kv,N,d]
    const float* lse2;         // [B*H][Np]: lse * log2(e); +inf for padding rows and rows with no key
    const float* dvec;         // [B*H][Np]: D_i = dO_i . O_i; 0 for padding rows
    const int32_t* kv_len;     // [B] or nullptr
    uint32_t* dev_err;
    int B, H, H_kv, N;
    int Np;                    // N rounded up to whole 128-row tiles
    int causal;
    float scale;
    float scale_log2;          // scale * log2(e)
    uint64_t watchdog_ns;
};

struct BwdBarriers {
    uint64_t fixed_full;       // the CTA's two fixed tiles have landed
    uint64_t st_full[4];
    uint64_t st_empty[4];
    uint64_t s_full;           // S of the current item is in TMEM
    uint64_t dp_full;          // dP of the current item is in TMEM
    uint64_t p_done;           // compute phase 1 done: P written (pass A) / S read (pass B)
    uint64_t ds_done;          // compute phase 2 done: dS written (256 arrivals each)
    uint64_t acc_done;         // every accumulating MMA has completed
    uint64_t teardown;
    uint32_t tmem_base;
    int abort;
    int skip;
};
static_assert(sizeof(BwdBarriers) <= 1024, "barrier region");

// lse2 and D for every (b, h, row), padded to Np rows per head: one warp per
// row, each lane d / 32 neighbouring columns of O and dO.
template <int D>
__global__ void __launch_bounds__(256)
    fa_bwd_prep(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ d_o,
                const float* __restrict__ lse, float* __restrict__ lse2,
                float* __restrict__ dvec, int64_t BH, int N, int Np) {
    constexpr int kPer = D / 32;
    constexpr float kLog2e = 1.4426950408889634f;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= BH * Np) return;
    const int64_t bh = row / Np;
    const int i = (int)(row - bh * Np);
    float acc = 0.f, l2 = INFINITY;
    if (i < N) {
        const int64_t base = (bh * N + i) * D + lane * kPer;
#pragma unroll
        for (int c = 0; c < kPer; c += 2) {
            const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(o + base + c);
            const __nv_bfloat162 g = *reinterpret_cast<const __nv_bfloat162*>(d_o + base + c);
            const float2 fa2 = __bfloat1622float2(a), fg2 = __bfloat1622float2(g);
            acc = fmaf(fa2.x, fg2.x, acc);
            acc = fmaf(fa2.y, fg2.y, acc);
        }
        const float l = lse[bh * N + i];
        l2 = (l == -INFINITY) ? INFINITY : l * kLog2e;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
        lse2[row] = l2;
        dvec[row] = acc;
    }
}

// Tile products shared by both passes. `tmem` is the CTA's TMEM base.
template <int D>
struct BwdMma {
    using C = BwdCfg<D>;
    uint32_t tmem;
    // [128 x 128] fp32 at column dcol = A[128 x D] . B[128 x D]^T, both K-major
    // (rows of d contiguous), from descriptors of the tiles' first blocks.
    __device__ __forceinline__ void rows_by_rows(uint32_t dcol, uint64_t a, uint64_t b) const {
        constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * C::kBlockBytes + (kk & 3) * 32) >> 4);
            umma_ss(tmem + dcol, a + off, b + off, idesc, kk > 0 ? 1u : 0u);
        }
    }
    // [128 x D] fp32 at column dcol (+)= A[128 x 128] (bf16 pairs in TMEM from
    // column acol, laid out by packed_col) . B[128 x D] (a tile in shared
    // memory, MN-major: d contiguous).
    __device__ __forceinline__ void tmem_by_tile(uint32_t dcol, uint32_t acol, uint64_t b,
                                                 bool accumulate) const {
        constexpr uint32_t idesc = idesc_bf16_f32(128, D, 0, 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            umma_ts(tmem + dcol, packed_col(tmem + acol, kk),
                    b + (uint64_t)((kk * 16 * 128) >> 4), idesc, (accumulate || kk > 0) ? 1u : 0u);
    }
};

// Common set-up: barriers, TMEM, tensor-map prefetch. Returns the TMEM base.
template <int D>
__device__ __forceinline__ uint32_t bwd_setup(BwdBarriers* bars, const BwdParams& p,
                                              const CUtensorMap* m0, const CUtensorMap* m1,
                                              const CUtensorMap* m2, const CUtensorMap* m3) {
    using C = BwdCfg<D>;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        mbar_init(&bars->fixed_full, 1);
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&bars->st_full[s], 1);
            mbar_init(&bars->st_empty[s], 1);
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->dp_full, 1);
        mbar_init(&bars->p_done, kBwdComputeThreads);
        mbar_init(&bars->ds_done, kBwdComputeThreads);
        mbar_init(&bars->acc_done, 1);
        mbar_init(&bars->teardown, 1);
        bars->abort = 0;
        bars->skip = (*reinterpret_cast<volatile uint32_t*>(p.dev_err) != 0u) ? 1 : 0;
        fence_mbarrier_init();
    }
    if (warp == kBwdMmaWarp) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == kBwdTmaWarp && lane == 0) {
        prefetch_tensormap(m0);
        prefetch_tensormap(m1);
        prefetch_tensormap(m2);
        prefetch_tensormap(m3);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return bars->tmem_base;
}

// The compute warps' work on one 128 x 128 tile, in two phases so the tensor
// cores can run between them. Each thread owns one row (TMEM lane) and the 64
// columns [c0, c0 + 64) of it.
//
// Phase 1: read S (fp32) and form P = exp2(s * c - lse2) on visible entries
// (0 elsewhere) into pv; when kWriteP, also write P (bf16 pairs) to S's
// columns [c0, c0 + 32). `visible(col)` tells whether column col of the row is
// a visible (query, key) pair, consulted only when kMask (tiles on the causal
// diagonal or across kv_len; elsewhere every pair is visible and rows past N
// get P = 0 from their lse2 = +inf); `col_l2(col, l2)` gives lse2 of columns
// col..col+3 (pass A: per column; pass B: the row's own).
template <bool kWriteP, bool kMask, typename Vis, typename ColL2>
__device__ __forceinline__ void bwd_p_half(uint32_t tS, int c0, float c, Vis visible,
                                           ColL2 col_l2, float (&pv)[64]) {
    uint32_t s0[32], s1[32];
    tmem_ld32(tS + (uint32_t)c0, s0);
    tmem_ld32(tS + (uint32_t)(c0 + 32), s1);
    tmem_wait_ld();
#pragma unroll
    for (int q = 0; q < 64; q += 4) {
        float l2[4];
        col_l2(c0 + q, l2);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int qe = q + e;
            const float sv = __uint_as_float(qe < 32 ? s0[qe] : s1[qe - 32]);
            const float pe = fast_exp2(fmaf(sv, c, -l2[e]));
            pv[qe] = (!kMask || visible(c0 + qe)) ? pe : 0.f;
        }
    }
    if (kWriteP) {
        uint32_t pk[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) pk[q] = pack_bf16x2(pv[2 * q], pv[2 * q + 1]);
        tmem_st32(tS + (uint32_t)c0, pk);
    }
}

// Phase 2: read dP (fp32), form dS = P * (dP - D) and write it (bf16 pairs) to
// dP's columns [c0, c0 + 32). `col_d(col, dd)` gives D of columns col..col+3.
template <typename ColD>
__device__ __forceinline__ void bwd_ds_half(uint32_t tDP, int c0, const float (&pv)[64],
                                            ColD col_d) {
    uint32_t d0[32], d1[32];
    tmem_ld32(tDP + (uint32_t)c0, d0);
    tmem_ld32(tDP + (uint32_t)(c0 + 32), d1);
    tmem_wait_ld();
    uint32_t dk[32];
#pragma unroll
    for (int q = 0; q < 64; q += 4) {
        float dd[4];
        col_d(c0 + q, dd);
        float dsv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int qe = q + e;
            dsv[e] = pv[qe] * (__uint_as_float(qe < 32 ? d0[qe] : d1[qe - 32]) - dd[e]);
        }
        dk[q / 2] = pack_bf16x2(dsv[0], dsv[1]);
        dk[q / 2 + 1] = pack_bf16x2(dsv[2], dsv[3]);
    }
    tmem_st32(tDP + (uint32_t)c0, dk);
}

// ------------------------------------------------------------------ pass A: dK, dV
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_dkdv(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const BwdParams p) {
    using C = BwdCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sK = smem;
    uint8_t* sV = smem + C::kTileBytes;
    uint8_t* sStage = smem + 2 * C::kTileBytes;   // stage s: Q tile, then dO tile
    BwdBarriers* bars = reinterpret_cast<BwdBarriers*>(smem + C::kSmemTiles);
    float* sCol = reinterpret_cast<float*>(smem + C::kSmemColVals);   // stage s: lse2[128], D[128]

    // unit: (key tile, batch x K/V head); key tile 0 first (most query tiles when causal)
    const int BHkv = p.B * p.H_kv;
    const int jt = blockIdx.x / BHkv;
    const int bkv = blockIdx.x - jt * BHkv;
    const int b = bkv / p.H_kv;
    const int hkv = bkv - b * p.H_kv;
    const int G = p.H / p.H_kv;
    const int kv_lim = p.kv_len ? max(0, min(p.N, p.kv_len[b])) : p.N;
    const int n_qt = p.Np / 128;
    const int it0 = p.causal ? jt : 0;         // first query tile that sees this key tile
    const int nq = n_qt - it0;
    const int items = (jt * 128 < kv_lim) ? G * nq : 0;   // (query head of the group, query tile)

    const uint32_t tmem = bwd_setup<D>(bars, p, &tm_q, &tm_k, &tm_v, &tm_do);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool skip = bars->skip != 0;
    const int n_items = skip ? 0 : items;
    const Watchdog wd{&bars->abort, p.dev_err, p.watchdog_ns};

    if (warp == kBwdTmaWarp) {
        if (lane == 0 && !skip) {
            if (n_items > 0) {
                mbar_arrive_expect_tx(&bars->fixed_full, 2 * C::kTileBytes);
                for (int blk = 0; blk < C::kBlocks; ++blk) {
                    tma_load_3d(&tm_k, &bars->fixed_full, sK + blk * C::kBlockBytes, blk * 64,
                                jt * 128, bkv);
                    tma_load_3d(&tm_v, &bars->fixed_full, sV + blk * C::kBlockBytes, blk * 64,
                                jt * 128, bkv);
                }
            }
            int w = 0;
            for (; w < n_items; ++w) {
                const int slot = w % C::kStages;
                const uint32_t round = (uint32_t)(w / C::kStages);
                if (!mbar_wait(&bars->st_empty[slot], (round & 1u) ^ 1u, wd)) break;
                const int g = w / nq;
                const int it = it0 + (w - g * nq);
                const int bh = b * p.H + hkv * G + g;
                uint8_t* sq = sStage + slot * 2 * C::kTileBytes;
                mbar_arrive_expect_tx(&bars->st_full[slot], 2 * C::kTileBytes + 1024);
                for (int blk = 0; blk < C::kBlocks; ++blk) {
                    tma_load_3d(&tm_q, &bars->st_full[slot], sq + blk * C::kBlockBytes, blk * 64,
                                it * 128, bh);
                    tma_load_3d(&tm_do, &bars->st_full[slot],
                                sq + C::kTileBytes + blk * C::kBlockBytes, blk * 64, it * 128, bh);
                }
                // the tile's 128 lse2 and D values (512-byte aligned rows of the workspace)
                const size_t col0 = (size_t)bh * p.Np + (size_t)it * 128;
                bulk_load(sCol + slot * 256, p.lse2 + col0, 512, &bars->st_full[slot]);
                bulk_load(sCol + slot * 256 + 128, p.dvec + col0, 512, &bars->st_full[slot]);
            }
            // drain: every copy issued lands before the CTA exits
            if (n_items > 0) mbar_wait_drain(&bars->fixed_full, 0u, wd);
            for (int l = max(0, w - C::kStages); l < w; ++l)
                mbar_wait_drain(&bars->st_full[l % C::kStages], (uint32_t)(l / C::kStages) & 1u, wd);
        }
        __syncwarp();
    } else if (warp == kBwdMmaWarp) {
        if (lane == 0 && !skip) {
            const BwdMma<D> mma{tmem};
            const uint64_t dk0 = smem_desc_sw128(smem_u32(sK), 16, 1024);
            const uint64_t dv0 = smem_desc_sw128(smem_u32(sV), 16, 1024);
            const uint64_t st_k = smem_desc_sw128(smem_u32(sStage), 16, 1024);             // K-major
            const uint64_t st_mn = smem_desc_sw128(smem_u32(sStage), C::kBlockBytes, 1024); // MN-major
            constexpr uint64_t kTileStep = (uint64_t)(C::kTileBytes >> 4);
            // Per item w: S^T(w), dP^T(w) | P(w) -> dV(w), S^T(w+1) | dS(w) -> dK(w),
            // dP^T(w+1). S^T(w+1) overwrites P(w) after dV(w) has read it, dP^T(w+1)
            // overwrites dS(w) after dK(w) (tcgen05 MMAs of one thread run in issue
            // order), so the exponentials of item w+1 overlap dK(w) and dP^T(w+1).
            auto q_off = [&](int w) { return (uint64_t)(w % C::kStages) * 2 * kTileStep; };
            auto wait_stage = [&](int w) {
                return mbar_wait(&bars->st_full[w % C::kStages],
                                 (uint32_t)(w / C::kStages) & 1u, wd);
            };
            bool ok = true;
            if (n_items > 0) {
                ok = mbar_wait(&bars->fixed_full, 0u, wd) && wait_stage(0);
                if (ok) {
                    tc_fence_after();
                    mma.rows_by_rows(C::kColS, dk0, st_k + q_off(0));               // S^T = K Q^T
                    umma_commit(&bars->s_full);
                    mma.rows_by_rows(C::kColDP, dv0, st_k + q_off(0) + kTileStep);  // dP^T = V dO^T
                    umma_commit(&bars->dp_full);
                }
            }
            for (int w = 0; ok && w < n_items; ++w) {
                ok = mbar_wait(&bars->p_done, (uint32_t)w & 1u, wd);
                if (!ok) break;
                tc_fence_after();
                mma.tmem_by_tile(C::kColAcc0, C::kColS, st_mn + q_off(w) + kTileStep, w > 0);  // dV += P^T dO
                if (w + 1 < n_items) {
                    ok = wait_stage(w + 1);
                    if (!ok) break;
                    tc_fence_after();
                    mma.rows_by_rows(C::kColS, dk0, st_k + q_off(w + 1));
                    umma_commit(&bars->s_full);
                }
                ok = mbar_wait(&bars->ds_done, (uint32_t)w & 1u, wd);
                if (!ok) break;
                tc_fence_after();
                mma.tmem_by_tile(C::kColAcc1, C::kColDP, st_mn + q_off(w), w > 0);             // dK += dS^T Q
                umma_commit(&bars->st_empty[w % C::kStages]);
                if (w + 1 < n_items) {
                    mma.rows_by_rows(C::kColDP, dv0, st_k + q_off(w + 1) + kTileStep);
                    umma_commit(&bars->dp_full);
                }
            }
            umma_commit(&bars->acc_done);
            umma_commit(&bars->teardown);
            mbar_wait_drain(&bars->teardown, 0u, wd);
        }
        __syncwarp();
    } else if (skip) {
        // An earlier kernel on this device timed out (the status word is
        // sticky): no work, and this CTA's rows of dV (warpgroup 0) and dK
        // (warpgroup 1) read NaN rather than stale memory.
        const int jr = jt * 128 + (tid & 127);
        if (jr < p.N)
            fill_nan_bf16(((warp >> 2) != 0 ? p.dk : p.dv) + ((size_t)bkv * p.N + jr) * D, D);
    } else {
        // ====================================================== compute warpgroups
        const int row = tid & 127;                     // TMEM lane = key row in the tile
        const int c0 = (warp >> 2) * 64;               // this warpgroup's half of the columns
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + C::kColS;
        const uint32_t tDP = tmem + lane_base + C::kColDP;
        const int jr = jt * 128 + row;                 // this thread's key row
        const bool key_ok = jr < kv_lim;
        const bool tile_masked = (jt + 1) * 128 > kv_lim;   // the key tile crosses kv_len
        const float c = p.scale_log2;
        bool ok = true;
        for (int w = 0; ok && w < n_items; ++w) {
            const int slot = w % C::kStages;
            const int g = w / nq;
            const int it = it0 + (w - g * nq);
            // the stage's lse2 / D copies (their own barrier phase), then S
            ok = mbar_wait(&bars->st_full[slot], (uint32_t)(w / C::kStages) & 1u, wd);
            if (ok) ok = mbar_wait(&bars->s_full, (uint32_t)w & 1u, wd);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const float* L2 = sCol + slot * 256;
            const float* DD = L2 + 128;
            const int q0 = it * 128;
            float pv[64];
            auto vis = [&](int col) { return key_ok && (!p.causal || jr <= q0 + col); };
            auto cl2 = [&](int col, float (&l2)[4]) {
                const float4 a = *reinterpret_cast<const float4*>(L2 + col);
                l2[0] = a.x; l2[1] = a.y; l2[2] = a.z; l2[3] = a.w;
            };
            if (tile_masked || (p.causal && it == jt))
                bwd_p_half<true, true>(tS, c0, c, vis, cl2, pv);
            else
                bwd_p_half<true, false>(tS, c0, c, vis, cl2, pv);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->p_done);
            ok = mbar_wait(&bars->dp_full, (uint32_t)w & 1u, wd);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            bwd_ds_half(tDP, c0, pv, [&](int col, float (&dd)[4]) {
                const float4 d = *reinterpret_cast<const float4*>(DD + col);
                dd[0] = d.x; dd[1] = d.y; dd[2] = d.z; dd[3] = d.w;
            });
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->ds_done);
        }
        if (ok) {
            ok = mbar_wait(&bars->acc_done, 0u, wd);
            ok = __all_sync(0xffffffffu, ok);
        }
        if (ok) {
            // warpgroup 0 writes dV, warpgroup 1 writes dK (scaled)
            tc_fence_after();
            const bool is_dk = (warp >> 2) != 0;
            const uint32_t acc = tmem + lane_base + (is_dk ? C::kColAcc1 : C::kColAcc0);
            const float mul = is_dk ? p.scale : 1.f;
            const bool write = jr < p.N;
            __nv_bfloat16* dst_row = (is_dk ? p.dk : p.dv) +
                                     ((size_t)bkv * p.N + (size_t)(write ? jr : 0)) * D;
#pragma unroll 1
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t r[32];
                if (n_items > 0) {
                    tmem_ld32(acc + (uint32_t)(ch * 32), r);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int q = 0; q < 32; ++q) r[q] = 0u;
                }
                if (write) {
                    uint4* dst = reinterpret_cast<uint4*>(dst_row + ch * 32);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint4 a;
                        a.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]) * mul,
                                          __uint_as_float(r[8 * v + 1]) * mul);
                        a.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]) * mul,
                                          __uint_as_float(r[8 * v + 3]) * mul);
                        a.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]) * mul,
                                          __uint_as_float(r[8 * v + 5]) * mul);
                        a.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]) * mul,
                                          __uint_as_float(r[8 * v + 7]) * mul);
                        dst[v] = a;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kBwdMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ pass B: dQ
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_dq(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const BwdParams p) {
    using C = BwdCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sdO = smem + C::kTileBytes;
    uint8_t* sStage = smem + 2 * C::kTileBytes;   // stage s: K tile, then V tile
    BwdBarriers* bars = reinterpret_cast<BwdBarriers*>(smem + C::kSmemTiles);

    // unit: (query tile, batch x head); the last query tiles (most key tiles) first
    const int BH = p.B * p.H;
    const int n_qt = p.Np / 128;
    const int it = n_qt - 1 - (int)(blockIdx.x / BH);
    const int bh = blockIdx.x - (blockIdx.x / BH) * BH;
    const int b = bh / p.H;
    const int h = bh - b * p.H;
    const int bkv = b * p.H_kv + h / (p.H / p.H_kv);
    const int kv_lim = p.kv_len ? max(0, min(p.N, p.kv_len[b])) : p.N;
    int n_kt = (kv_lim + 127) / 128;
    if (p.causal) n_kt = min(n_kt, it + 1);

    const uint32_t tmem = bwd_setup<D>(bars, p, &tm_q, &tm_k, &tm_v, &tm_do);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool skip = bars->skip != 0;
    const int n_items = skip ? 0 : n_kt;
    const Watchdog wd{&bars->abort, p.dev_err, p.watchdog_ns};

    if (warp == kBwdTmaWarp) {
        if (lane == 0 && !skip) {
            if (n_items > 0) {
                mbar_arrive_expect_tx(&bars->fixed_full, 2 * C::kTileBytes);
                for (int blk = 0; blk < C::kBlocks; ++blk) {
                    tma_load_3d(&tm_q, &bars->fixed_full, sQ + blk * C::kBlockBytes, blk * 64,
                                it * 128, bh);
                    tma_load_3d(&tm_do, &bars->fixed_full, sdO + blk * C::kBlockBytes, blk * 64,
                                it * 128, bh);
                }
            }
            int w = 0;
            for (; w < n_items; ++w) {
                const int slot = w % C::kStages;
                const uint32_t round = (uint32_t)(w / C::kStages);
                if (!mbar_wait(&bars->st_empty[slot], (round & 1u) ^ 1u, wd)) break;
                uint8_t* sk = sStage + slot * 2 * C::kTileBytes;
                mbar_arrive_expect_tx(&bars->st_full[slot], 2 * C::kTileBytes);
                for (int blk = 0; blk < C::kBlocks; ++blk) {
                    tma_load_3d(&tm_k, &bars->st_full[slot], sk + blk * C::kBlockBytes, blk * 64,
                                w * 128, bkv);
                    tma_load_3d(&tm_v, &bars->st_full[slot],
                                sk + C::kTileBytes + blk * C::kBlockBytes, blk * 64, w * 128, bkv);
                }
            }
            if (n_items > 0) mbar_wait_drain(&bars->fixed_full, 0u, wd);
            for (int l = max(0, w - C::kStages); l < w; ++l)
                mbar_wait_drain(&bars->st_full[l % C::kStages], (uint32_t)(l / C::kStages) & 1u, wd);
        }
        __syncwarp();
    } else if (warp == kBwdMmaWarp) {
        if (lane == 0 && !skip) {
            const BwdMma<D> mma{tmem};
            const uint64_t dq0 = smem_desc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t ddo0 = smem_desc_sw128(smem_u32(sdO), 16, 1024);
            const uint64_t st_k = smem_desc_sw128(smem_u32(sStage), 16, 1024);
            const uint64_t st_mn = smem_desc_sw128(smem_u32(sStage), C::kBlockBytes, 1024);
            constexpr uint64_t kTileStep = (uint64_t)(C::kTileBytes >> 4);
            // Per item w: dP(w) | S read -> S(w+1) | dS(w) -> dQ(w), dP(w+1). S(w+1)
            // is computed while the compute warps work on item w (they hold S(w)
            // in registers once they signal p_done); dP(w+1) overwrites dS(w)
            // after dQ(w) has read it (issue order).
            auto k_off = [&](int w) { return (uint64_t)(w % C::kStages) * 2 * kTileStep; };
            auto wait_stage = [&](int w) {
                return mbar_wait(&bars->st_full[w % C::kStages],
                                 (uint32_t)(w / C::kStages) & 1u, wd);
            };
            bool ok = true;
            if (n_items > 0) {
                ok = mbar_wait(&bars->fixed_full, 0u, wd) && wait_stage(0);
                if (ok) {
                    tc_fence_after();
                    mma.rows_by_rows(C::kColS, dq0, st_k + k_off(0));                // S  = Q K^T
                    umma_commit(&bars->s_full);
                    mma.rows_by_rows(C::kColDP, ddo0, st_k + k_off(0) + kTileStep);  // dP = dO V^T
                    umma_commit(&bars->dp_full);
                }
            }
            for (int w = 0; ok && w < n_items; ++w) {
                if (w + 1 < n_items) {
                    ok = mbar_wait(&bars->p_done, (uint32_t)w & 1u, wd) && wait_stage(w + 1);
                    if (!ok) break;
                    tc_fence_after();
                    mma.rows_by_rows(C::kColS, dq0, st_k + k_off(w + 1));
                    umma_commit(&bars->s_full);
                }
                ok = mbar_wait(&bars->ds_done, (uint32_t)w & 1u, wd);
                if (!ok) break;
                tc_fence_after();
                mma.tmem_by_tile(C::kColAcc0, C::kColDP, st_mn + k_off(w), w > 0);   // dQ += dS K
                umma_commit(&bars->st_empty[w % C::kStages]);
                if (w + 1 < n_items) {
                    mma.rows_by_rows(C::kColDP, ddo0, st_k + k_off(w + 1) + kTileStep);
                    umma_commit(&bars->dp_full);
                }
            }
            umma_commit(&bars->acc_done);
            umma_commit(&bars->teardown);
            mbar_wait_drain(&bars->teardown, 0u, wd);
        }
        __syncwarp();
    } else if (skip) {
        // skipped launch (sticky status word): this CTA's half-rows of dQ read NaN
        const int i = it * 128 + (tid & 127);
        if (i < p.N)
            fill_nan_bf16(p.dq + ((size_t)bh * p.N + i) * D + (warp >> 2) * (D / 2), D / 2);
    } else {
        const int row = tid & 127;                     // TMEM lane = query row in the tile
        const int c0 = (warp >> 2) * 64;               // this warpgroup's half of the columns
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + C::kColS;
        const uint32_t tDP = tmem + lane_base + C::kColDP;
        const int i = it * 128 + row;                  // this thread's query row
        const size_t ridx = (size_t)bh * p.Np + (size_t)i;
        const float l2 = p.lse2[ridx];
        const float dd = p.dvec[ridx];
        const float c = p.scale_log2;
        bool ok = true;
        for (int w = 0; ok && w < n_items; ++w) {
            ok = mbar_wait(&bars->s_full, (uint32_t)w & 1u, wd);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const int k0 = w * 128;
            float pv[64];
            auto vis = [&](int col) { return k0 + col < kv_lim && (!p.causal || k0 + col <= i); };
            auto cl2 = [&](int, float (&l2v)[4]) {
#pragma unroll
                for (int e = 0; e < 4; ++e) l2v[e] = l2;
            };
            if (k0 + 128 > kv_lim || (p.causal && w == it))
                bwd_p_half<false, true>(tS, c0, c, vis, cl2, pv);
            else
                bwd_p_half<false, false>(tS, c0, c, vis, cl2, pv);
            tc_fence_before();
            mbar_arrive(&bars->p_done);          // S(w) is in registers: S(w+1) may overwrite it
            ok = mbar_wait(&bars->dp_full, (uint32_t)w & 1u, wd);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            bwd_ds_half(tDP, c0, pv, [&](int, float (&ddv)[4]) {
#pragma unroll
                for (int e = 0; e < 4; ++e) ddv[e] = dd;
            });
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->ds_done);
        }
        if (ok) {
            ok = mbar_wait(&bars->acc_done, 0u, wd);
            ok = __all_sync(0xffffffffu, ok);
        }
        if (ok) {
            // each warpgroup writes half of the row's d columns of dQ (scaled)
            tc_fence_after();
            const bool write = i < p.N;
            __nv_bfloat16* dqrow = p.dq + ((size_t)bh * p.N + (size_t)(write ? i : 0)) * D;
            const int ch0 = (warp >> 2) * (D / 64);
#pragma unroll 1
            for (int ch = ch0; ch < ch0 + D / 64; ++ch) {
                uint32_t r[32];
                if (n_items > 0) {
                    tmem_ld32(tmem + lane_base + C::kColAcc0 + (uint32_t)(ch * 32), r);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int q = 0; q < 32; ++q) r[q] = 0u;
                }
                if (write) {
                    uint4* dst = reinterpret_cast<uint4*>(dqrow + ch * 32);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint4 a;
                        a.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]) * p.scale,
                                          __uint_as_float(r[8 * v + 1]) * p.scale);
                        a.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]) * p.scale,
                                          __uint_as_float(r[8 * v + 3]) * p.scale);
                        a.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]) * p.scale,
                                          __uint_as_float(r[8 * v + 5]) * p.scale);
                        a.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]) * p.scale,
                                          __uint_as_float(r[8 * v + 7]) * p.scale);
                        dst[v] = a;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kBwdMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace fa
