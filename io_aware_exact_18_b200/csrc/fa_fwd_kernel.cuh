// Fused exact attention forward for sm_100a (B200).
//
// Computes O = softmax(scale * Q K^T + mask) V and lse = ln sum_j exp(s_ij)
// for bf16 (or e4m3, with per-tensor descales) Q, K, V laid out [B, H, N, d]
// (d innermost), accumulating in fp32.
// The N x N score matrix never leaves the SM: each 128 x 128 score tile lives
// in tensor memory (TMEM), is turned into probabilities there, and feeds the
// P.V product directly ("FlashAttention (UR)", sections "Tiling and block
// processing" and "Fusing operations into one CUDA kernel").
//
// Softmax is evaluated online, one key tile at a time, with a running row
// maximum m and running sum of exponentials l ("FlashAttention (UR)", section
// "Online softmax"). Exponentials use base 2 with the scale folded into one
// FFMA per score, and the division by l is deferred to the epilogue, which
// trims the non-matmul work that "FlashAttention-2 (HI)" section 1 targets.
// The reference maximum m_ref is set by a row's first key tile and is raised
// only rarely, so the per-tile rescale of the online softmax becomes an
// exception. With two query tiles, and for e4m3 inputs, a tile's row maximum
// is taken before its exponentials and moves m_ref only when it exceeds it by
// more than 64 in log2 units (8 for e4m3 P), after O and l are rescaled; with
// one bf16 query tile each tile is exponentiated against m_ref straight away
// and the rare tile whose probabilities would sum past 2^64 is redone after the
// rescale. Both O and l
// share the reference, so the final O / l is unchanged by this choice (the
// ratio is exact), and every probability stays at most 2^64, far inside the
// fp32 and bf16 range.
//
// Work partitioning ("FlashAttention-2 (HI)", sections 2 and 3). A work unit
// is one (batch, head, pair of 128-row query tiles) -- one tile at d = 256 --
// and the grid has one CTA per unit, so one long head still spreads over every
// SM. The general instantiation (kGen) adds what decoding against a key-value
// cache needs ("FlashAttention (UR)", section "Specialised solutions"): fewer
// query rows than keys (row i at key position i + Nk - Nq), the query heads of
// a K/V group packed into one tile so each K/V tile serves all of them, and
// units that take one range of key tiles each, writing a normalised partial O
// and lse for a separate merge (split-KV). Units are numbered in
// launch order: heads in groups whose K/V fit in L2 together, and within a
// group the query-tile pairs heaviest first (the last pairs, for causal
// masking) across the group's heads. CTAs are persistent: near the end of
// its current unit a running CTA asks the hardware (cluster launch control)
// to cancel the next CTA that has not started and processes that CTA's unit
// instead, so the hardware hands out units in launch order to whichever SM
// frees up first, the per-CTA set-up is paid once per SM, and one unit's
// epilogue overlaps the next unit's loads and first Q.K^T.
//
// Grouped / multi-query attention (the FlashAttention-2 extension to MQA,
// "FlashAttention (UR)", section "FlashAttention-2 (2023)"): K and V may have
// H_kv heads shared by groups of H / H_kv query heads; a unit's K/V tiles come
// from its query head's group head, and neighbouring query heads (same group)
// run next to each other so the shared K/V stays in L2.
//
// Instantiations fa_fwd_sm100<D, QT, kGen, E>: head dim D; QT query tiles per
// unit (2 at d <= 128 for square attention; 1 with S double-buffered at
// d = 256 and in the general kernel); kGen the general (split-KV) form; E the
// element bytes of Q, K, V (2: bf16, 1: e4m3 with kind::f8f6f4 products).
//
// Roles inside a CTA (320 threads):
//   warps 0-3   softmax for query tile 0 (thread r owns row r = TMEM lane r)
//   warps 4-7   softmax for query tile 1 (QT = 2), or for the odd key tiles of
//               the one query tile (general kernel at d <= 128), or idle
//   warp  8     issues tcgen05 MMAs (one thread) and owns the TMEM allocation
//   warp  9     issues TMA loads and the unit requests (one thread)
// With one thread per row no cross-thread reduction is needed for the row
// max and row sum. The two softmax warpgroups ping-pong: while one works on
// its score tile the tensor cores run the other tile's P.V and next Q.K^T.
//
// TMEM (512 columns x 128 lanes of 32 bit), QT = 2:
//   [0,128)    S0 (fp32 scores of tile 0); P0 (bf16 pairs) overwrites [0,64)
//   [128,256)  S1 / P1
//   [256,256+d)      O0 accumulator (fp32)
//   [256+d,256+2d)   O1 accumulator
// QT = 1: Sa | Sb (alternate key tiles) | O, or | O0 | O1 in the general kernel
// at d <= 128, where each softmax warpgroup keeps its own accumulator and the
// epilogue merges the two by log-sum-exp. e4m3 P takes 32 columns.
// Shared memory: the Q tiles and a ring of K/V slots, each a 128-row tile
// stored as 128-byte column blocks of 128 rows in the 128-byte swizzled layout
// that TMA writes and tcgen05 descriptors read; then the barriers.
//
// Synchronisation (mbarriers; every wait is bounded). Each barrier's phases
// are counted per role across units; per unit and tile there is exactly one
// q_full, q_empty and o_empty phase, max(n_t, 1) o_done phases and n_t s_full
// and p_full phases, where n_t is the tile's number of key tiles (an idle
// tile still takes part in its once-per-unit hand-offs), so every role can
// compute every phase index and no barrier runs two phases ahead of a waiter.
// (With one query tile and one accumulator the epilogue could find o_done one
// phase short of, or one phase past, the unit's last; the second-last phase is
// therefore waited for inside the last tile, before its P is handed over.)
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace fa {

constexpr int kTile = 128;         // rows per query tile and keys per KV tile
constexpr int kThreads = 320;      // 2 softmax warpgroups + MMA warp + TMA warp
constexpr int kMmaWarp = 8;
constexpr int kTmaWarp = 9;
constexpr float kLn2 = 0.69314718055994530942f;

// Per head dimension and query tiles per unit. QT = 2 (square attention at
// d = 64, 128): a unit is two query tiles, each with one S buffer (TMEM:
// S0 | S1 | O0 | O1), and the two softmax warpgroups ping-pong. QT = 1: a unit
// is one query tile whose S is double-buffered (TMEM: Sa | Sb | O): the tensor
// cores compute the next key tile's scores while the softmax works on the
// current ones. d = 256 needs it (O alone takes 256 TMEM columns); the
// split-KV kernel uses it at every d, since a short query block gives the
// second tile of a pair nothing to do.
// E is the element size of Q, K and V: 2 (bf16) or 1 (e4m3). Tiles are stored
// in column blocks of swizzle rows: 128-byte rows with the 128-byte swizzle,
// or, when a whole row is 64 bytes (e4m3 at d = 64), 64-byte rows with the
// 64-byte swizzle.
template <int D, int QT, int E = 2>
struct Cfg {
    static_assert(D == 64 || D == 128 || D == 256, "head dim 64, 128 or 256");
    static_assert(QT == 1 || (QT == 2 && D <= 128), "two query tiles need d <= 128");
    static_assert(E == 1 || E == 2, "bf16 or e4m3");
    static constexpr int kQT = QT;                        // query tiles per unit
    static constexpr int kRowBytes = D * E < 128 ? D * E : 128;   // bytes of one swizzle row
    static constexpr int kSwizzle = kRowBytes == 128 ? 2 : 4;     // descriptor code: 128- / 64-byte
    static constexpr int kBlocks = D * E / kRowBytes;     // column blocks per row
    static constexpr int kBlockElems = kRowBytes / E;     // columns of one block
    static constexpr int kBlockBytes = kTile * kRowBytes; // 16 KB (8 KB with 64-byte rows)
    static constexpr int kAtomBytes = 8 * kRowBytes;      // 8 rows: the swizzle pattern's period
    static constexpr int kStepsPerBlock = kRowBytes / 32; // 32-byte K-steps in one row
    static constexpr int kTileBytes = kTile * D * E;      // one Q/K/V tile
    static constexpr int kSlots =                         // K/V ring depth
        (D * E == 256) ? (QT == 2 ? 4 : 5) : (D * E == 512) ? 2 : 8;   // 8 at 64 or 128 bytes
    static constexpr int kSmemTiles = (kQT + kSlots) * kTileBytes;
    static constexpr int kSmemBytes = kSmemTiles + 1024 /*alignment*/ + 4096 /*barriers*/;
    static constexpr uint32_t kTmemCols = 512;
    // S buffer b (a query tile's, or with one tile the buffer of key-tile parity b)
    __device__ static constexpr uint32_t col_s(int b) { return (uint32_t)(b * 128); }
    __device__ static constexpr uint32_t col_o(int t) { return 256u + (uint32_t)(t * D); }
    static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
    static_assert(kSlots <= 8, "K/V ring barriers");
    static_assert(256 + kQT * D <= (int)kTmemCols, "TMEM columns");
};

struct FwdParams {
    __nv_bfloat16* o;          // [B,H,Nq,d]
    float* lse;                // [B,H,Nq]
    float* o_part;             // split-KV partials [splits][B*H][Nq][d] fp32, or nullptr
    float* lse_part;           // [splits][B*H][Nq]
    const int32_t* kv_len;     // [B] or nullptr
    uint32_t* dev_err;         // status word
    int B, H;
    int H_kv;                  // K/V heads; query head h reads K/V head h / (H / H_kv)
    int Nq, Nk;                // query rows, keys
    int q_off;                 // causal offset: query row i stands at key position i + q_off
    int G;                     // query heads packed into one tile (they share a K/V head)
    int nq_blk;                // query rows per head in one tile (G * nq_blk <= 128)
    int n_rb;                  // row blocks per head: ceil(Nq / nq_blk)
    int splits;                // key ranges per row block (1 = no split)
    int n_units;               // units per head block: ceil(n_rb / query tiles per unit) * splits
    int group_heads;           // head blocks per L2 group (launch order)
    int causal;
    float scale_log2;          // scale * log2(e) (times the Q and K descales for e4m3 inputs)
    float o_mul;               // 1, or the V descale for e4m3 inputs
    uint64_t watchdog_ns;
};

struct SmemBarriers {
    uint64_t q_full[2];
    uint64_t q_empty[2];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t o_done[2];
    uint64_t o_empty[2];
    uint64_t unit_full[2];
    uint64_t unit_empty[2];
    uint64_t clc_bar[2];
    uint64_t teardown;
    uint64_t kv_full[8];
    uint64_t kv_empty[8];
    uint64_t merge_full[2];    // two-accumulator mode: warpgroup 1's (m, l) per row, by unit parity
    float merge_m[2][kTile];
    float merge_l[2][kTile];   // exact row sum
    float merge_lr[2][kTile];  // sum of the rounded probabilities
    uint4 clc_resp[2];         // 16-byte aligned (offset is a multiple of 16)
    int unit_id[2];
    uint32_t tmem_base;
    int abort;
    int skip;
};
static_assert(sizeof(SmemBarriers) <= 4096, "barrier region");
static_assert(offsetof(SmemBarriers, clc_resp) % 16 == 0, "CLC response alignment");

// One work unit, decoded from its launch-order index. A tile's 128 rows hold
// G heads x nq_blk query rows (row r: head h0 + r / nq_blk, query row
// q_first + r % nq_blk); with G = 1, nq_blk = 128 a tile is 128 rows of one head.
struct Unit {
    int b, h0;                 // batch, first query head of the tile
    int bkv;                   // K/V head row in the [B*H_kv, Nk, d] view
    int rb0;                   // row block of query tile 0 (tile t: rb0 + t)
    int s, kt0;                // split index and its first key tile
    int kv_lim;
    int n[2];                  // key tiles each query tile visits (0 = idle tile)
    int n_max;
};

// Tile-shape parameters: read from FwdParams by the general (split-KV,
// packed-heads, Nq <= Nk) kernel, compile-time constants for square attention
// (one head of 128 rows per tile, one key range, Nq == Nk).
template <bool kGen>
struct Shape {
    int G, nq_blk, splits, q_off, Nq;
    __device__ __forceinline__ explicit Shape(const FwdParams& p)
        : G(kGen ? p.G : 1),
          nq_blk(kGen ? p.nq_blk : kTile),
          splits(kGen ? p.splits : 1),
          q_off(kGen ? p.q_off : 0),
          Nq(kGen ? p.Nq : p.Nk) {}
};

// Key tiles a row block must visit: keys below its last row's causal limit
// (key position of the row + 1) and below kv_lim.
template <bool kGen>
__device__ __forceinline__ int kv_tiles_for(int rb, const FwdParams& p, const Shape<kGen>& sh,
                                            int kv_lim) {
    const int q_first = rb * sh.nq_blk;
    if (q_first >= sh.Nq) return 0;
    int lim = kv_lim;
    if (p.causal) lim = min(lim, min(q_first + sh.nq_blk, sh.Nq) + sh.q_off);
    return (max(lim, 0) + kTile - 1) / kTile;
}

template <int QT, bool kGen>
__device__ __forceinline__ Unit decode_unit(int id, const FwdParams& p) {
    const Shape<kGen> sh(p);
    Unit u;
    const int hpb = p.H / sh.G;                // head blocks per batch
    const int BHB = p.B * hpb;
    const int per_group = p.group_heads * p.n_units;
    const int grp = id / per_group;
    const int in_grp = id - grp * per_group;
    const int heads_here = min(p.group_heads, BHB - grp * p.group_heads);
    const int ps = p.n_units - 1 - in_grp / heads_here;   // (row-block pair, split), heaviest first
    const int hb = grp * p.group_heads + in_grp % heads_here;
    u.b = hb / hpb;
    u.h0 = (hb - u.b * hpb) * sh.G;
    u.bkv = u.b * p.H_kv + u.h0 / (p.H / p.H_kv);
    const int pair = ps / sh.splits;
    u.s = ps - pair * sh.splits;
    u.rb0 = pair * QT;
    u.kv_lim = p.Nk;
    if (p.kv_len != nullptr) u.kv_lim = max(0, min(p.Nk, p.kv_len[u.b]));
    // split s takes key tiles [s * nkb / splits, (s + 1) * nkb / splits)
    const int nkb = (u.kv_lim + kTile - 1) / kTile;
    u.kt0 = kGen ? (int)((long long)u.s * nkb / sh.splits) : 0;
    const int kt1 = kGen ? (int)((long long)(u.s + 1) * nkb / sh.splits) : nkb;
    u.n[0] = max(0, min(kv_tiles_for(u.rb0, p, sh, u.kv_lim), kt1) - u.kt0);
    u.n[1] = (QT == 2) ? max(0, min(kv_tiles_for(u.rb0 + 1, p, sh, u.kv_lim), kt1) - u.kt0) : 0;
    u.n_max = max(u.n[0], u.n[1]);
    return u;
}

// Fill the O rows and lse entries of unit `id` with NaN (all threads of the
// CTA take part): the output of a launch that skipped its work because the
// device status word was already set.
template <int D, int QT, bool kGen>
__device__ void poison_unit(int id, const FwdParams& p, int tid, int nthreads) {
    const Shape<kGen> sh(p);
    const Unit u = decode_unit<QT, kGen>(id, p);
    for (int e = tid; e < QT * kTile; e += nthreads) {
        const int t = e / kTile, r = e - (e / kTile) * kTile;
        const int g = r / sh.nq_blk;
        const int i = (u.rb0 + t) * sh.nq_blk + (r - g * sh.nq_blk);
        if (g >= sh.G || i >= sh.Nq) continue;
        const size_t row = (size_t)(u.b * p.H + u.h0 + g) * sh.Nq + i;
        fill_nan_bf16(p.o + row * D, D);
        p.lse[row] = __int_as_float(0x7FC00000);
    }
}

// Row maximum of a 128-score row held in registers: 64 three-input maxima in
// four independent chains.
__device__ __forceinline__ float row_max(const float (&s)[kTile]) {
    static_assert(kTile == 128, "the chains below cover 128 scores");
    float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
    for (int q = 4; q < 116 + 8; q += 8) {
        mx0 = fmax3(mx0, s[q], s[q + 1]);
        mx1 = fmax3(mx1, s[q + 2], s[q + 3]);
        mx2 = fmax3(mx2, s[q + 4], s[q + 5]);
        mx3 = fmax3(mx3, s[q + 6], s[q + 7]);
    }
    mx0 = fmax3(mx0, s[124], s[125]);
    mx1 = fmax3(mx1, s[126], s[127]);
    return fmaxf(fmax3(mx0, mx1, mx2), mx3);
}

// P = exp2(s*c - mc), rounded to bf16 pairs (E = 2: 64 TMEM columns) or to
// e4m3 quadruples (E = 1: 32 columns) and written to TMEM at tP (warp-wide
// stores, 16 columns at a time). Returns two row sums: x, of the fp32
// probabilities (the exact sum, for lse), and y, of the values as rounded for
// the P.V product (bf16 P; for e4m3 P, y = x). O divided by y is a convex
// combination of V rows whatever the rounding, so a row dominated by one key
// returns that key's V row to within the output rounding, where O divided by x
// would carry the dominant probability's rounding (up to 2^-8 of |V|): the
// reference maximum of a row need not be its true maximum, so its largest
// probability need not be exactly 1. The scale-subtract and the exact sum
// take one packed (two-lane fp32) instruction per pair of scores.
template <int E>
__device__ __forceinline__ float2 exp_tile(const float (&s)[kTile], float c, float mc,
                                           uint32_t tP) {
    if constexpr (E == 2) {
        float rs0 = 0.f, rs1 = 0.f;
        float2 sum = make_float2(0.f, 0.f);
        const float2 c2 = make_float2(c, c), nmc2 = make_float2(-mc, -mc);
#pragma unroll
        for (int ch = 0; ch < kTile / 32; ++ch) {
            uint32_t packed[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const float2 x = __ffma2_rn(
                    make_float2(s[ch * 32 + 2 * q], s[ch * 32 + 2 * q + 1]), c2, nmc2);
                const float p0 = fast_exp2(x.x);
                const float p1 = fast_exp2(x.y);
                sum = __fadd2_rn(sum, make_float2(p0, p1));
                packed[q] = pack_bf16x2(p0, p1);
                rs0 = add_bf16_lo(packed[q], rs0);
                rs1 = add_bf16_hi(packed[q], rs1);
            }
            tmem_st16(tP + (uint32_t)(ch * 16), packed);
        }
        return make_float2(sum.x + sum.y, rs0 + rs1);
    } else {
        float2 sum = make_float2(0.f, 0.f);
        const float2 c2 = make_float2(c, c), nmc2 = make_float2(-mc, -mc);
#pragma unroll
        for (int ch = 0; ch < kTile / 64; ++ch) {
            uint32_t packed[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const float* sq = &s[ch * 64 + 4 * q];
                const float2 x0 = __ffma2_rn(make_float2(sq[0], sq[1]), c2, nmc2);
                const float2 x1 = __ffma2_rn(make_float2(sq[2], sq[3]), c2, nmc2);
                const float p0 = fast_exp2(x0.x), p1 = fast_exp2(x0.y);
                const float p2 = fast_exp2(x1.x), p3 = fast_exp2(x1.y);
                sum = __fadd2_rn(sum, __fadd2_rn(make_float2(p0, p1), make_float2(p2, p3)));
                packed[q] = pack_e4m3x4(p0, p1, p2, p3);
            }
            tmem_st16(tP + (uint32_t)(ch * 16), packed);
        }
        return make_float2(sum.x + sum.y, sum.x + sum.y);
    }
}

// Max-first rule (two query tiles, and e4m3 at any tile count): a row's
// reference maximum is raised only when a tile's maximum exceeds it by more
// than this (log2 units), so every probability is at most 2^64 for bf16 P, or
// 2^8 for e4m3 P, whose largest finite value is 448.
template <int E>
__device__ __forceinline__ constexpr float rescale_log2() {
    return E == 2 ? 64.0f : 8.0f;
}

// Exponentiate-first rule (one bf16 query tile): the largest row sum of a
// tile's probabilities, computed against the reference, before the row takes
// its true maximum and the tile is redone (2^64).
template <int E>
__device__ __forceinline__ constexpr float redo_tile_sum() {
    static_assert(E == 2, "e4m3 takes the max-first rule");
    return 18446744073709551616.0f;
}

// O (d columns of this thread's TMEM lane) *= alpha, kCols columns at a time.
// With a tile's scores live (two query tiles) 16 columns in a rolled loop keep
// the scores in registers; otherwise 32 columns fully unrolled (a rolled loop
// there measured slower even though it rarely runs).
template <int D, int kCols>
__device__ __forceinline__ void rescale_o(uint32_t tO, float alpha) {
    static_assert(kCols == 16 || kCols == 32, "TMEM load width");
    if constexpr (kCols == 16) {
#pragma unroll 1
        for (int ch = 0; ch < D / 16; ++ch) {
            uint32_t r[16];
            tmem_ld16(tO + (uint32_t)(ch * 16), r);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 16; ++q) r[q] = __float_as_uint(__uint_as_float(r[q]) * alpha);
            tmem_st16(tO + (uint32_t)(ch * 16), r);
        }
    } else {
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t r[32];
            tmem_ld32(tO + (uint32_t)(ch * 32), r);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 32; ++q) r[q] = __float_as_uint(__uint_as_float(r[q]) * alpha);
            tmem_st32(tO + (uint32_t)(ch * 32), r);
        }
    }
}

template <int D, int QT, bool kGen, int E = 2>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = Cfg<D, QT, E>;
    const Shape<kGen> sh(p);
    // Two-accumulator mode (the general kernel at d <= 128): the one query tile's
    // key tiles alternate between the two softmax warpgroups, each with its own
    // reference maximum, running sum and O accumulator (TMEM: Sa | Sb | O0 | O1);
    // the epilogue merges the two halves by their log-sum-exp, as the split-KV
    // merge does. It keeps both warpgroups busy when a unit has one live tile.
    constexpr bool kDual = kGen && QT == 1 && D <= 128;
    constexpr int kSoftmaxWarps = 4 * (kDual ? 2 : QT);
    constexpr int kConsumers = 1 + kSoftmaxWarps;   // MMA thread + one lane per softmax warp
    // Reference-maximum rule (see the softmax loop): fixed before the
    // exponentials with two query tiles, where it measured faster; exponentiate
    // first and redo the rare overshooting tile with one bf16 tile (S
    // double-buffered, the row maximum pass would sit on the critical path).
    // e4m3 P allows an overshoot of 2^8 only, so a redo would not be rare: e4m3
    // takes the max-first rule at every tile count.
    constexpr bool kMaxFirst = QT == 2 || E == 1;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // Q tiles (kQT of them), then the K/V ring, then the barriers.
    uint8_t* sQ[2] = {smem, smem + C::kTileBytes};   // sQ[1] is used only when kQT == 2
    uint8_t* sKV = smem + C::kQT * C::kTileBytes;
    SmemBarriers* bars = reinterpret_cast<SmemBarriers*>(smem + C::kSmemTiles);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // ---------------------------------------------------------- setup
    if (tid == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars->q_full[t], 1);
            mbar_init(&bars->q_empty[t], 1);
            mbar_init(&bars->s_full[t], 1);
            mbar_init(&bars->p_full[t], kTile);
            mbar_init(&bars->o_done[t], 1);
            mbar_init(&bars->o_empty[t], kTile);
            mbar_init(&bars->unit_full[t], 1);
            mbar_init(&bars->unit_empty[t], kConsumers);
            mbar_init(&bars->merge_full[t], kTile);
            mbar_init(&bars->clc_bar[t], 1);
        }
        mbar_init(&bars->teardown, 1);
        for (int s = 0; s < C::kSlots; ++s) {
            mbar_init(&bars->kv_full[s], 1);
            mbar_init(&bars->kv_empty[s], 1);
        }
        bars->abort = 0;
        bars->skip = (*reinterpret_cast<volatile uint32_t*>(p.dev_err) != 0u) ? 1 : 0;
        fence_mbarrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&bars->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == kTmaWarp && lane == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const bool skip = bars->skip != 0;
    const Watchdog wd{&bars->abort, p.dev_err, p.watchdog_ns};
    if (skip && (!kGen || p.o_part == nullptr)) {
        // An earlier kernel on this device timed out (the status word is
        // sticky): this launch does no attention work (the unit hand-out below
        // publishes no unit, so every CTA of the grid runs just this) and each
        // CTA fills its own unit's O and lse with NaN, so a caller who does not
        // read the status word finds no stale values. Split-KV partials are
        // left alone: the merge kernel checks the same word.
        poison_unit<D, C::kQT, kGen>((int)blockIdx.x, p, tid, kThreads);
    }

    if (warp == kTmaWarp) {
        // ====================================================== TMA producer + unit requests
        if (lane == 0) {
            const uint64_t pol_kv = policy_evict_last();
            const uint64_t pol_q = policy_evict_first();
            const uint32_t q_bytes = (uint32_t)(C::kBlocks * sh.G * sh.nq_blk * C::kRowBytes);
            int id = skip ? -1 : (int)blockIdx.x;
            int L = 0;                 // K/V loads issued (K_j and V_j of every unit, in order)
            int k = 0;                 // units published
            int clc_pending = -1;      // slot of an unanswered cancel request
            uint32_t clc_pending_parity = 0;
            int q_unit[2] = {-1, -1};  // last unit whose Q tile t was requested
            bool ok = true;
            // jj-th K/V load of unit u, in the order the MMAs consume them:
            // two query tiles: K0 V0 K1 V1 ...; one query tile (S double-
            // buffered): K0 K1 V0 K2 V1 K3 V2 ... V(n-2) V(n-1).
            auto load_kv = [&](const Unit& u, int jj) -> bool {
                bool is_v;
                int tile;
                if (C::kQT == 2) {
                    is_v = (jj & 1) != 0;
                    tile = jj >> 1;
                } else {
                    const int n = u.n[0];
                    const int kfirst = min(2, n);
                    const int paired = 2 * max(0, n - 2);
                    const int q = jj - kfirst;
                    if (q < 0) {
                        is_v = false;
                        tile = jj;
                    } else if (q < paired) {
                        is_v = (q & 1) == 0;
                        tile = is_v ? q / 2 : q / 2 + 2;
                    } else {
                        is_v = true;
                        tile = max(0, n - 2) + (q - paired);
                    }
                }
                const int slot = L % C::kSlots;
                const uint32_t round = (uint32_t)(L / C::kSlots);
                if (!mbar_wait(&bars->kv_empty[slot], (round & 1u) ^ 1u, wd)) return false;
                const CUtensorMap* map = is_v ? &tm_v : &tm_k;
                uint8_t* dst = sKV + slot * C::kTileBytes;
                mbar_arrive_expect_tx(&bars->kv_full[slot], C::kTileBytes);
                for (int blk = 0; blk < C::kBlocks; ++blk)
                    tma_load_3d_hint(map, &bars->kv_full[slot], dst + blk * C::kBlockBytes,
                                     blk * C::kBlockElems, (u.kt0 + tile) * kTile, u.bkv,
                                     pol_kv);
                ++L;
                return true;
            };
            for (;; ++k) {
                const int us = k & 1;
                ok = mbar_wait(&bars->unit_empty[us], (uint32_t)((k >> 1) & 1) ^ 1u, wd);
                if (!ok) break;
                bars->unit_id[us] = id;
                mbar_arrive(&bars->unit_full[us]);
                if (id < 0) break;
                const Unit u = decode_unit<C::kQT, kGen>(id, p);
                // Q tile t (one q_full phase per unit and tile, possibly with no
                // bytes). One box per 64-column block: nq_blk rows of G heads.
                auto load_q = [&](int t) -> bool {
                    if (k > 0 && !mbar_wait(&bars->q_empty[t], (uint32_t)((k - 1) & 1), wd))
                        return false;
                    mbar_arrive_expect_tx(&bars->q_full[t], u.n[t] > 0 ? q_bytes : 0u);
                    q_unit[t] = k;
                    if (u.n[t] > 0)
                        for (int blk = 0; blk < C::kBlocks; ++blk)
                            tma_load_3d_hint(&tm_q, &bars->q_full[t], sQ[t] + blk * C::kBlockBytes,
                                             blk * C::kBlockElems, (u.rb0 + t) * sh.nq_blk,
                                             u.b * p.H + u.h0, pol_q);
                    return true;
                };
                // The first two K/V loads go first: the ring has room while the
                // previous unit's last tiles are consumed, and Q may have to wait.
                const int early = min(2, 2 * u.n_max);
                for (int jj = 0; ok && jj < early; ++jj) ok = load_kv(u, jj);
#pragma unroll
                for (int t = 0; t < C::kQT; ++t) ok = ok && load_q(t);
                // the rest of K_0, V_0, K_1, V_1, ... of this unit
                for (int jj = early; ok && jj < 2 * u.n_max; ++jj) ok = load_kv(u, jj);
                if (!ok) break;
                // Only now (loads run about two key tiles ahead of the MMAs) ask
                // for the next unit: a CTA takes a new unit when it is nearly
                // free, so the heaviest remaining unit goes to the first SM that
                // frees up, and its first loads still overlap this unit's tail.
                mbar_arrive_expect_tx(&bars->clc_bar[us], 16);
                clc_try_cancel(&bars->clc_resp[us], &bars->clc_bar[us]);
                clc_pending = us;
                clc_pending_parity = (uint32_t)((k >> 1) & 1);
                ok = mbar_wait(&bars->clc_bar[us], clc_pending_parity, wd);
                if (!ok) break;
                clc_pending = -1;
                id = clc_decode(&bars->clc_resp[us]);
                fence_proxy_async_smem();
            }
            // Drain: every copy issued must have landed before the CTA exits.
            if (clc_pending >= 0) mbar_wait_drain(&bars->clc_bar[clc_pending], clc_pending_parity, wd);
            for (int l2 = max(0, L - C::kSlots); l2 < L; ++l2)
                mbar_wait_drain(&bars->kv_full[l2 % C::kSlots], (uint32_t)(l2 / C::kSlots) & 1u,
                                wd);
            for (int t = 0; t < C::kQT; ++t)
                if (q_unit[t] >= 0) mbar_wait_drain(&bars->q_full[t], (uint32_t)(q_unit[t] & 1), wd);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ====================================================== MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = (E == 2) ? idesc_bf16_f32(128, kTile, 0, 0)
                                                   : idesc_e4m3_f32(128, kTile, 0, 0);
            constexpr int kPvN = (D > 128) ? 128 : D;          // N of one P.V MMA
            constexpr int kPvHalves = D / kPvN;
            constexpr uint32_t idesc_pv = (E == 2) ? idesc_bf16_f32(128, kPvN, 0, 1)
                                                   : idesc_e4m3_f32(128, kPvN, 0, 1);
            constexpr int kStepRows = 32 / E;                  // keys per 32-byte K-step
            // Descriptors are built once; a tile's start address is added in
            // 16-byte units to the low field (addresses stay below 256 KB).
            const uint64_t dq0 = smem_desc(smem_u32(sQ[0]), 16, C::kAtomBytes, C::kSwizzle);
            const uint64_t dk0 = smem_desc(smem_u32(sKV), 16, C::kAtomBytes, C::kSwizzle);  // K-major
            const uint64_t dv0 =                                                              // MN-major
                smem_desc(smem_u32(sKV), C::kBlockBytes, C::kAtomBytes, C::kSwizzle);
            constexpr uint64_t kTileStep = (uint64_t)(C::kTileBytes >> 4);
            // S buffer sb = Q tile t . K tile in `slot`
            auto issue_qk = [&](int t, int sb, int slot) {
                const uint64_t a = dq0 + (uint64_t)t * kTileStep;
                const uint64_t b = dk0 + (uint64_t)slot * kTileStep;
#pragma unroll
                for (int kk = 0; kk < D * E / 32; ++kk) {      // 32-byte K-steps
                    const uint64_t off =
                        (uint64_t)(((kk / C::kStepsPerBlock) * C::kBlockBytes +
                                    (kk % C::kStepsPerBlock) * 32) >> 4);
                    if constexpr (E == 2)
                        umma_ss(tmem + C::col_s(sb), a + off, b + off, idesc_qk, kk > 0 ? 1u : 0u);
                    else
                        umma_ss_f8(tmem + C::col_s(sb), a + off, b + off, idesc_qk,
                                   kk > 0 ? 1u : 0u);
                }
            };
            // O of tile t (+)= P in S buffer sb . V tile in `slot`. At d = 256 each
            // K-step is issued as two N = 128 MMAs, one per half of V's columns
            // (the same instruction shape as d = 128): two 128-byte column
            // blocks of bf16, one of e4m3.
            auto issue_pv = [&](int t, int sb, int slot, bool accumulate) {
                const uint64_t b = dv0 + (uint64_t)slot * kTileStep;
                const uint32_t tP = tmem + C::col_s(sb);
#pragma unroll
                for (int kk = 0; kk < kTile / kStepRows; ++kk) {
#pragma unroll
                    for (int h = 0; h < kPvHalves; ++h) {
                        const uint64_t bk = b + (uint64_t)((kk * kStepRows * C::kRowBytes +
                                                            h * (kPvN * E / C::kRowBytes) * C::kBlockBytes) >> 4);
                        if constexpr (E == 2)
                            umma_ts(tmem + C::col_o(t) + (uint32_t)(h * kPvN),
                                    tP + (uint32_t)(kk * 8), bk, idesc_pv,
                                    (accumulate || kk > 0) ? 1u : 0u);
                        else
                            umma_ts_f8(tmem + C::col_o(t) + (uint32_t)(h * kPvN),
                                       tP + (uint32_t)(kk * 8), bk, idesc_pv,
                                       (accumulate || kk > 0) ? 1u : 0u);
                    }
                }
            };
            bool ok = true;
            int L0 = 0;                         // index of this unit's first K/V load
            // Per-tile state is indexed by compile-time constants only (the tile
            // loops are unrolled; one tile keeps bits of one word), so none of
            // it is placed in local memory.
            uint32_t ph_p[2] = {0u, 0u};        // p_full phases consumed (two tiles)
            uint32_t ph_pb = 0u;                // one tile: bit b = parity of p_full[b]'s next phase
            if constexpr (C::kQT == 2) {
            for (int k = 0; ok; ++k) {
                const int us = k & 1;
                ok = mbar_wait(&bars->unit_full[us], (uint32_t)((k >> 1) & 1), wd);
                if (!ok) break;
                const int id = bars->unit_id[us];
                mbar_arrive(&bars->unit_empty[us]);
                if (id < 0) break;
                const Unit u = decode_unit<C::kQT, kGen>(id, p);
                // O_t is free once the previous unit's epilogue has read it
                bool o_ready[2] = {k == 0, k == 0};
#pragma unroll
                for (int t = 0; t < 2; ++t)
                    ok = ok && mbar_wait(&bars->q_full[t], (uint32_t)(k & 1), wd);
                if (ok && u.n_max > 0) {
                    ok = mbar_wait(&bars->kv_full[L0 % C::kSlots],
                                   (uint32_t)(L0 / C::kSlots) & 1u, wd);
                    if (ok) {
                        tc_fence_after();
#pragma unroll
                        for (int t = 0; t < 2; ++t) {
                            if (u.n[t] > 0) {
                                issue_qk(t, t, L0 % C::kSlots);
                                umma_commit(&bars->s_full[t]);
                                if (u.n[t] == 1) umma_commit(&bars->q_empty[t]);  // last Q.K^T
                            }
                        }
                        umma_commit(&bars->kv_empty[L0 % C::kSlots]);
                    }
                }
                for (int j = 0; ok && j < u.n_max; ++j) {
                    const int LV = L0 + 2 * j + 1, LK = L0 + 2 * j + 2;
                    const int sV = LV % C::kSlots, sK = LK % C::kSlots;
                    ok = mbar_wait(&bars->kv_full[sV], (uint32_t)(LV / C::kSlots) & 1u, wd);
                    if (!ok) break;
                    bool k_ready = false;
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        if (!ok || j >= u.n[t]) continue;
                        ok = mbar_wait(&bars->p_full[t], ph_p[t] & 1u, wd);
                        ++ph_p[t];
                        if (ok && !o_ready[t]) {
                            ok = mbar_wait(&bars->o_empty[t], (uint32_t)((k - 1) & 1), wd);
                            o_ready[t] = true;
                        }
                        if (!ok) continue;
                        tc_fence_after();
                        issue_pv(t, t, sV, j > 0);
                        umma_commit(&bars->o_done[t]);
                        if (j + 1 < u.n[t]) {
                            if (!k_ready) {
                                ok = mbar_wait(&bars->kv_full[sK],
                                               (uint32_t)(LK / C::kSlots) & 1u, wd);
                                if (!ok) continue;
                                tc_fence_after();
                                k_ready = true;
                            }
                            issue_qk(t, t, sK);
                            umma_commit(&bars->s_full[t]);
                            if (j + 2 == u.n[t]) umma_commit(&bars->q_empty[t]);  // last Q.K^T
                        }
                    }
                    if (!ok) break;
                    umma_commit(&bars->kv_empty[sV]);
                    if (k_ready) umma_commit(&bars->kv_empty[sK]);
                }
                if (!ok) break;
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (ok && u.n[t] == 0) {           // idle tile: its once-per-unit hand-offs
                        umma_commit(&bars->q_empty[t]);
                        if (!o_ready[t])
                            ok = mbar_wait(&bars->o_empty[t], (uint32_t)((k - 1) & 1), wd);
                        umma_commit(&bars->o_done[t]);
                    }
                }
                L0 += 2 * u.n_max;
            }
            } else {
            // One query tile, S double-buffered: QK(0) QK(1) | PV(0) QK(2) | PV(1) QK(3) ...
            // QK(j+2) overwrites the buffer PV(j) reads, after it in issue order.
            for (int k = 0; ok; ++k) {
                const int us = k & 1;
                ok = mbar_wait(&bars->unit_full[us], (uint32_t)((k >> 1) & 1), wd);
                if (!ok) break;
                const int id = bars->unit_id[us];
                mbar_arrive(&bars->unit_empty[us]);
                if (id < 0) break;
                const Unit u = decode_unit<C::kQT, kGen>(id, p);
                const int n = u.n[0];
                uint32_t o_ready = (k == 0) ? 3u : 0u;   // bit ob: O accumulator ob is free
                // positions of K_t and V_j in this unit's load order (see the producer)
                auto posK = [&](int t) { return t < 2 ? t : 2 * t - 1; };
                auto posV = [&](int j) { return (j <= n - 3) ? 2 + 2 * j : n + j; };
                auto slot_of = [&](int pos) { return (L0 + pos) % C::kSlots; };
                auto wait_load = [&](int pos) -> bool {
                    const int L = L0 + pos;
                    return mbar_wait(&bars->kv_full[L % C::kSlots],
                                     (uint32_t)(L / C::kSlots) & 1u, wd);
                };
                ok = mbar_wait(&bars->q_full[0], (uint32_t)(k & 1), wd);
                for (int t = 0; ok && t < min(2, n); ++t) {
                    ok = wait_load(posK(t));
                    if (!ok) break;
                    tc_fence_after();
                    issue_qk(0, t, slot_of(posK(t)));
                    umma_commit(&bars->s_full[t]);
                    umma_commit(&bars->kv_empty[slot_of(posK(t))]);
                    if (t == n - 1) umma_commit(&bars->q_empty[0]);   // last Q.K^T
                }
                for (int j = 0; ok && j < n; ++j) {
                    const int b = j & 1;
                    ok = wait_load(posV(j));
                    if (!ok) break;
                    ok = mbar_wait(&bars->p_full[b], (ph_pb >> b) & 1u, wd);
                    ph_pb ^= 1u << b;
                    const int ob = kDual ? b : 0;          // O accumulator of this tile
                    if (ok && !((o_ready >> ob) & 1u)) {
                        ok = mbar_wait(&bars->o_empty[ob], (uint32_t)((k - 1) & 1), wd);
                        o_ready |= 1u << ob;
                    }
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(ob, b, slot_of(posV(j)), kDual ? j > 1 : j > 0);
                    umma_commit(&bars->o_done[ob]);
                    umma_commit(&bars->kv_empty[slot_of(posV(j))]);
                    if (j + 2 < n) {
                        ok = wait_load(posK(j + 2));
                        if (!ok) break;
                        tc_fence_after();
                        issue_qk(0, b, slot_of(posK(j + 2)));
                        umma_commit(&bars->s_full[b]);
                        umma_commit(&bars->kv_empty[slot_of(posK(j + 2))]);
                        if (j + 2 == n - 1) umma_commit(&bars->q_empty[0]);   // last Q.K^T
                    }
                }
                if (!ok) break;
                if (n == 0) umma_commit(&bars->q_empty[0]);   // idle unit: its Q hand-off
                // an O accumulator that took no tile this unit: its once-per-unit hand-offs
                for (int ob = 0; ok && ob < (kDual ? 2 : 1); ++ob) {
                    if (n > ob) continue;
                    if (!((o_ready >> ob) & 1u))
                        ok = mbar_wait(&bars->o_empty[ob], (uint32_t)((k - 1) & 1), wd);
                    umma_commit(&bars->o_done[ob]);
                }
                L0 += 2 * n;
            }
            }
            // Drain: all MMAs issued by this thread complete before teardown.
            umma_commit(&bars->teardown);
            mbar_wait_drain(&bars->teardown, 0u, wd);
        }
        __syncwarp();
    } else if (warp < kSoftmaxWarps) {
        // ====================================================== softmax warpgroups
        const int wg = warp >> 2;                     // warpgroup
        const int t = kDual ? 0 : wg;                 // query tile 0 or 1
        const int ob = wg;                            // O accumulator / o_done of this warpgroup
        const int row = tid & (kTile - 1);            // row within the tile == TMEM lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tO = tmem + lane_base + C::col_o(ob);
        const float c = p.scale_log2;
        // Barrier parities, one word: bit b (b = 0, 1) is the parity of s_full[b]'s
        // next phase, bit 2 that of the o_done phases of earlier units.
        uint32_t par = 0u;
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int us = k & 1;
            ok = mbar_wait(&bars->unit_full[us], (uint32_t)((k >> 1) & 1), wd);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            const int id = bars->unit_id[us];
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->unit_empty[us]);
            if (id < 0) break;
            const Unit u = decode_unit<C::kQT, kGen>(id, p);
            const int n = t ? u.n[1] : u.n[0];   // a select: an index would put u in local memory
            int row_id;    // (b*H + h)*Nq + i of this thread's row, -1 for a padding row
            int lim_rel;   // visible keys j < lim_rel + kt0*128 (padding rows see none)
            {
                const int g = row / sh.nq_blk;        // head within the tile
                const int i = (u.rb0 + t) * sh.nq_blk + (row - g * sh.nq_blk);   // query row
                const bool valid = g < sh.G && i < sh.Nq;
                row_id = valid ? (u.b * p.H + u.h0 + g) * sh.Nq + i : -1;
                const int lim_row =
                    !valid ? 0 : p.causal ? min(u.kv_lim, i + sh.q_off + 1) : u.kv_lim;
                lim_rel = lim_row - u.kt0 * kTile;
            }
            // A warp whose 32 rows are all padding (packed or short query
            // blocks) keeps every barrier hand-off but skips the arithmetic;
            // its rows of P and O are never read back.
            const bool idle_warp = kGen && !__any_sync(0xffffffffu, row_id >= 0);
            float m_ref = -INFINITY;   // reference maximum (raw score units)
            float l = 0.f;             // running sum of exp2((s - m_ref) * c)
            float lr = 0.f;            // the same over the probabilities as rounded for P.V
            // tiles of this warpgroup: all of them, or (two accumulators) j = wg, wg + 2, ...
            const int j_first = kDual ? wg : 0, j_step = kDual ? 2 : 1;
            const int n_own = kDual ? (n > wg ? (n - wg + 1) / 2 : 0) : n;

            // One query tile with one accumulator: the last score tile was issued
            // after P.V(n-3) only, so when the epilogue starts o_done may be one
            // phase short of P.V(n-2) -- or, if P.V(n-1) has already finished,
            // one phase past the last, with the same parity as phase n-2. The
            // wait for phase n-2 is therefore made inside the last tile, before
            // its P is handed over: P.V(n-1) cannot have been issued yet, so
            // o_done is at phase n-2 or n-1 and the parity test is exact. The
            // epilogue then waits for phase n-1 alone (o_done is at n-1 or n).
            auto wait_second_last = [&](int j) -> bool {
                if constexpr (!kDual && C::kQT == 1) {
                    if (j == n - 1 && n >= 2) {
                        bool w = mbar_wait(&bars->o_done[ob], ((par >> 2) + (uint32_t)(n - 2)) & 1u, wd);
                        return __all_sync(0xffffffffu, w);
                    }
                }
                return true;
            };

            for (int j = j_first; j < n; j += j_step) {
                const int jo = kDual ? (j - wg) / 2 : j;       // index among this warpgroup's tiles
                const int sb = (C::kQT == 2) ? t : (j & 1);   // this tile's S buffer
                const uint32_t tS = tmem + lane_base + C::col_s(sb);
                ok = mbar_wait(&bars->s_full[sb], (par >> sb) & 1u, wd);
                par ^= 1u << sb;
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                if (idle_warp) {
                    ok = wait_second_last(j);
                    if (!ok) break;
                    mbar_arrive(&bars->p_full[sb]);
                    continue;
                }
                tc_fence_after();
                float s[kTile];
#pragma unroll
                for (int ch = 0; ch < kTile / 32; ++ch) {
                    uint32_t r[32];
                    tmem_ld32(tS + (uint32_t)(ch * 32), r);
#pragma unroll
                    for (int q = 0; q < 32; ++q) s[ch * 32 + q] = __uint_as_float(r[q]);
                }
                tmem_wait_ld();
                const int j0 = j * kTile;
                if (j0 + kTile > lim_rel) {
                    const int lim = lim_rel - j0;
#pragma unroll
                    for (int q = 0; q < kTile; ++q)
                        if (q >= lim) s[q] = -INFINITY;
                }
                bool rescale = false;
                float alpha = 1.f;
                float2 l_tile;
                if constexpr (kMaxFirst) {
                    // The reference maximum m_ref is fixed before any exponential
                    // of the tile: the row's first visible tile sets it to its row
                    // maximum, and a later tile moves it only when the tile's
                    // maximum exceeds it by more than rescale_log2 (log2 units),
                    // after O and l are brought to the new reference. Every
                    // probability is then at most 2^64 (bf16 P), l < N * 2^64 and
                    // O stay far inside the fp32 range, and O / l is exact
                    // whatever m_ref is.
                    const float m_tile = row_max(s);
                    if (m_ref == -INFINITY) {
                        m_ref = m_tile;
                    } else if ((m_tile - m_ref) * c > rescale_log2<E>()) {
                        alpha = fast_exp2((m_ref - m_tile) * c);
                        m_ref = m_tile;
                        l *= alpha;
                        lr *= alpha;
                        rescale = true;
                    }
                    if (__any_sync(0xffffffffu, rescale)) {
                        // O holds the P.V sums of tiles < j: wait for the last of
                        // them (P of this tile is not handed over yet, so o_done is
                        // exactly at that phase or one short), then rescale it, 16
                        // columns at a time while the tile's scores are live.
                        ok = mbar_wait(&bars->o_done[ob], ((par >> 2) + (uint32_t)(jo - 1)) & 1u, wd);
                        ok = __all_sync(0xffffffffu, ok);
                        if (!ok) break;
                        tc_fence_after();
                        rescale_o<D, 16>(tO, alpha);
                    }
                    const float mc = (m_ref == -INFINITY) ? 0.f : m_ref * c;
                    l_tile = exp_tile<E>(s, c, mc, tS);
                    l += l_tile.x;
                    lr += l_tile.y;
                } else {
                    // The first tile sets the reference maximum m_ref from its row
                    // maximum. Later tiles exponentiate against the current m_ref
                    // straight away; only if that makes the tile's row sum exceed
                    // redo_tile_sum (some p > 2^64) does the row take its true
                    // maximum, rescale O and l, and redo the tile. Below that bound
                    // every probability, l (< N * 2^64) and O stay far inside the
                    // fp32 and bf16 range, and O / l is exact whatever m_ref is.
                    if (m_ref == -INFINITY) m_ref = row_max(s);
                    float mc = (m_ref == -INFINITY) ? 0.f : m_ref * c;
                    l_tile = exp_tile<E>(s, c, mc, tS);
                    const bool stale = !(l_tile.x <= redo_tile_sum<E>());
                    if (__any_sync(0xffffffffu, stale)) {
                        if (stale) {
                            const float m_new = fmaxf(m_ref, row_max(s));
                            alpha = fast_exp2((m_ref - m_new) * c);
                            m_ref = m_new;
                            l *= alpha;
                            lr *= alpha;
                            rescale = true;
                        }
                        mc = m_ref * c;
                        l_tile = exp_tile<E>(s, c, mc, tS);   // tcgen05.st is warp-wide: redo all rows
                    }
                    l += l_tile.x;
                    lr += l_tile.y;
                    if (__any_sync(0xffffffffu, rescale)) {
                        // O holds the P.V sums of tiles < j: wait for the last of
                        // them, then bring it to the new reference maximum.
                        ok = mbar_wait(&bars->o_done[ob], ((par >> 2) + (uint32_t)(jo - 1)) & 1u, wd);
                        ok = __all_sync(0xffffffffu, ok);
                        if (!ok) break;
                        tc_fence_after();
                        rescale_o<D, 32>(tO, alpha);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                ok = wait_second_last(j);
                if (!ok) break;
                mbar_arrive(&bars->p_full[sb]);
            }
            if (!ok) break;

            // ------------------------------------------------ epilogue
            // the unit's last o_done phase for this accumulator (its idle phase if none)
            const uint32_t last = (par >> 2) + (uint32_t)(n_own > 0 ? n_own - 1 : 0);
            par ^= (uint32_t)((n_own > 0 ? n_own : 1) & 1) << 2;
            ok = mbar_wait(&bars->o_done[ob], last & 1u, wd);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            // Two accumulators: warpgroup 1 hands its row's (m, l, lr) to warpgroup 0
            // (its O1 is complete: it has just waited for its last P.V), and
            // warpgroup 0 writes the merged row.
            float a0 = 1.f, a1 = 0.f;          // weights of O0 and O1 in the merged row
            bool have1 = false;                // O1 holds a tile of this unit
            if constexpr (kDual) {
                const int mb = k & 1;
                if (wg == 1) {
                    bars->merge_m[mb][row] = (l > 0.f) ? m_ref * c : -INFINITY;
                    bars->merge_l[mb][row] = l;
                    bars->merge_lr[mb][row] = lr;
                    mbar_arrive(&bars->merge_full[mb]);
                    continue;
                }
                ok = mbar_wait(&bars->merge_full[mb], (uint32_t)((k >> 1) & 1), wd);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                const float m0 = (l > 0.f) ? m_ref * c : -INFINITY;
                const float m1 = bars->merge_m[mb][row], l1 = bars->merge_l[mb][row];
                const float mm = fmaxf(m0, m1);
                a0 = (l > 0.f) ? fast_exp2(m0 - mm) : 0.f;
                a1 = (l1 > 0.f) ? fast_exp2(m1 - mm) : 0.f;
                l = l * a0 + l1 * a1;
                lr = lr * a0 + bars->merge_lr[mb][row] * a1;
                m_ref = (mm == -INFINITY) ? -INFINITY : mm / c;   // merged reference (score units)
                have1 = n > 1;
            }
            tc_fence_after();
            const bool write = row_id >= 0;
            // O is divided by the sum of the rounded probabilities the P.V product
            // used (with two accumulators, both sums merged like O); lse takes
            // the exact sum.
            const float o_div = lr;
            const float inv_l = (o_div > 0.f) ? p.o_mul / o_div : 0.f;
            const float row_lse = (l > 0.f) ? (m_ref * c + log2f(l)) * kLn2 : -INFINITY;
            const size_t orow_idx = (size_t)row_id;
            const size_t prow_idx = (size_t)u.s * ((size_t)p.B * p.H * sh.Nq) + (size_t)row_id;
            // O leaves TMEM kW columns at a time (16 with two accumulators,
            // whose columns are both live at once).
            constexpr int kW = kDual ? 16 : 32;
            auto ld_cols = [&](uint32_t taddr, uint32_t (&r)[kW]) {
                if constexpr (kW == 16) tmem_ld16(taddr, r);
                else tmem_ld32(taddr, r);
            };
#pragma unroll
            for (int ch = 0; ch < D / kW; ++ch) {
                uint32_t r[kW];
                if (n > 0 && !idle_warp) {
                    ld_cols(tO + (uint32_t)(ch * kW), r);
                    if constexpr (kDual) {
                        uint32_t r1[kW];
                        if (have1) {
                            ld_cols(tmem + lane_base + C::col_o(1) + (uint32_t)(ch * kW), r1);
                            tmem_wait_ld();
                        } else {
                            tmem_wait_ld();
#pragma unroll
                            for (int q = 0; q < kW; ++q) r1[q] = 0u;
                        }
#pragma unroll
                        for (int q = 0; q < kW; ++q)
                            r[q] = __float_as_uint(__uint_as_float(r[q]) * a0 +
                                                   __uint_as_float(r1[q]) * a1);
                    } else {
                        tmem_wait_ld();
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < kW; ++q) r[q] = 0u;
                }
                if (ch == D / kW - 1) {
                    // O has been read: the next unit's first P.V may overwrite it
                    tc_fence_before();
                    mbar_arrive(&bars->o_empty[ob]);
                    if (kDual) mbar_arrive(&bars->o_empty[1]);
                }
                if (write && (!kGen || p.o_part == nullptr)) {
                    uint4* dst = reinterpret_cast<uint4*>(p.o + orow_idx * D + ch * kW);
#pragma unroll
                    for (int v = 0; v < kW / 8; ++v) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]) * inv_l,
                                          __uint_as_float(r[8 * v + 1]) * inv_l);
                        w.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]) * inv_l,
                                          __uint_as_float(r[8 * v + 3]) * inv_l);
                        w.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]) * inv_l,
                                          __uint_as_float(r[8 * v + 5]) * inv_l);
                        w.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]) * inv_l,
                                          __uint_as_float(r[8 * v + 7]) * inv_l);
                        dst[v] = w;
                    }
                } else if (write) {
                    // split-KV partial: this key range's O / l in fp32
                    float4* dst = reinterpret_cast<float4*>(p.o_part + prow_idx * D + ch * kW);
#pragma unroll
                    for (int v = 0; v < kW / 4; ++v)
                        dst[v] = make_float4(__uint_as_float(r[4 * v + 0]) * inv_l,
                                             __uint_as_float(r[4 * v + 1]) * inv_l,
                                             __uint_as_float(r[4 * v + 2]) * inv_l,
                                             __uint_as_float(r[4 * v + 3]) * inv_l);
                }
            }
            if (write) {
                if (!kGen || p.o_part == nullptr) p.lse[orow_idx] = row_lse;
                else p.lse_part[prow_idx] = row_lse;
            }
        }
    }

    // ---------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace fa
