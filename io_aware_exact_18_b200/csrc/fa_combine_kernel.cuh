// Merge of split-KV partial results.
//
// When the keys of a row are split into S ranges, range s yields its own
// normalised output O_s = (sum_j p_j V_j) / (sum_j p_j) and log-sum-exp lse_s
// over the keys it holds. The softmax over all keys is their lse-weighted
// mixture: lse = ln sum_s exp(lse_s) and O = sum_s exp(lse_s - lse) O_s. This
// is the same rescaling the online softmax applies between key blocks
// ("FlashAttention (UR)", section "Online softmax"), taken once over whole
// ranges instead of tile by tile; a range with no visible key has lse_s = -inf
// and weight 0. The merge reads S * (d + 1) fp32 values per row and writes one
// bf16 row and one lse: a memory-bound pass, one warp per row, each lane owning
// d / 32 neighbouring columns so every split's row is read coalesced.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace fa {

constexpr int kCombineWarps = 8;   // rows per 256-thread block

template <int D>
__global__ void __launch_bounds__(32 * kCombineWarps)
    fa_splitkv_combine(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                       __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int64_t rows,
                       int splits, const uint32_t* dev_err) {
    constexpr int kPer = D / 32;   // columns per lane: 2, 4 or 8
    constexpr float kLog2e = 1.4426950408889634f;
    // Launched as a programmatic dependent of the decoding kernel it may start
    // early: nothing is read before that kernel has completed.
    pdl_wait_prerequisites();
    const int64_t row = (int64_t)blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    if (*reinterpret_cast<const volatile uint32_t*>(dev_err) != 0u) {
        // The attention kernel before this merge skipped or abandoned its work
        // (the device status word is set): its partials are not this call's, so
        // the row reads NaN instead of a merge of stale values.
        const uint32_t nan2 = 0x7FC07FC0u;
#pragma unroll
        for (int c = 0; c < kPer; c += 2)
            *reinterpret_cast<uint32_t*>(o + row * D + lane * kPer + c) = nan2;
        if (lane == 0) lse[row] = __int_as_float(0x7FC00000);
        return;
    }

    // Pass 1: the largest lse_s (lane l reads splits l, l + 32, ...; the first
    // is kept for pass 2).
    const float ls0 = (lane < splits) ? lse_part[(int64_t)lane * rows + row] : -INFINITY;
    float m = ls0;
    for (int s = lane + 32; s < splits; s += 32) m = fmaxf(m, lse_part[(int64_t)s * rows + row]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));

    // Pass 2: weights exp(lse_s - m), one split per lane, broadcast by shuffle;
    // the O_s rows are loaded unconditionally (an empty range wrote O_s = 0 and
    // has weight 0) as 16-byte vectors, eight splits per unrolled step, so a
    // warp has that many rows' loads in flight (the merge is latency-bound: a
    // handful of rows per SM).
    float acc[kPer];
#pragma unroll
    for (int c = 0; c < kPer; ++c) acc[c] = 0.f;
    float wsum = 0.f;
    if (m != -INFINITY) {
        for (int base = 0; base < splits; base += 32) {
            const int sl = base + lane;
            const float ls = (base == 0) ? ls0
                             : (sl < splits) ? lse_part[(int64_t)sl * rows + row] : -INFINITY;
            const float wl = (ls == -INFINITY) ? 0.f : exp2f((ls - m) * kLog2e);
            wsum += wl;
            const int cnt = min(32, splits - base);
            const float* src = o_part + ((int64_t)base * rows + row) * D + lane * kPer;
#pragma unroll 8
            for (int j = 0; j < cnt; ++j) {
                const float w = __shfl_sync(0xffffffffu, wl, j);
                const float* r = src + (int64_t)j * rows * D;
                if constexpr (kPer % 4 == 0) {
#pragma unroll
                    for (int c = 0; c < kPer; c += 4) {
                        const float4 x = *reinterpret_cast<const float4*>(r + c);
                        acc[c] = fmaf(w, x.x, acc[c]);
                        acc[c + 1] = fmaf(w, x.y, acc[c + 1]);
                        acc[c + 2] = fmaf(w, x.z, acc[c + 2]);
                        acc[c + 3] = fmaf(w, x.w, acc[c + 3]);
                    }
                } else {
                    const float2 x = *reinterpret_cast<const float2*>(r);
                    acc[0] = fmaf(w, x.x, acc[0]);
                    acc[1] = fmaf(w, x.y, acc[1]);
                }
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
    }
    const float inv = (wsum > 0.f) ? 1.f / wsum : 0.f;
    __nv_bfloat16* dst = o + row * D + lane * kPer;
#pragma unroll
    for (int c = 0; c < kPer; c += 2)
        *reinterpret_cast<__nv_bfloat162*>(dst + c) =
            __floats2bfloat162_rn(acc[c] * inv, acc[c + 1] * inv);
    if (lane == 0) lse[row] = (wsum > 0.f) ? m + logf(wsum) : -INFINITY;
}

}  // namespace fa
