// pack_groupwise.cuh -- offline packing of group-wise W4A8 weights.
//
// "ComfyUI-INT-Crush", "Weight Format": the INT4 weight scales have one value
// per output row and K group ([out, num_groups]); stable-diffusion.cpp "feat:
// packed int4 convrot model loading and dispatch", "Summary": an asymmetric
// W4A8 format next to the symmetric one.  Per row: the block Hadamard
// rotation along K (as for the per-row weights), then, per group of
// kWeightGroup consecutive K values:
//   symmetric:  s = absmax / 7, q = clamp(rne(v / s), -7, 7), two's complement
//               nibbles;
//   asymmetric: lo = min(0, min v), hi = max(0, max v), s = (hi - lo) / 15,
//               z = clamp(rne(-lo / s), 0, 15), q = clamp(rne(v / s) + z, 0, 15),
//               plain 4-bit nibbles; the weight is s (q - z);
//   an all-zero group: s = 0, z = 0, q = 0.
// Everything in fp32 with IEEE divisions (the codes are decisions).
//
// Layout of the work: one warp per 256-value chunk of a row, 8 consecutive
// values per lane (the rotation's layout: fwht_lane8), so a weight group is
// 16 lanes and its extremes are a 4-step shuffle reduction.  Offline and
// small: no attempt at streaming rows ahead.
#pragma once

#include "quantize.cuh"

namespace tint4 {

constexpr int kWeightGroup = 128;   // K values per weight group (one GEMM K step)

// S16: the scales are stored as IEEE fp16 ("Weight Format": the pages'
// stored format): each is rounded to the nearest fp16 (ties to even) and the
// zero point and codes are taken against that stored value.
template <int G, bool S16 = false>
__global__ void __launch_bounds__(256)
pack_weights_groupwise_kernel(const float* __restrict__ W, int N, int K, int asym,
                              uint8_t* __restrict__ packed, void* __restrict__ scale,
                              uint8_t* __restrict__ zero) {
    static_assert(kWeightGroup == 16 * 8, "a weight group is 16 lanes of 8 values");
    const int lane = threadIdx.x & 31;
    const int nchunks = (K + kQuantChunk - 1) / kQuantChunk;
    const int ng = K / kWeightGroup;
    const long total = static_cast<long>(N) * nchunks;
    const long wstride = static_cast<long>(gridDim.x) * (blockDim.x >> 5);
    for (long item = static_cast<long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
         item < total; item += wstride) {   // warp-uniform
        const int n = static_cast<int>(item / nchunks);
        const int c = static_cast<int>(item % nchunks);
        const int base = c * kQuantChunk + lane * 8;
        const bool have = base < K;   // K % 128 == 0: all lanes, or lanes 0-15
        RawChunk<float> raw;
        if (have) raw.load(W + static_cast<size_t>(n) * K + base);
        else raw.zero();
        float v[8];
        raw.to_f32(v);
        if (G > 0) fwht_lane8<(G > 0 ? G : 16)>(v, lane);
        float lo = 0.0f, hi = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            lo = fminf(lo, v[j]);
            hi = fmaxf(hi, v[j]);
        }
#pragma unroll
        for (int d = 8; d >= 1; d >>= 1) {   // within each half-warp = one group
            lo = fminf(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, d));
            hi = fmaxf(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, d));
        }
        // lo <= 0 <= hi, so the absolute maximum is max(-lo, hi)
        const float s32 = asym ? __fdiv_rn(__fsub_rn(hi, lo), 15.0f) : __fdiv_rn(fmaxf(-lo, hi), 7.0f);
        const __half s16 = __float2half_rn(s32);
        const float s = S16 ? __half2float(s16) : s32;
        int z = 0;
        if (asym && s > 0.0f) z = static_cast<int>(fminf(fmaxf(rintf(__fdiv_rn(-lo, s)), 0.0f), 15.0f));
        uint32_t word = 0u;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            int q = 0;
            if (s > 0.0f) {
                const int t = static_cast<int>(rintf(__fdiv_rn(v[j], s)));
                q = asym ? min(max(t + z, 0), 15) : min(max(t, -7), 7);
            }
            word |= static_cast<uint32_t>(q & 0xF) << (4 * j);
        }
        if (!have) continue;
        *reinterpret_cast<uint32_t*>(packed + static_cast<size_t>(n) * (K / 2) + base / 2) = word;
        if ((lane & 15) == 0) {
            const size_t gi = static_cast<size_t>(n) * ng + base / kWeightGroup;
            if (S16) static_cast<__half*>(scale)[gi] = s16;
            else static_cast<float*>(scale)[gi] = s;
            if (asym) zero[gi] = static_cast<uint8_t>(z);
        }
    }
}

}  // namespace tint4
