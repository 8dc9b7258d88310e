// quantize.cuh -- block Hadamard rotation + per-row symmetric quantization.
//
// One kernel serves two entry points:
//  * convrot_quantize_act: bf16 activations [M, K] -> int8 codes [M, K] (W4A8)
//    or packed int4 codes [M, K/2] (W4A4), plus one fp32 scale per token
//    ("ComfyUI-INT-Crush", "Forward Pass" step 2 rotate and step 5 quantize;
//    "Inference > INT4 > Triton backend": dynamic per-token activation quant).
//  * tint4_pack_weights: fp32 weights [N, K] -> packed int4 [N, K/2] + fp32
//    row scales (offline; "ComfyUI-INT-Crush", "Weight Format"; stable-
//    diffusion.cpp "feat: packed int4 convrot model loading and dispatch",
//    "Summary": packed nibbles with row scales).
//
// Layout of the work: one CTA per row, one warp per 256-value chunk (two
// chunks per warp above 32 chunks); each lane holds 8 consecutive values of
// a chunk in registers (16-byte bf16 loads, fully coalesced), so registers
// stay few and many rows are in flight per SM.  A rotation block of g values (g = 16, 64 or 256) spans g/8
// lanes, so the fast Walsh-Hadamard transform runs as three in-register
// butterfly stages (spans 1, 2, 4) followed by log2(g/8) shuffle stages (spans
// 8 .. g/2), in that order; every butterfly forms (a + b, a - b) with a the
// value at the lower index, so the rotated fp32 values do not depend on which
// thread computes them.  Then the CTA reduces |v| to the row maximum, forms
// scale = absmax / Q with an IEEE division, and writes the codes
// clamp(rne(v / scale), -Q, Q) straight from registers (quant8: the same
// codes without a division per value).  HBM traffic is one
// read of the input and one write of the codes: the kernel is bandwidth
// bound.
#pragma once

#include "ptx.cuh"

namespace tint4 {

constexpr int kQuantMaxWarps = 32;
constexpr int kQuantChunk = 256;       // values per warp chunk (32 lanes x 8)
constexpr int kQuantMaxChunksPerWarp = 2;
constexpr int kQuantMaxK = kQuantMaxWarps * kQuantMaxChunksPerWarp * kQuantChunk;  // 16384

// 8 consecutive inputs as loaded (one 16-byte load of bf16, two of fp32),
// converted to fp32 only when used: a CTA holds the next row's raw chunks
// while it works on the current one.
template <typename InT>
struct RawChunk;

template <>
struct RawChunk<__nv_bfloat16> {
    uint4 u;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { u = __ldg(reinterpret_cast<const uint4*>(p)); }
    __device__ __forceinline__ void zero() { u = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ void to_f32(float (&v)[8]) const {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};

template <>
struct RawChunk<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* p) {
        a = __ldg(reinterpret_cast<const float4*>(p));
        b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.0f, 0.0f, 0.0f, 0.0f); }
    __device__ __forceinline__ void to_f32(float (&v)[8]) const {
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
};

// Orthonormal FWHT over blocks of G values spread as 8 per lane.
template <int G>
__device__ __forceinline__ void fwht_lane8(float (&v)[8], int lane) {
    // in-register stages, spans 1, 2, 4
#pragma unroll
    for (int h = 1; h < 8; h *= 2) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if ((j & h) == 0) {
                const float a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
        }
    }
    // cross-lane stages, spans 8 .. G/2 (lane distance 1 .. G/16)
#pragma unroll
    for (int d = 1; d < G / 8; d *= 2) {
        // lower index holds a, upper holds b: lower -> a + b, upper -> a - b;
        // fma(+-1, own, other) is that sum or difference, rounded once
        const float sgn = (lane & d) ? -1.0f : 1.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float other = __shfl_xor_sync(0xFFFFFFFFu, v[j], d);
            v[j] = fmaf(sgn, v[j], other);
        }
    }
    // 1/sqrt(G): a power of two for G = 4^k, so this is exact
    constexpr float s = (G == 16) ? 0.25f : (G == 64) ? 0.125f : (G == 256) ? 0.0625f : 1.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] *= s;
}

// Codes clamp(rint(v_j / s), -Q, Q) of 8 values, with v_j / s the IEEE fp32
// quotient, from the products t_j = v_j * fl(1/s).  |t - fl(v/s)| <= 3 *
// 2^-24 * |v/s| <= 2.3e-5 here (|v/s| <= Q + tiny), so whenever every t_j of
// the warp lies at least 2^-15 away from a half-integer, t and fl(v/s) round
// to the same integers; otherwise (rare, warp-uniform branch) the codes are
// recomputed with the IEEE division itself.  Same codes as a division per
// value, a fraction of the instructions.  scale == 0 gives rs == 0 and codes 0.
//
// Rounding without the conversion unit: adding 1.5 * 2^23 to a float of
// magnitude < 2^22 rounds it to an integer (to nearest, ties to even, as
// rintf) and leaves that integer in the low bits of the sum, two's
// complement in the low byte.  m[j] are those sums' bit patterns.
//
// CLAMP = false is for scales >= 1e-30 (fl(1/s) finite): then |t| <= Q (1 +
// 3 * 2^-24) < Q + 1/2 for every |v| <= absmax, so the codes are within
// [-Q, Q] without a clamp; __fmul_rn keeps the product from fusing with the
// rounding addition.
template <int Q, bool CLAMP>
__device__ __forceinline__ void quant8(const float (&v)[8], float scale, float rs, uint32_t (&m)[8]) {
    constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23
    bool near = false;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float t = CLAMP ? fminf(fmaxf(v[j] * rs, static_cast<float>(-Q)), static_cast<float>(Q))
                              : __fmul_rn(v[j], rs);
        const float r = t + kMagic;
        near |= fabsf(t - (r - kMagic)) > 0.5f - 3.0517578125e-5f;
        m[j] = __float_as_uint(r);
    }
    if (__any_sync(0xFFFFFFFFu, near) && scale > 0.0f) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float t = fminf(fmaxf(__fdiv_rn(v[j], scale), static_cast<float>(-Q)), static_cast<float>(Q));
            m[j] = __float_as_uint(t + kMagic);
        }
    }
}

// For the fused small-M linear: rotate + quantize up to kFuseMaxRows rows of
// x (bf16 [M, K], K <= 256 * warps) into one int8 code per byte in shared
// memory ([M][K]) and fp32 scales, with every warp of the CTA: warp w owns
// chunk w of every row, all rows' loads are in flight together, and one
// barrier gives the row maxima.  Same arithmetic, so the same codes, as
// rotate_quantize_rows_kernel.  Ends with a barrier.  Every CTA of the GEMM
// repeats this work, so it pays only for a single token: at 4 tokens the
// fused launch took 13.1 us against 11.1 us for two launches.
constexpr int kFuseMaxRows = 1;

template <int G, int Q>
__device__ __forceinline__ void rotate_quantize_rows_to_smem(const __nv_bfloat16* __restrict__ x,
                                                             int M, int K, int8_t* codes,
                                                             float* scales,
                                                             float (&red)[kFuseMaxRows][kQuantMaxWarps]) {
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nchunks = (K + kQuantChunk - 1) / kQuantChunk;
    const int base = warp * kQuantChunk + lane * 8;
    const bool mine = warp < nchunks;   // warp-uniform
    RawChunk<__nv_bfloat16> raw[kFuseMaxRows];
#pragma unroll
    for (int r = 0; r < kFuseMaxRows; ++r) {
        if (r < M && mine && base < K) raw[r].load(x + static_cast<size_t>(r) * K + base);
        else raw[r].zero();
    }
    float v[kFuseMaxRows][8];
#pragma unroll
    for (int r = 0; r < kFuseMaxRows; ++r) {
        raw[r].to_f32(v[r]);
        float amax = 0.0f;
        if (r < M && mine) {
            if (G > 0) fwht_lane8<(G > 0 ? G : 16)>(v[r], lane);
#pragma unroll
            for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[r][j]));
        }
#pragma unroll
        for (int d = 16; d >= 1; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, d));
        if (lane == 0) red[r][warp] = amax;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kFuseMaxRows; ++r) {
        if (r >= M) break;
        float amax = red[r][0];
        for (int w = 1; w < nchunks; ++w) amax = fmaxf(amax, red[r][w]);
        const float scale = __fdiv_rn(amax, static_cast<float>(Q));
        const float rscale = scale > 0.0f ? __frcp_rn(scale) : 0.0f;
        if (threadIdx.x == 0) scales[r] = scale;
        if (!mine) continue;
        uint32_t m[8];
        if (scale < 1e-30f) quant8<Q, true>(v[r], scale, rscale, m);
        else quant8<Q, false>(v[r], scale, rscale, m);
        if (base >= K) continue;
        const uint32_t lo = __byte_perm(__byte_perm(m[0], m[1], 0x0040), __byte_perm(m[2], m[3], 0x0040), 0x5410);
        const uint32_t hi = __byte_perm(__byte_perm(m[4], m[5], 0x0040), __byte_perm(m[6], m[7], 0x0040), 0x5410);
        *reinterpret_cast<uint2*>(codes + r * K + base) = make_uint2(lo, hi);
    }
    __syncthreads();
}

// Q = 127 (int8 codes) or 7 (int4 codes); PACKED: int4 codes two per byte,
// else one code per int8.  CH = chunks per warp held in registers; the CTA
// has blockDim.x / 32 warps (K <= warps * CH * 256).  Persistent: CTA b
// handles rows b, b + gridDim.x, ..., and the loads of its next row are in
// flight while it rotates and quantizes the current one.
// The rows of one CTA.  FULL: the CTA's warps hold exactly K values (every
// chunk present and complete), so no per-chunk guard is needed.
// EVOD (int8 codes only): each block of 8 codes is stored with its even
// positions first (codes 0, 2, 4, 6, 1, 3, 5, 7), the layout whose weights
// the tensor-core GEMM unpacks without byte permutes; a private layout of the
// fused linears' workspace (the sums over K are the same numbers).
template <typename InT, int G, int Q, bool PACKED, int CH, bool FULL, bool EVOD = false>
__device__ __forceinline__ void rotate_quantize_rows(const InT* __restrict__ in, int rows, int K,
                                                     void* __restrict__ codes,
                                                     float* __restrict__ scales,
                                                     float (&red)[2][kQuantMaxWarps]) {
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const int nchunks = (K + kQuantChunk - 1) / kQuantChunk;
    auto present = [&](int c) { return FULL || warp + c * nwarps < nchunks; };   // warp-uniform
    auto base_of = [&](int c) { return (warp + c * nwarps) * kQuantChunk + lane * 8; };

    RawChunk<InT> raw[CH];
    auto fetch = [&](int r) {
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            const int base = base_of(c);
            if (r < rows && present(c) && (FULL || base < K))
                raw[c].load(in + static_cast<size_t>(r) * K + base);
            else
                raw[c].zero();
        }
    };
    fetch(blockIdx.x);

    int it = 0;
    for (int row = blockIdx.x; row < rows; row += gridDim.x, ++it) {
        float v[CH][8];
#pragma unroll
        for (int c = 0; c < CH; ++c) raw[c].to_f32(v[c]);
        fetch(row + gridDim.x);

        float amax = 0.0f;
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            if (present(c)) {
                if (G > 0) fwht_lane8<(G > 0 ? G : 16)>(v[c], lane);
#pragma unroll
                for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[c][j]));
            }
        }
#pragma unroll
        for (int d = 16; d >= 1; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, d));
        float* rb = red[it & 1];
        if (lane == 0) rb[warp] = amax;
        __syncthreads();
        amax = rb[0];
        for (int w = 1; w < nwarps; ++w) amax = fmaxf(amax, rb[w]);

        const float scale = __fdiv_rn(amax, static_cast<float>(Q));
        const float rscale = scale > 0.0f ? __frcp_rn(scale) : 0.0f;
        const bool tiny = scale < 1e-30f;   // row-uniform: take the clamped path
        if (threadIdx.x == 0) scales[row] = scale;

#pragma unroll
        for (int c = 0; c < CH; ++c) {
            if (!present(c)) continue;   // warp-uniform (quant8 votes across the warp)
            const int base = base_of(c);
            uint32_t m[8];
            if (tiny) quant8<Q, true>(v[c], scale, rscale, m);
            else quant8<Q, false>(v[c], scale, rscale, m);
            if (!FULL && base >= K) continue;
            // the code of value j is the low byte of m[j] (two's complement)
            const uint32_t lo = __byte_perm(__byte_perm(m[0], m[1], 0x0040), __byte_perm(m[2], m[3], 0x0040), 0x5410);
            const uint32_t hi = __byte_perm(__byte_perm(m[4], m[5], 0x0040), __byte_perm(m[6], m[7], 0x0040), 0x5410);
            if (!PACKED) {
                int8_t* dst = static_cast<int8_t*>(codes) + static_cast<size_t>(row) * K + base;
                if (EVOD)
                    *reinterpret_cast<uint2*>(dst) =
                        make_uint2(__byte_perm(lo, hi, 0x6420), __byte_perm(lo, hi, 0x7531));
                else
                    *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
            } else {
                // low nibble = even index, high nibble = odd index: gather the
                // even-index codes and the odd-index codes, then interleave nibbles
                const uint32_t ev = __byte_perm(lo, hi, 0x6420);   // codes 0, 2, 4, 6
                const uint32_t od = __byte_perm(lo, hi, 0x7531);   // codes 1, 3, 5, 7
                const uint32_t out = (ev & 0x0F0F0F0Fu) | ((od & 0x0F0F0F0Fu) << 4);
                uint8_t* dst = static_cast<uint8_t*>(codes) + static_cast<size_t>(row) * (K / 2) + base / 2;
                *reinterpret_cast<uint32_t*>(dst) = out;
            }
        }
    }
}

// Q = 127 (int8 codes) or 7 (int4 codes); PACKED: int4 codes two per byte,
// else one code per int8.  CH = chunks per warp held in registers; the CTA
// has blockDim.x / 32 warps (K <= warps * CH * 256).  Persistent: CTA b
// handles rows b, b + gridDim.x, ..., and the loads of its next row are in
// flight while it rotates and quantizes the current one.
template <typename InT, int G, int Q, bool PACKED, int CH, bool EVOD = false>
__global__ void __launch_bounds__(CH == 1 ? 8 * 32 : kQuantMaxWarps * 32)   // one chunk per warp: K <= 2048
rotate_quantize_rows_kernel(const InT* __restrict__ in, int rows, int K,
                            void* __restrict__ codes, float* __restrict__ scales) {
    __shared__ float red[2][kQuantMaxWarps];   // per-warp maxima, alternate rows
    // Under programmatic dependent launch, let the consumer grid start its
    // prologue while this grid runs; it waits for our completion before
    // reading the codes.
    grid_launch_dependents();
    if (K == static_cast<int>(blockDim.x / 32) * CH * kQuantChunk)
        rotate_quantize_rows<InT, G, Q, PACKED, CH, true, EVOD>(in, rows, K, codes, scales, red);
    else
        rotate_quantize_rows<InT, G, Q, PACKED, CH, false, EVOD>(in, rows, K, codes, scales, red);
}

}  // namespace tint4
