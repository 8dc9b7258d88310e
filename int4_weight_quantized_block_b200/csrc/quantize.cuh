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
    // through L2, for kernels that may run while the grid writing p finishes
    __device__ __forceinline__ void load_l2(const __nv_bfloat16* p) { u = __ldcg(reinterpret_cast<const uint4*>(p)); }
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
        if (r < M && mine && base < K) raw[r].load_l2(x + static_cast<size_t>(r) * K + base);
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

// ================================================================ row kernels
//
// Rotate + quantize whole rows with a team of W warps per row (the CTA).
// Each lane holds CPL chunks of 8 consecutive values (CPL = 1, 2 or 4; one
// 16-byte bf16 load per chunk), so a lane keeps up to 32 values of its row in
// registers and the team covers K = 256 W CPL values.  The chunks of a lane
// are placed so that as many butterfly spans as possible fall inside the
// lane (RqLayout): a rotation block of G values is CB = G/8 chunks; a lane
// holds min(CB, CPL) of them, spaced LPB = CB/CPL chunks apart, so the spans
// of the chunk index's low bits cross lanes (lane distance 1 .. LPB/2) and
// those of its high bits stay in registers.  With G = 256 and CPL = 4 that is
// three in-register spans (1, 2, 4), three shuffle spans (8, 16, 32) and two
// in-register spans (64, 128), in that order: the order every butterfly of
// the transform is taken in, so the rotated values are bit-identical to a
// sequential transform whichever lane computes them.
//
// Arithmetic runs on packed fp32 pairs (add / sub / fma .f32x2, one rounding
// per element as the scalar forms): a pair holds the same element of two
// neighbouring chunks, so every butterfly span except the one between those
// two chunks is one packed add and one packed subtract per two butterflies.
//
// The transform is left unnormalised: with u the unnormalised value and k =
// log2(sqrt(G)), the rotated value is v = u 2^-k, the token scale s = fl(
// absmax(v) / Q) = fl(absmax(u) / Q) 2^-k and v / s = u / (s 2^k) exactly,
// so the codes and the stored scale are those of the normalised transform as
// long as nothing is subnormal (rows whose absmax(u) is below 2^-100 take the
// normalised path value by value).

// (a, b) -> (a + b, a - b) for two element pairs at once
__device__ __forceinline__ void f2_bfly(uint64_t& a, uint64_t& b) {
    const uint64_t s = f2_add(a, b);
    b = f2_sub(a, b);
    a = s;
}

// (lo, hi) -> (lo + hi, lo - hi) inside one pair
__device__ __forceinline__ uint64_t f2_bfly_inner(uint64_t p) {
    float lo, hi;
    f2_unpack(p, lo, hi);
    return f2_pack(lo + hi, lo - hi);
}

template <int G, int CPL>
struct RqLayout {
    static_assert(CPL == 1 || CPL == 2 || CPL == 4, "chunks per lane");
    static constexpr int CB = G == 0 ? CPL : G / 8;          // chunks per rotation block
    static constexpr int LPB = CB >= CPL ? CB / CPL : 1;     // lanes sharing a block
    static constexpr int CPBL = CB >= CPL ? CPL : CB;        // chunks of one block in a lane
    static constexpr int BPL = CPL / CPBL;                   // blocks per lane
    static_assert(LPB <= 32, "a rotation block stays inside one warp");
    // chunk (8 values) of the row held as register chunk i by team lane L of
    // TL; without rotation consecutive lanes take consecutive chunks
    __device__ __forceinline__ static int chunk(int i, int L, int TL) {
        if (G == 0) return i * TL + L;
        const int bi = i / CPBL, ji = i % CPBL;
        return ((L / LPB) * BPL + bi) * CB + ji * LPB + (L % LPB);
    }
};

// Pairs: CPL >= 2: p[8k + e] = (element e of chunk 2k, element e of chunk
// 2k + 1); CPL = 1: p[e] = (element e, element e + 4), e < 4.
template <int CPL>
struct RqPairs {
    static constexpr int N = CPL * 4;
};

// Unnormalised FWHT of the lane's values (see above for the span order).
template <int G, int CPL>
__device__ __forceinline__ void fwht_team(uint64_t (&p)[RqPairs<CPL>::N], int lane) {
    if constexpr (G != 0) {
        using Lt = RqLayout<G, CPL>;
        // spans 1, 2, 4: inside each chunk
        if constexpr (CPL >= 2) {
#pragma unroll
            for (int h = 1; h < 8; h *= 2)
#pragma unroll
                for (int k = 0; k < CPL / 2; ++k)
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        if ((e & h) == 0) f2_bfly(p[8 * k + e], p[8 * k + e + h]);
        } else {
#pragma unroll
            for (int h = 1; h < 4; h *= 2)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if ((e & h) == 0) f2_bfly(p[e], p[e + h]);
#pragma unroll
            for (int e = 0; e < 4; ++e) p[e] = f2_bfly_inner(p[e]);
        }
        // spans 8 .. 8 (LPB / 2): across lanes; the lower lane holds a, the
        // upper b: fma(+-1, own, other) is a + b or a - b, rounded once
#pragma unroll
        for (int d = 1; d < Lt::LPB; d *= 2) {
            const float sg = (lane & d) ? -1.0f : 1.0f;
            const uint64_t s2 = f2_pack(sg, sg);
#pragma unroll
            for (int q = 0; q < RqPairs<CPL>::N; ++q) {
                float lo, hi;
                f2_unpack(p[q], lo, hi);
                const float olo = __shfl_xor_sync(0xFFFFFFFFu, lo, d);
                const float ohi = __shfl_xor_sync(0xFFFFFFFFu, hi, d);
                p[q] = f2_fma(s2, p[q], f2_pack(olo, ohi));
            }
        }
        // the spans of the lane's chunk index: bit 0 inside each pair, bit 1
        // between the two pairs of chunks
        if constexpr (CPL >= 2 && Lt::CPBL >= 2) {
#pragma unroll
            for (int q = 0; q < RqPairs<CPL>::N; ++q) p[q] = f2_bfly_inner(p[q]);
        }
        if constexpr (CPL == 4 && Lt::CPBL == 4) {
#pragma unroll
            for (int e = 0; e < 8; ++e) f2_bfly(p[e], p[8 + e]);
        }
    }
}

// The 8 codes of a chunk from the bit patterns of their rounding sums (the
// code of a value is the low byte, two's complement), in the natural K order
// or with the even positions first (EVOD).
template <bool EVOD>
__device__ __forceinline__ uint2 rq_bytes8(const uint32_t (&w)[8]) {
    if (EVOD)
        return make_uint2(__byte_perm(__byte_perm(w[0], w[2], 0x0040), __byte_perm(w[4], w[6], 0x0040), 0x5410),
                          __byte_perm(__byte_perm(w[1], w[3], 0x0040), __byte_perm(w[5], w[7], 0x0040), 0x5410));
    return make_uint2(__byte_perm(__byte_perm(w[0], w[1], 0x0040), __byte_perm(w[2], w[3], 0x0040), 0x5410),
                      __byte_perm(__byte_perm(w[4], w[5], 0x0040), __byte_perm(w[6], w[7], 0x0040), 0x5410));
}

// The sums of the pairs -> the code words of every register chunk
template <int CPL, bool EVOD>
__device__ __forceinline__ void rq_pairs_to_chunks(const uint64_t* m, int k, uint2 (&cw)[CPL]) {
    uint32_t lo[8], hi[8];
    if constexpr (CPL >= 2) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float a, b;
            f2_unpack(m[e], a, b);
            lo[e] = __float_as_uint(a);
            hi[e] = __float_as_uint(b);
        }
        cw[2 * k] = rq_bytes8<EVOD>(lo);
        cw[2 * k + 1] = rq_bytes8<EVOD>(hi);
    } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float a, b;
            f2_unpack(m[e], a, b);
            lo[e] = __float_as_uint(a);
            lo[e + 4] = __float_as_uint(b);
        }
        cw[0] = rq_bytes8<EVOD>(lo);
    }
}

// The codes of a lane's values.  Fast path (rs = fl(1/s), s the scale of the
// unnormalised values): r = fma(u, rs, 1.5 2^23) rounds the exact product
// u rs to the nearest integer n and leaves n in the low byte of r's bits; d =
// fma(u, rs, -n) is u rs - n rounded once.  u rs is within 1.6e-5 of
// fl(u / s) (|u / s| <= Q + 1/2, two roundings of 2^-24), so whenever |d| <=
// 1/2 - 2^-15, n = rint(fl(u / s)), the oracle's code.  Returns whether some
// value of the lane came closer to a half-integer than that (the warp then
// recomputes with the IEEE division).  No clamp is needed: |u rs| <= Q (1 +
// 2^-23) < Q + 1/2.
template <int Q, int CPL, bool EVOD>
__device__ __forceinline__ bool rq_codes_fast(const uint64_t (&p)[RqPairs<CPL>::N], float rs,
                                              uint2 (&cw)[CPL]) {
    constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23
    const uint64_t rs2 = f2_pack(rs, rs);
    const uint64_t mg2 = f2_pack(kMagic, kMagic);
    float dmax = 0.0f;
    constexpr int G8 = CPL >= 2 ? 8 : 4;   // pairs per group of chunks
#pragma unroll
    for (int k = 0; k < RqPairs<CPL>::N / G8; ++k) {
        uint64_t m[G8];
#pragma unroll
        for (int e = 0; e < G8; ++e) {
            m[e] = f2_fma(p[G8 * k + e], rs2, mg2);
            const uint64_t nn = f2_sub(mg2, m[e]);   // -n, exact
            float dlo, dhi;
            f2_unpack(f2_fma(p[G8 * k + e], rs2, nn), dlo, dhi);
            dmax = fmaxf(dmax, fmaxf(fabsf(dlo), fabsf(dhi)));
        }
        rq_pairs_to_chunks<CPL, EVOD>(m, k, cw);
    }
    return dmax > 0.5f - 3.0517578125e-5f;
}

// The oracle's steps value by value: v = fl(u norm), q = clamp(rint(fl(v /
// s)), -Q, Q); all codes 0 for s = 0.  The fallback of the fast path (norm =
// 1, s unnormalised: fl(u / s) is then the same quotient) and the path of
// rows whose normalised scale would be subnormal.
template <int Q, int CPL, bool EVOD>
__device__ __forceinline__ void rq_codes_div(const uint64_t (&p)[RqPairs<CPL>::N], float norm, float s,
                                             uint2 (&cw)[CPL]) {
    constexpr float kMagic = 12582912.0f;
    constexpr int G8 = CPL >= 2 ? 8 : 4;
#pragma unroll
    for (int k = 0; k < RqPairs<CPL>::N / G8; ++k) {
        uint64_t m[G8];
#pragma unroll
        for (int e = 0; e < G8; ++e) {
            float lo, hi;
            f2_unpack(p[G8 * k + e], lo, hi);
            float tlo = 0.0f, thi = 0.0f;
            if (s > 0.0f) {
                tlo = fminf(fmaxf(__fdiv_rn(lo * norm, s), static_cast<float>(-Q)), static_cast<float>(Q));
                thi = fminf(fmaxf(__fdiv_rn(hi * norm, s), static_cast<float>(-Q)), static_cast<float>(Q));
            }
            m[e] = f2_pack(tlo + kMagic, thi + kMagic);
        }
        rq_pairs_to_chunks<CPL, EVOD>(m, k, cw);
    }
}

// Rows blockIdx.x, blockIdx.x + gridDim.x, ... of [0, rows), one row per
// pass of the CTA (blockDim.x / 32 warps, CPL chunks per lane, K <= 8 CPL
// blockDim.x); the next row's loads are in flight while the current one is
// transformed.  Q = 127 (int8 codes) or 7 (int4 codes); PACKED: int4 codes
// two per byte (low nibble = even K index), else one code per byte.  EVOD
// (one code per byte only): each block of 8 codes stored with its even
// positions first (0, 2, 4, 6, 1, 3, 5, 7), the order the tensor-core GEMM
// widens its weights in.
// S16: the scales are stored as IEEE fp16 (the int8 weights of the W8A8
// path in the pages' stored format, "Weight Format"): each is rounded to the
// nearest fp16 and the codes are taken against that stored scale.
template <typename InT, int G, int Q, bool PACKED, bool EVOD, int CPL, bool S16 = false>
__device__ __forceinline__ void rq_team_rows(const InT* __restrict__ in, int rows, int K,
                                             void* __restrict__ codes, void* __restrict__ scales,
                                             float (&red)[2][kQuantMaxWarps]) {
    static_assert(!(PACKED && EVOD), "even/odd order is for one code per byte");
    using Lt = RqLayout<G, CPL>;
    constexpr int NP = RqPairs<CPL>::N;
    const int TL = blockDim.x;
    const int L = threadIdx.x;
    const int lane = L & 31, warp = L >> 5, nwarps = TL >> 5;
    const int nC = K >> 3;
    // chunk of register chunk i (recomputed where used: registers are scarce)
    auto cidx = [&](int i) { return Lt::chunk(i, L, TL); };
    RawChunk<InT> raw[CPL];
    auto fetch = [&](int r) {
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            if (r < rows && cidx(i) < nC) raw[i].load(in + static_cast<size_t>(r) * K + cidx(i) * 8);
            else raw[i].zero();
        }
    };
    // 2^-k: the normalisation of the transform (exact for G = 4^j)
    constexpr float kNorm = (G == 16) ? 0.25f : (G == 64) ? 0.125f : (G == 256) ? 0.0625f : 1.0f;

    int row = static_cast<int>(blockIdx.x);
    fetch(row);
    for (int it = 0; row < rows; ++it) {
        const int nrow = row + static_cast<int>(gridDim.x);
        uint64_t p[NP];
        {
            float v[CPL][8];
#pragma unroll
            for (int i = 0; i < CPL; ++i) raw[i].to_f32(v[i]);
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                if constexpr (CPL >= 2) p[q] = f2_pack(v[2 * (q / 8)][q % 8], v[2 * (q / 8) + 1][q % 8]);
                else p[q] = f2_pack(v[0][q], v[0][q + 4]);
            }
        }
        fetch(nrow);
        fwht_team<G, CPL>(p, lane);

        float amax = 0.0f;
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            float lo, hi;
            f2_unpack(p[q], lo, hi);
            amax = fmaxf(amax, fmaxf(fabsf(lo), fabsf(hi)));
        }
#pragma unroll
        for (int d = 16; d >= 1; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, d));
        float* rb = red[it & 1];
        if (lane == 0) rb[warp] = amax;
        __syncthreads();
        amax = rb[0];
        for (int w = 1; w < nwarps; ++w) amax = fmaxf(amax, rb[w]);

        uint2 cw[CPL];
        if constexpr (!S16) {
            float scale;
            if (amax >= 0x1p-100f) {
                const float su = __fdiv_rn(amax, static_cast<float>(Q));
                scale = su * kNorm;
                const bool near = rq_codes_fast<Q, CPL, EVOD>(p, __frcp_rn(su), cw);
                if (__any_sync(0xFFFFFFFFu, near)) rq_codes_div<Q, CPL, EVOD>(p, 1.0f, su, cw);
            } else {
                // tiny or zero row: normalise first, as the oracle does
                scale = __fdiv_rn(amax * kNorm, static_cast<float>(Q));
                rq_codes_div<Q, CPL, EVOD>(p, kNorm, scale, cw);
            }
            if (L == 0) static_cast<float*>(scales)[row] = scale;
        } else {
            // the fp32 scale as above, rounded to fp16; the codes against it
            const float s32 = amax >= 0x1p-100f ? __fdiv_rn(amax, static_cast<float>(Q)) * kNorm
                                                : __fdiv_rn(amax * kNorm, static_cast<float>(Q));
            const __half h = __float2half_rn(s32);
            const float sf = __half2float(h);
            if (L == 0) static_cast<__half*>(scales)[row] = h;
            if (sf >= 0x1p-14f && sf <= 65504.0f) {
                // a normal fp16 scale: the fast path on the unnormalised values
                // (|u / su| <= Q (1 + 2^-11) < Q + 1/2: still no clamp)
                const float su = sf / kNorm;
                const bool near = rq_codes_fast<Q, CPL, EVOD>(p, __frcp_rn(su), cw);
                if (__any_sync(0xFFFFFFFFu, near)) rq_codes_div<Q, CPL, EVOD>(p, 1.0f, su, cw);
            } else {
                // subnormal, zero or infinite: value by value, clamped
                rq_codes_div<Q, CPL, EVOD>(p, kNorm, sf, cw);
            }
        }

#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            if (cidx(i) >= nC) continue;
            if constexpr (!PACKED) {
                *reinterpret_cast<uint2*>(static_cast<int8_t*>(codes) + static_cast<size_t>(row) * K +
                                          cidx(i) * 8) = cw[i];
            } else {
                // low nibble = even index, high nibble = odd index
                const uint32_t ev = __byte_perm(cw[i].x, cw[i].y, 0x6420);
                const uint32_t od = __byte_perm(cw[i].x, cw[i].y, 0x7531);
                *reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(codes) + static_cast<size_t>(row) * (K / 2) +
                                             cidx(i) * 4) =
                    (ev & 0x0F0F0F0Fu) | ((od & 0x0F0F0F0Fu) << 4);
            }
        }
        row = nrow;
    }
}

// Persistent grid over all rows (convrot_quantize_act, tint4_pack_weights,
// tint4_quantize_weights_int8, the fused linears).  Under programmatic
// dependent launch the consumer grid may start its prologue while this grid
// runs; it waits for this grid's completion before reading the codes.
// At most 80 registers per thread: with the SM's register file split between
// its four sub-partitions, 100-register warps of 3-warp CTAs fit 5 CTAs per
// SM and 12-warp CTAs only one; at 80 the QKV quantize takes 16.0 instead of
// 17.0 us and the K = 12288 one 54 instead of 69 us.  (Blocks of up to 512
// threads.)
template <typename InT, int G, int Q, bool PACKED, bool EVOD, int CPL, bool S16 = false>
__global__ void __maxnreg__(80)
rotate_quantize_rows_kernel(const InT* __restrict__ in, int rows, int K, void* __restrict__ codes,
                            void* __restrict__ scales) {
    __shared__ float red[2][kQuantMaxWarps];
    grid_launch_dependents();
    rq_team_rows<InT, G, Q, PACKED, EVOD, CPL, S16>(in, rows, K, codes, scales, red);
}

// Packed int4 activation codes [rows, K/2] (two's complement nibbles, low
// nibble = even K index) -> one int8 code per byte [rows, K] in the even/odd
// K order of the tensor-core GEMM (0, 2, 4, 6, 1, 3, 5, 7 in every block of
// 8): per packed word, the low nibbles sign-extended into the first four
// bytes, the high nibbles into the last four.  Grid-stride over 16-byte
// pieces of the packed rows (K % 32 == 0: a row is whole pieces).
__global__ void __launch_bounds__(256)
widen_int4_codes_kernel(const uint8_t* __restrict__ packed, int8_t* __restrict__ codes, long pieces) {
    grid_dependency_wait();   // the codes may come from the grid just before
    for (long i = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; i < pieces;
         i += static_cast<long>(gridDim.x) * blockDim.x) {
        const uint4 p = __ldcg(reinterpret_cast<const uint4*>(packed) + i);
        const uint32_t w[4] = {p.x, p.y, p.z, p.w};
        uint32_t o[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            // (n ^ 8) - 8 sign-extends a nibble; byte-wise, no borrow between bytes
            o[2 * j] = __vsub4((w[j] & 0x0F0F0F0Fu) ^ 0x08080808u, 0x08080808u);
            o[2 * j + 1] = __vsub4(((w[j] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u, 0x08080808u);
        }
        uint4* dst = reinterpret_cast<uint4*>(codes) + 2 * i;
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
    grid_launch_dependents();
}

}  // namespace tint4
