// w4a8_small.cuh -- the W4A8 / W4A4 ConvRot GEMM for small M (decode).
//
//   acc[m, n] = sum_k qa[m, k] * qw[n, k]            (int32, exact)
//   y[m, n]   = bf16(float(acc) * s_tok[m] * s_row[n] (+ bias[n]))
//
// "ComfyUI-INT-Crush", "Inference > INT4": packed signed int4 weights with a
// per-row scale, streamed raw and unpacked next to the integer MMA; the
// activation codes come from the rotate + quantize step (int8 for W4A8, int4
// packed two per byte for W4A4).
//
// With at most 16 tokens every weight is used at most 16 times: the cost is
// streaming the packed weights (0.5 byte each) from HBM.  The big GEMM's
// 192-token tiles would waste almost all of their tensor-core work here, so
// this kernel runs the warp-level int8 MMA (m16n8k32) with the weights as
// the A operand straight from registers and the tokens as B (n = 8 per
// block).  A nibble moves into the top half of its byte by one AND (high
// nibbles) or one shift + AND (low nibbles), which gives the int8 value
// 16 q exactly; the factor 16 (256 with int4 activations) leaves the int32
// sums by a shift.  The K order inside an MMA is permuted: each lane takes 8
// consecutive weights of a row from one packed word, even positions in its
// first k slot and odd positions in its second, and gathers the activation
// codes in the same order, which leaves each dot product unchanged.
//
// Work split (as the W4A16 kernel): one CTA per SM owns a contiguous run of
// 16-row blocks (at most kS8MB); a unit is 256 K x one block pair, a 32-row x
// 128-byte TMA box (4 KB, 128-byte swizzle; MMA row m holds weight row
// pi(m) = 4 (m & 1) + (m >> 1) (m < 8, +8 above) so that the 8 lanes of a
// load phase hit disjoint banks).  The run's units, K-chunk-major, are split
// into equal contiguous ranges, one per warp; every warp is its own TMA
// producer with a private ring of boxes.  A warp keeps its activation
// fragments for the current K chunk and its int32 sums for every block of
// the run in registers; the warps' sums meet in shared memory at the end
// (integer adds: any order gives the same bits).
//
// Group-wise weight scales (GW = 1 symmetric, 2 asymmetric; "ComfyUI-INT-
// Crush", "Weight Format": scales [out, num_groups]; stable-diffusion.cpp
// "feat: packed int4 convrot model loading and dispatch": asym_w4a8_int8):
// a half chunk (128 K) is exactly one weight group, so each half's four MMAs
// sum into a fresh int32 fragment that is scaled by the group scale of its
// row (an exact conversion: |sum| < 2^24) and added to fp32 sums; the warps'
// fp32 sums meet in shared memory in warp order.  Asymmetric nibbles q with a
// zero point z per row and group widen to the int8 value 8 (q - z): 8 q in
// bits 3-6 of each byte, plus 128 - 8 z without a carry between bytes, then
// bit 7 flipped.
#pragma once

#include <type_traits>

#include "ptx.cuh"
#include "quantize.cuh"

namespace tint4 {

constexpr int kS8Box = 32 * 128;    // one unit: 2 row blocks x 256 K of packed weights
constexpr int kS8MB = 8;            // 16-row blocks per CTA at most
constexpr int kS8MaxM = 16;         // tokens per launch
constexpr int kS8Ring = 128 * 1024;

// The int32 sums of every block of the run (kS8MB x NB x 4) and a K chunk's
// activation fragments (NB x 16 words) stay in registers: 16 warps of at most
// 128 registers for one token block, 8 warps of up to 255 for two.
template <int NB>
struct S8Cfg {
    static constexpr int WARPS = NB == 1 ? 16 : 8;
    static constexpr int THREADS = WARPS * 32;
    static constexpr int SLOTS = kS8Ring / (WARPS * kS8Box);   // boxes in flight per warp
    // ring | barriers, abort flag | epilogue operands (row scales, bias, token
    // scales of the run) | fused linear's codes | alignment slack
    static constexpr int EPI_OFF = kS8Ring + WARPS * SLOTS * 8 + 16;
    static constexpr int EPI_BYTES = kS8MB * 16 * 4 + kS8MB * 16 * 2 + kS8MaxM * 4;
    static constexpr int FUSE_OFF = EPI_OFF + EPI_BYTES;
    static constexpr int SMEM = FUSE_OFF + 1024;
    static_assert(EPI_OFF % 16 == 0 && FUSE_OFF % 16 == 0, "16-byte aligned regions");
    static_assert(WARPS * kS8MB * NB * 32 * 16 <= kS8Ring, "the reduction reuses the ring");
};

// MMA row m (0..15) of a block holds weight row s8_perm(m) of the block
__host__ __device__ constexpr int s8_perm(int m) {
    return (m & 8) | ((m & 1) << 2) | ((m >> 1) & 3);
}

__device__ __forceinline__ void mma_s8_16832(int32_t (&d)[4], const uint32_t (&a)[4],
                                             uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Group-wise weights: the scales and zero points of the CTA's whole run of
// rows (at most kS8MB blocks x 16 rows x kS8GwMaxGroups groups), one bulk copy
// each at the start, behind the ring and barriers where the fused linear
// keeps its codes (the two are never combined).  K <= 128 kS8GwMaxGroups.
constexpr int kS8GwMaxGroups = 64;
constexpr int kS8GwBytes = 16 + kS8MB * 16 * kS8GwMaxGroups * 5;

// Shared memory of the fused linear: the codes of up to kFuseMaxRows tokens
// (one per byte) and their scales, behind the ring and barriers.
constexpr int kS8FuseMaxK = 16 * kQuantChunk;   // one chunk per warp of the 16-warp CTA
constexpr int kS8FuseBytes = kFuseMaxRows * kS8FuseMaxK + 64 + kFuseMaxRows * kQuantMaxWarps * 4;

// NB 8-token blocks (M <= 8 NB <= 16); A_INT4: activation codes packed two
// per byte; OUT_I32: write the exact int32 sums instead of bf16 (test entry).
// FG, FQ (fused linear, NB = 1, M <= kFuseMaxRows, K <= kS8FuseMaxK): `act`
// is x (bf16) and the CTA rotates (group FG, 0 = none) and quantizes it (to
// [-FQ, FQ], one code per byte) into shared memory itself, while its first
// weight boxes are in flight; tok_scale is then unused.  FQ = 0: not fused.
// GW (group-wise weight scales): row_scale is then the scale matrix
// [N, K/128] and wzero (GW = 2) the zero points [N, K/128].
// S16 (group-wise only): the scales are IEEE fp16 ("ComfyUI-INT-Crush",
// "Weight Format": the stored format), copied as such and widened exactly.
template <int NB, bool A_INT4, bool OUT_I32, int FG = 0, int FQ = 0, int GW = 0, bool S16 = false>
__global__ void __launch_bounds__(S8Cfg<NB>::THREADS, 1)
w4a8_small_kernel(const __grid_constant__ CUtensorMap tmap_w, const uint8_t* __restrict__ act,
                  const float* __restrict__ tok_scale, const float* __restrict__ row_scale,
                  const __nv_bfloat16* __restrict__ bias, void* __restrict__ out, int M, int N,
                  int K, uint32_t hi_mask, int early_weights, uint64_t wait_ns,
                  const uint8_t* __restrict__ wzero) {
    constexpr bool FUSED = FQ != 0;
    static_assert(!FUSED || (NB == 1 && !A_INT4 && !OUT_I32), "fused: int8 codes, bf16 out, <= 8 tokens");
    static_assert(GW == 0 || (!FUSED && !A_INT4 && !OUT_I32), "group-wise: int8 codes, bf16 out");
    using Acc = typename std::conditional<GW != 0, float, int32_t>::type;
    constexpr float kGwUnscale = GW == 2 ? 0.125f : 0.0625f;   // the unpack's 8 x / 16 x
    const int ngr = K / 128;                                    // weight groups per row
    using C = S8Cfg<NB>;
    constexpr int kS8Warps = C::WARPS, kS8Slots = C::SLOTS, kS8Threads = C::THREADS;
    extern __shared__ uint8_t s8_smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(s8_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full_all = reinterpret_cast<uint64_t*>(sm + kS8Ring);
    volatile uint32_t* abort_flag =
        reinterpret_cast<volatile uint32_t*>(full_all + kS8Warps * kS8Slots);
    Acc* red = reinterpret_cast<Acc*>(sm);   // reused after the main loop

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2;   // MMA group id: MMA rows g / g + 8, token column g
    const int t = lane & 3;    // which 32-value slice of a 128-K half chunk
    const int nchunks = (K + 255) / 256;
    const int nblk = N / 16;
    int b0, b1;   // this CTA's run of blocks (32-bit arithmetic: 64-bit division is a long
    even_split(nblk, gridDim.x, blockIdx.x, b0, b1);   // software routine on the prologue's path)
    const int nb = b1 - b0;             // 1..kS8MB (the host sizes the grid)
    const int nbp = (nb + 1) / 2;       // block pairs (an odd run's last box reads 16 rows it skips)
    const int rA = s8_perm(g), rB = s8_perm(g + 8);
    const int swz = rA & 7;             // = rB & 7

    // the run's units in chunk-major order, u = P * nbp + bp; this warp's range
    const int ntot = nchunks * nbp;
    int u0, u1;
    even_split(ntot, kS8Warps, warp, u0, u1);
    const int nunits = u1 - u0;
    uint64_t* full = full_all + warp * kS8Slots;
    uint8_t* ring = sm + warp * kS8Slots * kS8Box;

    if (lane == 0) {
        for (int i = 0; i < kS8Slots; ++i) mbar_init(&full[i], 1);
        if (warp == 0) *abort_flag = 0u;
        fence_mbarrier_init();
        prefetch_tensormap(&tmap_w);
    }
    __syncthreads();

    int issued = 0;
    auto issue = [&](int i) {
        const int slot = i % kS8Slots;
        const int P = (u0 + i) / nbp;
        const int bp = (u0 + i) % nbp;
        mbar_arrive_expect_tx(&full[slot], kS8Box);
        tma_load_2d(&tmap_w, &full[slot], ring + slot * kS8Box, P * 128, (b0 + 2 * bp) * 16);
    };
    // The weights may start streaming before the previous kernel of the
    // stream has finished only when the caller said they are not written by
    // it (tint4_set_decode_weight_prefetch); everything else waits for it.
    // One box per warp first, the rest once the first activation fragments
    // are in: every warp's first box then reaches the front of the memory
    // queues.
    if (early_weights && lane == 0 && issued < nunits) issue(issued++);
    grid_dependency_wait();
    grid_launch_dependents();
    if (lane == 0 && issued == 0 && nunits > 0) issue(issued++);

    // group-wise: the run's scales (and zero points), contiguous in global
    // memory, by two bulk copies completing on their own barrier
    uint64_t* gw_bar = reinterpret_cast<uint64_t*>(sm + C::FUSE_OFF);
    const float* sGwScale = reinterpret_cast<const float*>(sm + C::FUSE_OFF + 16);
    const uint8_t* sGwZero = sm + C::FUSE_OFF + 16 + kS8MB * 16 * kS8GwMaxGroups * 4;
    if constexpr (GW != 0) {
        if (threadIdx.x == 0) {
            mbar_init(gw_bar, 1);
            fence_mbarrier_init();
            const uint32_t nsc = static_cast<uint32_t>(nb * 16 * ngr);
            constexpr uint32_t kSB = S16 ? 2u : 4u;   // bytes per scale
            mbar_arrive_expect_tx(gw_bar, nsc * kSB + (GW == 2 ? nsc : 0u));
            bulk_load_1d(const_cast<float*>(sGwScale),
                         reinterpret_cast<const uint8_t*>(row_scale) + static_cast<size_t>(b0) * 16 * ngr * kSB,
                         nsc * kSB, gw_bar);
            if (GW == 2)
                bulk_load_1d(const_cast<uint8_t*>(sGwZero), wzero + static_cast<size_t>(b0) * 16 * ngr,
                             nsc, gw_bar);
        }
        __syncthreads();   // the barrier is initialised before anyone waits on it
    }

    // The epilogue's operands of this run go to shared memory now, while the
    // first weight boxes are in flight: read from global memory at the end
    // they would add a memory round trip to every launch.  Through L2 (the
    // token scales may come from the grid just before; see ld_scale).
    float* sRowScale = reinterpret_cast<float*>(sm + C::EPI_OFF);
    __nv_bfloat16* sBias = reinterpret_cast<__nv_bfloat16*>(sm + C::EPI_OFF + kS8MB * 16 * 4);
    float* sTok = reinterpret_cast<float*>(sm + C::EPI_OFF + kS8MB * 16 * 6);
    if constexpr (!OUT_I32) {
        const int tid = threadIdx.x;
        if (GW == 0 && tid < nb * 16) sRowScale[tid] = __ldcg(row_scale + b0 * 16 + tid);
        if (bias != nullptr && tid < nb * 8)
            reinterpret_cast<unsigned*>(sBias)[tid] =
                __ldcg(reinterpret_cast<const unsigned*>(bias + b0 * 16) + tid);
        if (!FUSED && tid < M) sTok[tid] = __ldcg(tok_scale + tid);
    }

    // fused linear: x -> codes and scales in shared memory, under the first boxes
    uint8_t* sfuse = sm + C::FUSE_OFF;
    const int8_t* sCodes = reinterpret_cast<const int8_t*>(sfuse);
    const float* sTokScale = reinterpret_cast<const float*>(sfuse + kFuseMaxRows * kS8FuseMaxK);
    if constexpr (FUSED) {
        rotate_quantize_rows_to_smem<FG, FQ>(
            reinterpret_cast<const __nv_bfloat16*>(act), M, K, reinterpret_cast<int8_t*>(sfuse),
            reinterpret_cast<float*>(sfuse + kFuseMaxRows * kS8FuseMaxK),
            *reinterpret_cast<float(*)[kFuseMaxRows][kQuantMaxWarps]>(sfuse + kFuseMaxRows * kS8FuseMaxK + 64));
    }

    Acc total[kS8MB][NB][4];
#pragma unroll
    for (int j = 0; j < kS8MB; ++j)
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int q = 0; q < 4; ++q) total[j][b][q] = Acc(0);

    bool gw_failed = false;
    if constexpr (GW != 0) {
        if (!warp_wait(gw_bar, 0, abort_flag, wait_ns, kDevErrTimeoutConsumer)) gw_failed = true;
    }
    int consumed = 0, cslot = 0;
    uint32_t cphase = 0u;
    bool aborted = gw_failed;
    const int P0 = u0 / nbp, P1 = nunits > 0 ? (u1 - 1) / nbp : P0 - 1;
    for (int P = P0; P <= P1 && !aborted; ++P) {
        const int bp_lo = P == P0 ? u0 % nbp : 0;                 // this warp's block pairs of chunk P
        const int bp_hi = P == P1 ? (u1 - 1) % nbp + 1 : nbp;
        // activation fragments of chunk P: token 8b + g, K positions
        // 256 P + 128 h + 32 t + 8 i + {0, 2, 4, 6} (first slot) and + {1, 3, 5, 7}
        // (second slot) of MMA i of half h; zeros for tokens >= M and K >= K
        uint32_t bfr[2][NB][4][2];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                const int tok = 8 * b + g;
                const int kb = 256 * P + 128 * h + 32 * t;   // K % 32 == 0: a slice is all in or all out
                if (tok < M && kb < K) {
                    if constexpr (A_INT4) {
                        const uint4 c = __ldcg(reinterpret_cast<const uint4*>(
                            act + static_cast<size_t>(tok) * (K / 2) + kb / 2));
                        const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            bfr[h][b][i][0] = (cw[i] << 4) & hi_mask;   // 16 x even positions
                            bfr[h][b][i][1] = cw[i] & hi_mask;          // 16 x odd positions
                        }
                    } else {
                        uint4 c0, c1;
                        if constexpr (FUSED) {
                            c0 = lds128(reinterpret_cast<const uint8_t*>(sCodes) + tok * K + kb);
                            c1 = lds128(reinterpret_cast<const uint8_t*>(sCodes) + tok * K + kb + 16);
                        } else {
                            const uint4* ar = reinterpret_cast<const uint4*>(act + static_cast<size_t>(tok) * K + kb);
                            c0 = __ldcg(ar);
                            c1 = __ldcg(ar + 1);
                        }
                        const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            bfr[h][b][i][0] = __byte_perm(cw[2 * i], cw[2 * i + 1], 0x6420);
                            bfr[h][b][i][1] = __byte_perm(cw[2 * i], cw[2 * i + 1], 0x7531);
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i) bfr[h][b][i][0] = bfr[h][b][i][1] = 0u;
                }
            }
        if (lane == 0)
            for (; issued < kS8Slots && issued < nunits; ++issued) issue(issued);
#pragma unroll
        for (int bp = 0; bp < kS8MB / 2; ++bp) {
            if (bp >= bp_hi) break;   // warp-uniform
            if (bp < bp_lo) continue;
            // group-wise: the scales (and zero points) of this unit's rows and
            // two groups, from the run's copy in shared memory
            float gsc[2][2][2] = {};         // [block of the pair][half][row A / B]
            uint32_t gzc[2][2][2] = {};      // (128 - 8 z) in every byte
            if constexpr (GW != 0) {
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {
                    const int j = 2 * bp + hb;
                    if (j >= nb) break;
                    const int ra = (j * 16 + rA) * ngr + 2 * P;
                    const int rb = (j * 16 + rB) * ngr + 2 * P;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (256 * P + 128 * h >= K) break;   // a half past K (its sums are 0)
                        if constexpr (S16) {
                            const __half* s16 = reinterpret_cast<const __half*>(sGwScale);
                            gsc[hb][h][0] = __half2float(s16[ra + h]) * kGwUnscale;
                            gsc[hb][h][1] = __half2float(s16[rb + h]) * kGwUnscale;
                        } else {
                            gsc[hb][h][0] = sGwScale[ra + h] * kGwUnscale;
                            gsc[hb][h][1] = sGwScale[rb + h] * kGwUnscale;
                        }
                        if constexpr (GW == 2) {
                            gzc[hb][h][0] = (128u - 8u * sGwZero[ra + h]) * 0x01010101u;
                            gzc[hb][h][1] = (128u - 8u * sGwZero[rb + h]) * 0x01010101u;
                        }
                    }
                }
            }
            const int slot = cslot;
            if (!warp_wait(&full[slot], cphase, abort_flag, wait_ns, kDevErrTimeoutConsumer)) {
                aborted = true;
                break;
            }
            const uint8_t* box = ring + slot * kS8Box;
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
                const int j = 2 * bp + hb;         // block of the run
                if (j >= nb) break;                // CTA-uniform
                const uint8_t* bbox = box + hb * 16 * 128;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    // this lane's 16-byte chunk of half h in rows rA / rB (swizzled)
                    const int coff = ((4 * h + t) ^ swz) << 4;
                    const uint4 pa = *reinterpret_cast<const uint4*>(bbox + rA * 128 + coff);
                    const uint4 pb = *reinterpret_cast<const uint4*>(bbox + rB * 128 + coff);
                    const uint32_t wa[4] = {pa.x, pa.y, pa.z, pa.w};
                    const uint32_t wb[4] = {pb.x, pb.y, pb.z, pb.w};
                    if constexpr (GW == 0) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            // word i: 8 consecutive weights; low nibbles = even positions
                            uint32_t a[4];
                            a[0] = (wa[i] << 4) & hi_mask;   // MMA row g,   first slot
                            a[1] = (wb[i] << 4) & hi_mask;   // MMA row g+8, first slot
                            a[2] = wa[i] & hi_mask;          // MMA row g,   second slot
                            a[3] = wb[i] & hi_mask;          // MMA row g+8, second slot
#pragma unroll
                            for (int b = 0; b < NB; ++b)
                                mma_s8_16832(total[j][b], a, bfr[h][b][i][0], bfr[h][b][i][1]);
                        }
                    } else {
                        // half h is weight group 2 P + h: its own int32 sums, then
                        // scaled into the fp32 totals
                        int32_t part[NB][4];
#pragma unroll
                        for (int b = 0; b < NB; ++b)
#pragma unroll
                            for (int q = 0; q < 4; ++q) part[b][q] = 0;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            uint32_t a[4];
                            if constexpr (GW == 2) {
                                const uint32_t za = gzc[hb][h][0], zb = gzc[hb][h][1];
                                a[0] = (((wa[i] << 3) & 0x78787878u) + za) ^ 0x80808080u;
                                a[1] = (((wb[i] << 3) & 0x78787878u) + zb) ^ 0x80808080u;
                                a[2] = (((wa[i] >> 1) & 0x78787878u) + za) ^ 0x80808080u;
                                a[3] = (((wb[i] >> 1) & 0x78787878u) + zb) ^ 0x80808080u;
                            } else {
                                a[0] = (wa[i] << 4) & hi_mask;
                                a[1] = (wb[i] << 4) & hi_mask;
                                a[2] = wa[i] & hi_mask;
                                a[3] = wb[i] & hi_mask;
                            }
#pragma unroll
                            for (int b = 0; b < NB; ++b)
                                mma_s8_16832(part[b], a, bfr[h][b][i][0], bfr[h][b][i][1]);
                        }
                        // fragment: [0], [1] row g (A), [2], [3] row g + 8 (B); exact
                        // conversions (|sum| < 2^24), one rounding per FMA
#pragma unroll
                        for (int b = 0; b < NB; ++b)
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                total[j][b][q] = __fmaf_rn(gsc[hb][h][q >> 1],
                                                           static_cast<float>(part[b][q]),
                                                           total[j][b][q]);
                    }
                }
            }
            ++consumed;
            if (++cslot == kS8Slots) { cslot = 0; cphase ^= 1u; }
            // the slot is free again: refill it with this warp's unit kS8Slots ahead
            __syncwarp();
            if (lane == 0 && issued < nunits) {
                fence_proxy_async_smem();
                issue(issued);
                ++issued;
            }
        }
    }
    if (aborted && lane == 0) {
        // let this warp's copies in flight land before the ring is reused
        uint32_t never = 0u;
        for (int i = consumed; i < issued; ++i)
            (void)mbar_wait_bounded(&full[i % kS8Slots], (i / kS8Slots) & 1, &never, wait_ns, 0u);
    }

    // ---- the warps' partial sums meet in shared memory
    if constexpr (GW != 0) {
        // the run's scale copy has landed before the CTA can finish
        uint32_t never = 0u;
        if (threadIdx.x == 0) (void)mbar_wait_bounded(gw_bar, 0, &never, wait_ns, 0u);
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kS8MB; ++j) {
        if (j >= nb) break;
#pragma unroll
        for (int b = 0; b < NB; ++b)
            if constexpr (GW != 0)
                *reinterpret_cast<float4*>(red + (((warp * kS8MB + j) * NB + b) * 32 + lane) * 4) =
                    make_float4(total[j][b][0], total[j][b][1], total[j][b][2], total[j][b][3]);
            else
                *reinterpret_cast<int4*>(red + (((warp * kS8MB + j) * NB + b) * 32 + lane) * 4) =
                    make_int4(total[j][b][0], total[j][b][1], total[j][b][2], total[j][b][3]);
    }
    __syncthreads();
    if (*abort_flag) return;   // the device error word says why; the output is left as it was
    constexpr int kShift = A_INT4 ? 8 : 4;                 // the sums carry 16 (or 256) x
    constexpr float kUnscale = A_INT4 ? 1.0f / 256.0f : 1.0f / 16.0f;
    for (int e = threadIdx.x; e < nb * NB * 32; e += kS8Threads) {
        const int ln = e & 31;
        const int b = (e >> 5) % NB;
        const int j = (e >> 5) / NB;
        Acc v[4] = {Acc(0), Acc(0), Acc(0), Acc(0)};
#pragma unroll
        for (int w = 0; w < kS8Warps; ++w) {   // in warp order (fp32 sums: a fixed order)
            const Acc* p = red + (((w * kS8MB + j) * NB + b) * 32 + ln) * 4;
            v[0] += p[0]; v[1] += p[1]; v[2] += p[2]; v[3] += p[3];
        }
        const int gg = ln >> 2, tt = ln & 3;
        const int tok0 = 8 * b + 2 * tt;
        const int l0 = j * 16 + s8_perm(gg), l1 = j * 16 + s8_perm(gg + 8);   // rows of the run
        const int r0 = b0 * 16 + l0, r1 = b0 * 16 + l1;
        // v: [0] row r0 / token tok0, [1] r0 / tok0 + 1, [2] r1 / tok0, [3] r1 / tok0 + 1
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int tok = tok0 + (q & 1);
            const int row = (q & 2) ? r1 : r0;
            const int lrow = (q & 2) ? l1 : l0;
            if (tok >= M) continue;
            if constexpr (OUT_I32) {
                reinterpret_cast<int32_t*>(out)[static_cast<size_t>(tok) * N + row] =
                    static_cast<int32_t>(v[q]) >> kShift;
            } else if constexpr (GW != 0) {
                const float bsv = bias ? __bfloat162float(sBias[lrow]) : 0.0f;
                reinterpret_cast<__nv_bfloat16*>(out)[static_cast<size_t>(tok) * N + row] =
                    __float2bfloat16_rn(__fmaf_rn(v[q], sTok[tok], bsv));
            } else {
                const float bsv = bias ? __bfloat162float(sBias[lrow]) : 0.0f;
                const float st = FUSED ? sTokScale[tok] : sTok[tok];
                const float val = static_cast<float>(v[q]) * st *
                                  (sRowScale[lrow] * kUnscale) + bsv;
                reinterpret_cast<__nv_bfloat16*>(out)[static_cast<size_t>(tok) * N + row] =
                    __float2bfloat16_rn(val);
            }
        }
    }
}

}  // namespace tint4
