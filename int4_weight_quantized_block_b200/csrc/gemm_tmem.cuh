// gemm_tmem.cuh -- persistent GEMM with the unpacked weights in tensor memory
// (packed int4 activation codes), or int8 weights from shared memory (W8A8);
// shared-stage pipeline.  The int8-code x packed-int4-weight form, the fused
// linears' GEMM, is gemm_wide.cuh; the MMA helpers here serve it too.
//
//   acc[m, n] = sum_k qa[m, k] * qw[n, k]            (int32, exact)
//   y[m, n]   = bf16( acc * s_tok[m] * s_row[n] (+ bias[n]) )
//
// "ComfyUI-INT-Crush", "Inference > INT4 > CUDA backend": INT4 weights are
// unpacked to INT8 and run through an INT8 GEMM with fused dequant;
// stable-diffusion.cpp "feat: packed int4 convrot model loading and
// dispatch", "Summary": the packed nibbles stay packed in memory (about half a
// byte per weight).
//
// Shape of the product on the tensor core: the weights are the MMA's M side
// (128 rows = the 128 TMEM lanes) and the tokens its N side (192 per tile).
// Per 128-wide K step the TMA brings one activation tile (192 tokens x 128
// int8 codes, 128-byte swizzle: the MMA's B operand; or the packed int4 codes
// the unpack warps widen into it) and one weight tile (packed: 128 rows x 64
// bytes, 64-byte swizzle; int8: 128 x 128 bytes, the A operand from shared
// memory) into one shared-memory stage.  For packed weights each of 128
// unpack threads owns one weight row: it reads its 64 packed bytes
// (bank-conflict-free thanks to the swizzle), widens every nibble to an int8
// (x16, see below) and writes the 128 K values with one tcgen05.st into a
// TMEM A-operand stage.
//
// The CTA is persistent (one per SM) and walks a static list of 128 x 192
// tiles.  Warp roles (18 warps):
//   warp 0      TMA producer (4-deep ring of shared-memory stages)
//   warp 1      TMEM owner; one thread issues tcgen05.mma.cta_group::1.kind::i8
//               (A from TMEM or shared memory, B from shared memory, M 128,
//               N 192, K 32)
//   warps 2-9   unpack into the 4 TMEM A stages (32 columns each); warps 2-5
//               take the even K steps and warps 6-9 the odd ones, so two
//               chains run side by side on every SM sub-partition (each warp
//               may only reach its quarter of the TMEM lanes, warp % 4)
//   warps 10-17 epilogue: tcgen05.ld of one accumulator buffer while the MMAs
//               fill the other (two 192-column int32 buffers); two warps per
//               TMEM lane quarter, each on half of the tokens.  A thread holds
//               one weight row (= one output column), so it scales its values,
//               rounds them to bf16 and writes them with 2-byte shared-memory
//               stores into a [192 tokens][128 columns] staging tile, which the
//               8 warps then copy to y (row-major [M, N]) in 16-byte row pieces
//               (a TMA tensor store of the tile shared the copy engine with the
//               mainloop's loads and cost about 15 %).  The tile's token
//               scales are copied to shared memory while its MMAs run.
// TMEM columns: accumulators at 0 and 192, A stages at 384 + 32 s.
//
// A nibble moved into the high half of its byte, low half cleared, is the
// int8 value 16 * code; the accumulators hold 16 * acc and the epilogue
// shifts back exactly (|16 acc| < 2^31 for K <= 65536).
//
// W4A4 with packed activation codes (A_INT4): the TMA brings the packed
// activation tile (192 tokens x 64 bytes) into a staging area, and the
// unpack warps also widen it (x16 again, natural K order) into the swizzled
// int8 B tile before they signal the stage: the accumulators then hold
// 256 * acc (|256 acc| < 2^31 for K <= 65536 with codes in [-7, 7]).
//
// Even/odd K order (EVOD, and always for A_INT4): a packed word holds 8 K
// values, the even ones in its low nibbles and the odd ones in its high
// nibbles.  Widened as (w << 4) & 0xF0F0F0F0 and w & 0xF0F0F0F0 it gives
// the K order 0, 2, 4, 6, 1, 3, 5, 7 in every block of 8 at no extra cost,
// where the natural order needs two byte permutes more per word.  A dot
// product over K does not depend on the order as long as both operands use
// the same one: the fused linears store their int8 activation codes in that
// order (rotate_quantize_rows with EVOD), and the W4A4 form widens both
// operands from packed nibbles in the kernel.
#pragma once

#include "ptx.cuh"

namespace tint4 {

constexpr int kTmBM = 128;       // weight rows per tile (UMMA M, TMEM lanes)
constexpr int kTmBK = 128;       // K values per stage
constexpr int kTmStages = 4;     // TMEM A stages
constexpr int kTmThreads = 576;  // 18 warps
constexpr int kTmWBytes = kTmBM * kTmBK / 2;          // 8 KB packed weights per stage
constexpr int kTmW8Bytes = kTmBM * kTmBK;             // 16 KB int8 weights per stage (W8A8)

// Tile shape and ring of the two forms: 192 tokens, two accumulator buffers,
// 4 shared-memory stages (the packed-code staging or the int8 weight tile
// leave no room for a fifth).
template <bool A_INT4, bool W8>
struct TmCfg {
    static_assert(A_INT4 || W8, "int8 codes x packed int4 weights run w4a8_wide_gemm_kernel");
    static constexpr int BN = 192;                         // tokens per tile (UMMA N)
    static constexpr int NBUF = 2;                         // accumulator buffers
    static constexpr int S = 4;                            // shared-memory stages
    static constexpr int ACT = BN * kTmBK;                 // int8 codes per stage
    static constexpr int ACTP = A_INT4 ? BN * kTmBK / 2 : 0;   // packed int4 codes per stage
    static constexpr int WB = W8 ? kTmW8Bytes : kTmWBytes;
    static constexpr int OUT = BN * kTmBM * 2;             // bf16 staging tile
    static constexpr int SMEM = S * (ACT + WB + ACTP) + OUT + 256 + BN * 4 + 1024;
    static constexpr uint32_t COL_A = NBUF * BN;           // A stage s at COL_A + 32 s
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    static_assert(COL_A + 32 * kTmStages <= 512, "TMEM budget");
    static_assert(ACT % 1024 == 0 && kTmWBytes % 1024 == 0, "swizzled stage alignment");
};
constexpr uint32_t kTmColD = 0;                       // accumulator buffer b at b * BN

// The weight matrices one launch multiplies the same activation codes with:
// one for a plain GEMM, up to kTmMaxGroups for a grouped one (separate Q, K,
// V projections of one input, say).  The tile list runs group after group:
// tiles [tile_end[g-1], tile_end[g]) belong to group g.
constexpr int kTmMaxGroups = 4;
struct TmGroups {
    CUtensorMap w[kTmMaxGroups];              // packed weights [N_g, K/2]
    const float* row_scale[kTmMaxGroups];     // [N_g]
    const __nv_bfloat16* bias[kTmMaxGroups];  // [N_g] or null
    void* out[kTmMaxGroups];                  // y_g [M, N_g] (bf16, or int32 sums)
    int N[kTmMaxGroups];
    int tile_end[kTmMaxGroups];
    int count;
};

__device__ __forceinline__ void umma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The four K-32 MMAs of one 128-wide K step in one asm block: one predicate
// for the step's first MMA (overwrite at the start of a tile), the others
// accumulate; fewer instructions on the issuing thread, whose time per step
// paces the tensor pipe.  TS: A from TMEM columns a, a+8, a+16, a+24.
__device__ __forceinline__ void umma_i8_ts_step(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.b32 q, %4, %4;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%5], %6, %3, q;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%7], %8, %3, q;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%9], %10, %3, q;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(a_tmem + 8), "l"(b_desc + 2),
        "r"(a_tmem + 16), "l"(b_desc + 4), "r"(a_tmem + 24), "l"(b_desc + 6)
        : "memory");
}

// SS: A from shared memory (descriptor advancing 32 bytes = 2 units per MMA)
__device__ __forceinline__ void umma_i8_ss_step(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.b32 q, %4, %4;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %5, %6, %3, q;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %7, %8, %3, q;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %9, %10, %3, q;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "l"(a_desc + 2), "l"(b_desc + 2),
        "l"(a_desc + 4), "l"(b_desc + 4), "l"(a_desc + 6), "l"(b_desc + 6)
        : "memory");
}

// W8: the weights are int8 codes already (W8A8): the TMA brings a 128 x 128
// int8 tile (128-byte swizzle) and the MMA reads it from shared memory as its
// A operand (kind::i8, both operands in shared memory); no unpack, no x16.
// EVOD: the int8 activation codes are stored in the even/odd K order.
// S16: the row scales are IEEE fp16 (the stored format of "ComfyUI-INT-
// Crush", "Weight Format"), widened exactly in the epilogue.
template <bool OUT_I32, bool A_INT4, bool W8 = false, bool EVOD = false, bool S16 = false>
__global__ void __launch_bounds__(kTmThreads, 1)
w4a8_tmem_gemm_kernel(const __grid_constant__ CUtensorMap tmap_act,
                      const __grid_constant__ TmGroups grp,
                      const float* __restrict__ tok_scale, int M, int K, uint64_t wait_ns) {
    static_assert(!(W8 && A_INT4), "int8 weights run with int8 activation codes");
    static_assert(!(W8 && EVOD), "int8 weights are stored in the natural K order");
    constexpr bool kEvod = EVOD || A_INT4;   // widen in the even/odd K order
    constexpr int kWB = W8 ? kTmW8Bytes : kTmWBytes;   // weight bytes per stage
    using C = TmCfg<A_INT4, W8>;
    constexpr int kBN = C::BN;                          // tokens per tile
    constexpr int kS = C::S;                            // shared-memory stages
    constexpr int kT = kTmStages;                       // TMEM A stages
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sAct = smem;
    uint8_t* sW = smem + kS * C::ACT;
    uint8_t* sActP = sW + kS * kWB;                                    // A_INT4 only
    uint8_t* sOut = sActP + kS * C::ACTP;
    uint64_t* act_full = reinterpret_cast<uint64_t*>(sOut + C::OUT);
    uint64_t* empty = act_full + kS;               // [kS] stage consumed by the MMAs (commit)
    uint64_t* a_full = empty + kS;                 // [kT] TMEM A stage written (one arrival per warp)
    uint64_t* acc_full = a_full + kT;              // [2] accumulator ready (commit)
    uint64_t* acc_empty = acc_full + 2;            // [2] accumulator drained (8 warp arrivals)
    uint64_t* final_bar = acc_empty + 2;           // all MMAs done (teardown)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;
    volatile uint32_t* epi_go = tmem_slot + 2;     // epilogue: proceed with this tile
    float* sTok = reinterpret_cast<float*>(sOut + C::OUT + 256);   // the tile's token scales

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int m_tiles = (M + kBN - 1) / kBN;
    const int n_work = grp.tile_end[grp.count - 1];
    const int KT = (K + kTmBK - 1) / kTmBK;
    const int my_tiles = (blockIdx.x < n_work) ? (n_work - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    // tile -> (group, first token, first weight row of the group)
    struct TileAt {
        int g, m0, n0;
    };
    auto tile_at = [&](int tile) -> TileAt {
        int g = 0;
#pragma unroll
        for (int h = 0; h < kTmMaxGroups - 1; ++h)
            if (h + 1 < grp.count && tile >= grp.tile_end[h]) g = h + 1;
        const int t = tile - (g > 0 ? grp.tile_end[g - 1] : 0);
        return TileAt{g, (t % m_tiles) * kBN, (t / m_tiles) * kTmBM};
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kS; ++s) {
            mbar_init(&act_full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int t = 0; t < kT; ++t) mbar_init(&a_full[t], 4);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 8);
        }
        mbar_init(final_bar, 1);
        *abort_flag = 0u;
        fence_mbarrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmap_act);
        for (int g = 0; g < grp.count; ++g) prefetch_tensormap(&grp.w[g]);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tcgen05_fence_before();
    __syncthreads();
    tcgen05_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // the codes and token scales may come from the grid launched just before
    grid_dependency_wait();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t c = 0;
            int issued = 0;
            for (int i = 0; i < my_tiles && !*abort_flag; ++i) {
                const TileAt ta = tile_at(blockIdx.x + i * gridDim.x);
                const int m0 = ta.m0, n0 = ta.n0;
                const CUtensorMap* tmap_w = &grp.w[ta.g];
                for (int kt = 0; kt < KT; ++kt, ++c) {
                    const int s = c % kS;
                    const uint32_t ph = (c / kS) & 1;
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, wait_ns,
                                           kDevErrTimeoutProducer))
                        break;
                    if (A_INT4) {
                        mbar_arrive_expect_tx(&act_full[s], C::ACTP + kTmWBytes);
                        tma_load_2d(&tmap_act, &act_full[s], sActP + s * C::ACTP, kt * (kTmBK / 2), m0);
                    } else {
                        mbar_arrive_expect_tx(&act_full[s], C::ACT + kWB);
                        tma_load_2d(&tmap_act, &act_full[s], sAct + s * C::ACT, kt * kTmBK, m0);
                    }
                    tma_load_2d(tmap_w, &act_full[s], sW + s * kWB, kt * (W8 ? kTmBK : kTmBK / 2), n0);
                    ++issued;
                }
            }
            if (*abort_flag) {
                uint32_t never = 0u;
                const int first = issued > kS ? issued - kS : 0;
                for (int j = first; j < issued; ++j)
                    (void)mbar_wait_bounded(&act_full[j % kS], (j / kS) & 1, &never,
                                            wait_ns, 0u);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_i8(kTmBM, kBN);
            // B descriptors: stage s starts (s * bytes) / 16 units above stage 0,
            // MMA kk of a stage 32 bytes = 2 units further (the address field
            // cannot carry: shared addresses are below 2^18)
            const uint64_t bdesc0 = umma_desc_sw128(smem_u32(sAct));
            const uint64_t adesc0 = umma_desc_sw128(smem_u32(sW));   // W8 only
            static_assert(kTmBK == 4 * 32, "four MMAs per K step");
            // ring positions, advanced per step: shared-memory stage s (phase
            // sph) and TMEM stage t (phase tph)
            int s = 0, t = 0;
            uint32_t sph = 0u, tph = 0u;
            bool ok = true;
            for (int i = 0; i < my_tiles && ok; ++i) {
                const int buf = i & 1;
                const uint32_t aph = (i >> 1) & 1;
                if (!mbar_wait_bounded(&acc_empty[buf], aph ^ 1, abort_flag, wait_ns,
                                       kDevErrTimeoutConsumer)) {
                    ok = false;
                    break;
                }
                tcgen05_fence_after();
                const uint32_t d_tmem = tmem_base + kTmColD + buf * kBN;
                for (int kt = 0; kt < KT; ++kt) {
                    // a_full implies the stage has landed: the unpack warps arrive
                    // on it only after they have seen it (one wait per stage: the
                    // issuing thread's time per stage is the tensor pipe's budget);
                    // int8 weights need no unpack: the landing itself
                    const bool ready =
                        W8 ? mbar_wait_bounded(&act_full[s], sph, abort_flag, wait_ns,
                                               kDevErrTimeoutConsumer)
                           : mbar_wait_bounded(&a_full[t], tph, abort_flag, wait_ns,
                                               kDevErrTimeoutConsumer);
                    if (!ready) {
                        ok = false;
                        break;
                    }
                    tcgen05_fence_after();
                    const uint32_t a_tmem = tmem_base + C::COL_A + 32 * t;
                    const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(s * (C::ACT >> 4));
                    const uint64_t adesc = adesc0 + static_cast<uint64_t>(s * (kTmW8Bytes >> 4));
                    if constexpr (W8) umma_i8_ss_step(d_tmem, adesc, bdesc, idesc, kt);
                    else umma_i8_ts_step(d_tmem, a_tmem, bdesc, idesc, kt);
                    umma_commit(&empty[s]);
                    if (++s == kS) {
                        s = 0;
                        sph ^= 1u;
                    }
                    if (++t == kT) {
                        t = 0;
                        tph ^= 1u;
                    }
                }
                if (ok) umma_commit(&acc_full[buf]);
            }
            // everything issued lands before TMEM is released
            umma_commit(final_bar);
            uint32_t never = 0u;
            (void)mbar_wait_bounded(final_bar, 0, &never, wait_ns, 0u);
        }
        __syncwarp();   // lanes 1-31 park here instead of polling a barrier
    } else if (warp < 10) {
        // ------------------------------------------------ weight unpack -> TMEM (warps 2-9)
        if constexpr (!W8) {   // int8 weights: nothing to widen
            const int q = warp & 3;                 // TMEM lane quarter
            const int r = q * 32 + lane;            // weight row within the tile
            const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
            const int total = my_tiles * KT;        // K steps this CTA runs
            // 64-byte swizzle of the TMA tile: chunk v of row r sits at chunk
            // v ^ ((r >> 1) & 3); 8 consecutive rows then hit 8 distinct bank groups
            const int sw = (r >> 1) & 3;
            for (int j = (warp < 6 ? 0 : 1); j < total; j += 2) {
                const int s = j % kS, t = j % kT;
                if (!warp_wait(&act_full[s], (j / kS) & 1, abort_flag, wait_ns,
                               kDevErrTimeoutConsumer))
                    break;
                const uint8_t* row = sW + s * kTmWBytes + r * 64;
                uint32_t a[32];
    #pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint4 p = lds128(row + 16 * (v ^ sw));
                    const uint32_t w4[4] = {p.x, p.y, p.z, p.w};
    #pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        if constexpr (kEvod)
                            unpack8_evod(w4[u], a[8 * v + 2 * u], a[8 * v + 2 * u + 1]);
                        else
                            unpack8_natural(w4[u], a[8 * v + 2 * u], a[8 * v + 2 * u + 1]);
                    }
                }
                // the TMEM A stage t is free once the MMAs of step j - kT have
                // completed; with as many shared-memory stages as TMEM stages the
                // producer already waited for exactly that before this stage
                // landed
                if (kS != kT && j >= kT &&
                    !warp_wait(&empty[(j - kT) % kS], ((j - kT) / kS) & 1, abort_flag, wait_ns,
                               kDevErrTimeoutConsumer))
                    break;
                tcgen05_fence_after();
                tmem_st_32x32b_x32(tmem_base + lane_base + C::COL_A + 32 * t, a);
                if (A_INT4) {
                    // widen the packed activation codes of this stage (even/odd
                    // K order, like the weights) into the swizzled int8 B tile: 192 rows x 8 chunks of 16 codes, 12
                    // chunks per thread of this K-step parity (the B tile's last
                    // readers, the MMAs of 4 stages ago, completed before the
                    // producer refilled the stage)
                    const uint8_t* ap = sActP + s * C::ACTP;
                    uint8_t* ab = sAct + s * C::ACT;
                    const int tid = q * 32 + lane;
    #pragma unroll 4
                    for (int i = 0; i < kBN * 8 / 128; ++i) {
                        const int c = tid + 128 * i;
                        const int rr = c >> 3, k = c & 7;
                        const uint2 pk = *reinterpret_cast<const uint2*>(ap + rr * 64 + 8 * k);
                        uint4 o;
                        unpack8_evod(pk.x, o.x, o.y);
                        unpack8_evod(pk.y, o.z, o.w);
                        sts128(ab + rr * 128 + ((k ^ (rr & 7)) << 4), o);
                    }
                    fence_proxy_async_smem();   // generic-proxy writes -> tensor-core reads
                }
                tmem_st_wait();
                tcgen05_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&a_full[t]);
            }
        }
    } else if (warp < 18) {
        // ------------------------------------------------ epilogue (warps 10-17)
        const int e = warp - 10;                // 0..7
        const int q = warp & 3;                 // TMEM lane quarter
        const int half = e >> 2;                // tokens [BN/2 half, BN/2 (half + 1))
        const int r = q * 32 + lane;            // weight row in the tile = output column
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        const bool leader = (e == 0 && lane == 0);
        for (int i = 0; i < my_tiles; ++i) {
            const TileAt ta = tile_at(blockIdx.x + i * gridDim.x);
            const int m0 = ta.m0, n0 = ta.n0;
            const int N = grp.N[ta.g];
            const float* __restrict__ row_scale = grp.row_scale[ta.g];
            const __nv_bfloat16* __restrict__ bias = grp.bias[ta.g];
            void* __restrict__ out = grp.out[ta.g];
            const int n = n0 + r;
            const int buf = i & 1;
            const uint32_t fph = (i >> 1) & 1;
            // the tile's token scales into shared memory (0 beyond M), read
            // while the MMAs run: the accumulator is then drained without global
            // loads (the previous tile's readers passed the copy-out barrier)
            if (!OUT_I32)
                for (int t = e * 32 + lane; t < kBN; t += 256)
                    sTok[t] = (m0 + t < M) ? __ldcg(tok_scale + m0 + t) : 0.0f;
            // one thread waits for the accumulator; the named barrier hands the
            // decision to all 8 warps at once (and orders the previous tile's
            // copy-out before this tile's staging writes, the token scales
            // before their reads)
            if (leader) {
                const bool ok = mbar_wait_bounded(&acc_full[buf], fph, abort_flag,
                                                  wait_ns, kDevErrTimeoutEpilogue);
                *epi_go = ok ? 1u : 0u;
            }
            named_barrier_sync(1, 256);
            if (*epi_go == 0u) break;
            tcgen05_fence_after();
            const bool row_ok = n < N;
            // (16 acc) * s_tok * (s_row / 16) equals acc * s_tok * s_row in fp32:
            // scaling by a power of two commutes with the rounding (256 for A_INT4)
            constexpr float kUnscale = A_INT4 ? 1.0f / 256.0f : (W8 ? 1.0f : 0.0625f);
            constexpr int kShift = A_INT4 ? 8 : (W8 ? 0 : 4);
            const float sr16 = (row_ok && !OUT_I32) ? ld_scale<S16>(row_scale, n) * kUnscale : 0.0f;
            const float b = (row_ok && !OUT_I32 && bias != nullptr) ? __bfloat162float(__ldcg(bias + n)) : 0.0f;
            bool released = false;
            // one chunk of 32 tokens from registers: int32 sums, or scaled to
            // bf16 into the staging tile (row = token, 256 bytes; column = this
            // thread's row), two tokens at a time on packed fp32 pairs: (acc
            // s_tok) s_row + b, each element rounded as the scalar multiply and
            // fma would (rows beyond M are written, never copied out)
            auto emit = [&](int c0, const uint32_t (&acc)[32]) {
                const int mb = m0 + c0;
                if (OUT_I32) {
                    if (!row_ok) return;
                    const int mcount = min(32, M - mb);
                    int32_t* o = static_cast<int32_t*>(out) + static_cast<size_t>(mb) * N + n;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (j < mcount) o[static_cast<size_t>(j) * N] = static_cast<int32_t>(acc[j]) >> kShift;
                } else {
                    const float2* st2 = reinterpret_cast<const float2*>(sTok + c0);
                    const uint32_t dst = smem_u32(sOut + c0 * (kTmBM * 2) + r * 2);
                    const uint64_t sr2 = f2_pack(sr16, sr16), b2 = f2_pack(b, b);
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        const uint64_t a2 = f2_pack(static_cast<float>(static_cast<int32_t>(acc[j])),
                                                    static_cast<float>(static_cast<int32_t>(acc[j + 1])));
                        const float2 tj = st2[j / 2];
                        const uint32_t h2 = f2_to_bf16x2(f2_fma(f2_mul(a2, f2_pack(tj.x, tj.y)), sr2, b2));
                        asm volatile(
                            "{\n\t.reg .b16 l, h;\n\t"
                            "mov.b32 {l, h}, %2;\n\t"
                            "st.shared.b16 [%0], l;\n\t"
                            "st.shared.b16 [%1], h;\n\t}" ::"r"(dst + j * (kTmBM * 2)),
                            "r"(dst + (j + 1) * (kTmBM * 2)), "r"(h2)
                            : "memory");
                    }
                }
            };
            // the buffer goes back to the MMAs after this warp's last read
            const int cend = (half + 1) * (kBN / 2);
#pragma unroll 1
            for (int c0 = half * (kBN / 2); c0 < cend; c0 += 32) {
                if (m0 + c0 >= M) break;   // warp-uniform
                uint32_t acc[32];
                tmem_ld_32x32b_x32(tmem_base + lane_base + kTmColD + buf * kBN + c0, acc);
                tmem_ld_wait();
                if (c0 + 32 >= cend || m0 + c0 + 32 >= M) {   // this warp's last read (warp-uniform)
                    tcgen05_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acc_empty[buf]);
                    released = true;
                }
                emit(c0, acc);
            }
            if (!released) {   // no chunk of this warp's half lies below M
                tcgen05_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[buf]);
            }
            if (!OUT_I32) {
                // the staging tile is complete: the 8 warps copy it out, one
                // 16-byte piece of a token row per thread and step (coalesced
                // row segments of y; the TMA engine stays free for the loads)
                named_barrier_sync(1, 256);
                const int et = e * 32 + lane;
                __nv_bfloat16* yb = static_cast<__nv_bfloat16*>(out);
#pragma unroll 4
                for (int c = et; c < kBN * (kTmBM / 8); c += 256) {
                    const int tok = c >> 4, piece = c & 15;
                    if (m0 + tok < M && n0 + piece * 8 < N)
                        *reinterpret_cast<uint4*>(yb + static_cast<size_t>(m0 + tok) * N + n0 + piece * 8) =
                            lds128(sOut + tok * (kTmBM * 2) + piece * 16);
                }
            }
        }
    }

    // ---- teardown: every MMA has landed (warp 1 waited on final_bar)
    tcgen05_fence_before();
    __syncthreads();
    if (warp == 1) {
        tcgen05_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace tint4
