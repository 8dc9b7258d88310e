// gemm_tmem_gw.cuh -- persistent W4A8 GEMM with group-wise weight scales.
//
//   p_j[m, n] = sum_{k in group j} qa[m, k] * (qw[n, k] - z[n, j])   (int32, exact)
//   y[m, n]   = bf16( s_tok[m] * sum_j s[n, j] * p_j[m, n] (+ bias[n]) )
//
// "ComfyUI-INT-Crush", "Weight Format": INT4 weight scales [out, num_groups];
// "Inference > INT4 > CUDA backend": INT4 weights widened to INT8 for an INT8
// GEMM with fused dequant; stable-diffusion.cpp "feat: packed int4 convrot
// model loading and dispatch", "Summary": the asymmetric W4A8 format.
//
// A weight group is one 128-wide K step, so the tensor core sums each group
// on its own (int32, in TMEM) and CUDA cores fold the group sums into an fp32
// running sum with the group's scale.  Same skeleton as gemm_tmem.cuh
// (producer warp, one MMA-issuing thread, 8 unpack warps widening the packed
// weights into TMEM A stages, the activation codes as the MMA's B operand in
// shared memory), with these differences:
//  * tiles of 128 weight rows x 128 tokens; TMEM holds three int32
//    group-sum buffers (K step j uses buffer j % 3, so the MMAs run up to two
//    steps ahead of the fold) and the 4 A stages: 3 x 128 + 4 x 32 = 512
//    columns; the fp32 running sums live in the fold warps' registers (16
//    warps, 32 of a row's 128 tokens each);
//  * each step's first MMA overwrites its group-sum buffer; the fold turns a
//    finished sum p into fp32 without the conversion unit: p + 0x4B400000
//    (an integer add) is the bit pattern of the float 1.5 * 2^23 + p when
//    |p| < 2^22, and subtracting 1.5 * 2^23 leaves p exactly; then one FMA
//    per value, r = fma(s_j / 16, p, r), r starting at +0.  (Refilling the
//    buffers with that
//    start value from the fold warps, so that the MMAs add onto it, took
//    TMEM store bandwidth and ran about 6 % slower);
//  * warps 10-25 fold: they wait for the MMAs of a step (the stage-empty
//    commit), fold the step's group sums into their running sums and release
//    the buffer to the MMA issuer, which waits for it (and for the step's A
//    stage) before the step's MMAs.  After a tile's last step they
//    scale by the token scales, add the bias, round to bf16 into a staging
//    tile and one thread stores it with a TMA tensor store (rows and columns
//    outside y are clipped by the TMA unit);
//  * asymmetric weights (ASYM): the nibbles are plain 4-bit numbers q with a
//    zero point z per row and group, and the unpack writes the int8 value
//    8 (q - z) in [-120, 120]: 8 q sits in bits 3-6 of its byte, adding
//    128 - 8 z to every byte never carries across bytes (8 <= 8 q + 128 - 8 z
//    <= 248), and flipping bit 7 then leaves 8 (q - z) in two's complement.
//    The fold scale is s_j / 8 (s_j / 16 for the symmetric x16 form).
//
// Ranges: |p| <= 128 * 127 * 7 * 16 (symmetric) or 128 * 127 * 15 * 8
// (asymmetric), both below 2^22, so the conversion above is exact.
#pragma once

#include "gemm_tmem.cuh"
#include "pack_groupwise.cuh"

namespace tint4 {

constexpr int kGwBM = 128;                    // weight rows per tile (UMMA M)
constexpr int kGwBN = 128;                    // tokens per tile (UMMA N)
constexpr int kGwBK = kWeightGroup;           // K per step: one weight group
constexpr int kGwStages = 4;                  // shared-memory stages = TMEM A stages
constexpr int kGwFoldWarps = 16;
constexpr int kGwThreads = (10 + kGwFoldWarps) * 32;   // 26 warps
constexpr int kGwActBytes = kGwBN * kGwBK;    // 16 KB
constexpr int kGwWBytes = kGwBM * kGwBK / 2;  // 8 KB packed weights
constexpr int kGwOutBytes = kGwBN * kGwBM * 2;   // 32 KB bf16 staging tile
constexpr int kGwSmemBytes = kGwStages * (kGwActBytes + kGwWBytes) + kGwOutBytes + 256 + 1024;
static_assert(kGwSmemBytes <= 227 * 1024, "shared memory budget");
constexpr int kGwPBufs = 3;                   // group-sum buffers
constexpr uint32_t kGwColP = 0;               // group sums, buffer b at 128 b
constexpr uint32_t kGwColA = kGwPBufs * kGwBN;   // A stage s at kGwColA + 32 s
static_assert(kGwColA + 32 * kGwStages <= 512, "TMEM budget");
constexpr uint32_t kGwStart = 0x4B400000u;    // 1.5 * 2^23 as fp32 bits (the conversion)

// 8 unsigned nibbles q (K order, low nibble first) with zero point z ->
// 8 int8 values 8 (q - z), even/odd K order; zc = (128 - 8 z) * 0x01010101.
__device__ __forceinline__ void unpack8_asym_evod(uint32_t w, uint32_t zc, uint32_t& lo,
                                                  uint32_t& hi) {
    lo = (((w << 3) & 0x78787878u) + zc) ^ 0x80808080u;
    hi = (((w >> 1) & 0x78787878u) + zc) ^ 0x80808080u;
}

// ASYM: unsigned nibbles with zero points (wzero [N, K/128]); else signed.
// EVOD: the int8 activation codes are stored in the even/odd K order
// (0, 2, 4, 6, 1, 3, 5, 7 in every block of 8), the order the unpack
// produces without byte permutes.
// S16: the group scales are IEEE fp16 ("ComfyUI-INT-Crush", "Weight
// Format": the stored format), widened exactly where they are read.
template <bool ASYM, bool EVOD, bool S16 = false>
__global__ void __launch_bounds__(kGwThreads, 1)
w4a8_gw_tmem_gemm_kernel(const __grid_constant__ CUtensorMap tmap_act,
                         const __grid_constant__ CUtensorMap tmap_w,
                         const __grid_constant__ CUtensorMap tmap_y,
                         const float* __restrict__ tok_scale, const void* __restrict__ wscale,
                         const uint8_t* __restrict__ wzero,
                         const __nv_bfloat16* __restrict__ bias, int M, int N, int K,
                         uint64_t wait_ns) {
    constexpr int kS = kGwStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sAct = smem;
    uint8_t* sW = smem + kS * kGwActBytes;
    uint8_t* sOut = sW + kS * kGwWBytes;
    uint64_t* act_full = reinterpret_cast<uint64_t*>(sOut + kGwOutBytes);
    uint64_t* empty = act_full + kS;        // [kS] MMAs of the stage done (commit)
    uint64_t* a_full = empty + kS;          // [kS] TMEM A stage written (4 warp arrivals)
    uint64_t* p_free = a_full + kS;         // [3] group-sum buffer folded (16 warp arrivals)
    uint64_t* final_bar = p_free + kGwPBufs;   // all MMAs done (teardown)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int m_tiles = (M + kGwBN - 1) / kGwBN;
    const int n_tiles = (N + kGwBM - 1) / kGwBM;
    const int n_work = m_tiles * n_tiles;
    const int KT = K / kGwBK;
    const int ng = KT;   // weight groups per row
    const int my_tiles = (blockIdx.x < n_work) ? (n_work - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kS; ++s) {
            mbar_init(&act_full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&a_full[s], 4);
        }
        for (int b = 0; b < kGwPBufs; ++b) mbar_init(&p_free[b], kGwFoldWarps);
        mbar_init(final_bar, 1);
        *abort_flag = 0u;
        fence_mbarrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmap_act);
        prefetch_tensormap(&tmap_w);
        prefetch_tensormap(&tmap_y);
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
                const int tile = blockIdx.x + i * gridDim.x;
                const int m0 = (tile % m_tiles) * kGwBN, n0 = (tile / m_tiles) * kGwBM;
                for (int kt = 0; kt < KT; ++kt, ++c) {
                    const int s = c % kS;
                    const uint32_t ph = (c / kS) & 1;
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, wait_ns,
                                           kDevErrTimeoutProducer))
                        break;
                    mbar_arrive_expect_tx(&act_full[s], kGwActBytes + kGwWBytes);
                    tma_load_2d(&tmap_act, &act_full[s], sAct + s * kGwActBytes, kt * kGwBK, m0);
                    tma_load_2d(&tmap_w, &act_full[s], sW + s * kGwWBytes, kt * (kGwBK / 2), n0);
                    ++issued;
                }
            }
            if (*abort_flag) {
                uint32_t never = 0u;
                const int first = issued > kS ? issued - kS : 0;
                for (int j = first; j < issued; ++j)
                    (void)mbar_wait_bounded(&act_full[j % kS], (j / kS) & 1, &never, wait_ns, 0u);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_i8(kGwBM, kGwBN);
            const uint64_t bdesc0 = umma_desc_sw128(smem_u32(sAct));
            int j = 0;
            bool ok = true;
            for (int i = 0; i < my_tiles && ok; ++i) {
                for (int kt = 0; kt < KT; ++kt, ++j) {
                    const int s = j % kS;
                    // the step's A stage (the unpack warps arrive only after the
                    // stage landed), then its group-sum buffer, folded
                    if (!mbar_wait_bounded(&a_full[s], (j / kS) & 1, abort_flag, wait_ns,
                                           kDevErrTimeoutConsumer)) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait_bounded(&p_free[j % kGwPBufs], (j / kGwPBufs) & 1, abort_flag,
                                           wait_ns, kDevErrTimeoutConsumer)) {
                        ok = false;
                        break;
                    }
                    tcgen05_fence_after();
                    const uint32_t d_tmem = tmem_base + kGwColP + (j % kGwPBufs) * kGwBN;
                    const uint32_t a_tmem = tmem_base + kGwColA + 32 * s;
                    const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(s * (kGwActBytes >> 4));
                    umma_i8_ts_step(d_tmem, a_tmem, bdesc, idesc, 0u);   // a fresh group sum
                    umma_commit(&empty[s]);
                }
            }
            umma_commit(final_bar);
            uint32_t never = 0u;
            (void)mbar_wait_bounded(final_bar, 0, &never, wait_ns, 0u);
        }
        __syncwarp();
    } else if (warp < 10) {
        // ------------------------------------------------ weight unpack -> TMEM (warps 2-9)
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const int total = my_tiles * KT;
        const int sw = (r >> 1) & 3;   // 64-byte swizzle of the weight tile
        for (int j = (warp < 6 ? 0 : 1); j < total; j += 2) {
            const int s = j % kS;
            uint32_t zc = 0u;
            if constexpr (ASYM) {
                const int i = j / KT, kt = j % KT;
                const int n = ((blockIdx.x + i * gridDim.x) / m_tiles) * kGwBM + r;
                const uint32_t z = n < N ? __ldca(wzero + static_cast<size_t>(n) * ng + kt) : 0u;
                zc = (128u - 8u * z) * 0x01010101u;
            }
            if (!warp_wait(&act_full[s], (j / kS) & 1, abort_flag, wait_ns, kDevErrTimeoutConsumer))
                break;
            const uint8_t* row = sW + s * kGwWBytes + r * 64;
            // 128 K values of row r into the TMEM A stage s (the MMAs of step
            // j - 4, its last readers, completed before the producer refilled
            // shared-memory stage s)
            uint32_t a[32];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const uint4 p = lds128(row + 16 * (v ^ sw));
                const uint32_t w4[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint32_t lo, hi;
                    if constexpr (ASYM) unpack8_asym_evod(w4[u], zc, lo, hi);
                    else unpack8_evod(w4[u], lo, hi);
                    if constexpr (!EVOD) {   // natural K order: interleave the bytes back
                        const uint32_t L = lo, H = hi;
                        lo = __byte_perm(L, H, 0x5140);
                        hi = __byte_perm(L, H, 0x7362);
                    }
                    a[8 * v + 2 * u] = lo;
                    a[8 * v + 2 * u + 1] = hi;
                }
            }
            tcgen05_fence_after();
            tmem_st_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + kGwColA + 32 * s,
                               a);
            tmem_st_wait();
            tcgen05_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[s]);
        }
    } else if (warp < 10 + kGwFoldWarps) {
        // ------------------------------------------------ fold + epilogue (warps 10-25)
        const int e = warp - 10;                // 0..15
        const int q = warp & 3;                 // TMEM lane quarter
        const int part = e >> 2;                // tokens [32 part, 32 part + 32) of the tile
        const int r = q * 32 + lane;            // weight row in the tile = output column
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        const bool leader = (e == 0 && lane == 0);
        constexpr uint32_t kFoldThreads = kGwFoldWarps * 32;
        constexpr float kUnscale = ASYM ? 0.125f : 0.0625f;
        constexpr float kStartF = 12582912.0f;   // 1.5 * 2^23
        // every group-sum buffer is free at the start
        if (lane == 0)
            for (int b = 0; b < kGwPBufs; ++b) mbar_arrive(&p_free[b]);
        int j = 0;
        // after a failed wait a fold warp goes on through every step without
        // waiting (its values are then meaningless and the call reports the
        // error), so all fold warps meet at the same named barriers
        bool ok = true;
        bool stored = false;   // a TMA store of the staging tile is in flight (leader)
        float acc[32];         // running sums: row r, tokens 32 part + x
        for (int i = 0; i < my_tiles; ++i) {
#pragma unroll
            for (int x = 0; x < 32; ++x) acc[x] = 0.0f;
            const int tile = blockIdx.x + i * gridDim.x;
            const int m0 = (tile % m_tiles) * kGwBN, n0 = (tile / m_tiles) * kGwBM;
            const int n = n0 + r;
            const bool row_ok = n < N;
            const size_t srow = static_cast<size_t>(row_ok ? n : 0) * ng;
            float sg_next = row_ok ? ld_scale<S16>(wscale, srow) * kUnscale : 0.0f;
            for (int kt = 0; kt < KT; ++kt, ++j) {
                const float sg = sg_next;
                if (kt + 1 < KT) sg_next = row_ok ? ld_scale<S16>(wscale, srow + kt + 1) * kUnscale : 0.0f;
                if (ok && !warp_wait(&empty[j % kS], (j / kS) & 1, abort_flag, wait_ns,
                                     kDevErrTimeoutEpilogue))
                    ok = false;
                tcgen05_fence_after();
                const uint32_t pcol =
                    tmem_base + lane_base + kGwColP + (j % kGwPBufs) * kGwBN + part * 32;
#pragma unroll
                for (int c = 0; c < 2; ++c) {   // 16 columns at a time (registers)
                    uint32_t p[16];
                    tmem_ld_32x32b_x16(pcol + c * 16, p);
                    tmem_ld_wait();
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        // = p, exactly; then acc += s_j p, one rounding
                        const float d = __fsub_rn(__uint_as_float(p[x] + kGwStart), kStartF);
                        acc[16 * c + x] = __fmaf_rn(sg, d, acc[16 * c + x]);
                    }
                }
                // hand the buffer back: the MMAs of step j + 3 may overwrite it
                tmem_st_wait();
                tcgen05_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_free[j % kGwPBufs]);
            }
            // ---- epilogue: y = r * s_tok + bias -> bf16 staging tile (row =
            // token, 256 bytes; column = this thread's row) -> one TMA store
            if (leader && stored) bulk_wait_group_read0();   // previous store read the tile
            named_barrier_sync(1, kFoldThreads);
            const float b = (row_ok && bias != nullptr) ? __bfloat162float(__ldcg(bias + n)) : 0.0f;
            const int t0 = part * 32;
            const int mb = m0 + t0;
            uint8_t* dst = sOut + t0 * (kGwBM * 2) + r * 2;
#pragma unroll
            for (int x = 0; x < 32; x += 4) {
                float4 st4 = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if (mb + x + 3 < M) {
                    st4 = __ldcg(reinterpret_cast<const float4*>(tok_scale + mb + x));
                } else {
                    if (mb + x < M) st4.x = __ldcg(tok_scale + mb + x);
                    if (mb + x + 1 < M) st4.y = __ldcg(tok_scale + mb + x + 1);
                    if (mb + x + 2 < M) st4.z = __ldcg(tok_scale + mb + x + 2);
                }
                const float sv[4] = {st4.x, st4.y, st4.z, st4.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const __nv_bfloat16 h = __float2bfloat16_rn(__fmaf_rn(acc[x + u], sv[u], b));
                    asm volatile("st.shared.b16 [%0], %1;" ::"r"(smem_u32(dst + (x + u) * (kGwBM * 2))),
                                 "h"(*reinterpret_cast<const unsigned short*>(&h))
                                 : "memory");
                }
            }
            fence_proxy_async_smem();   // staging writes -> the TMA unit
            named_barrier_sync(1, kFoldThreads);
            if (leader) {
                tma_store_2d(&tmap_y, sOut, n0, m0);
                bulk_commit_group();
                stored = true;
            }
        }
        if (leader && stored) bulk_wait_group0();
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
