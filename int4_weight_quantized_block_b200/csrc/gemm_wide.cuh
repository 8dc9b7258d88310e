// gemm_wide.cuh -- the W4A8 GEMM of int8 activation codes x packed int4
// weights, with the weight stream decoupled from the activation stream.
//
//   acc[m, n] = sum_k qa[m, k] * qw[n, k]            (int32, exact)
//   y[m, n]   = bf16( acc * s_tok[m] * s_row[n] (+ bias[n]) )
//
// "ComfyUI-INT-Crush", "Inference > INT4 > CUDA backend": INT4 weights are
// unpacked to INT8 and run through an INT8 GEMM with fused dequant;
// stable-diffusion.cpp "feat: packed int4 convrot model loading and
// dispatch", "Summary": the packed nibbles stay packed in memory.
//
// The product on the tensor core is that of gemm_tmem.cuh with 256-token
// tiles: weights as the MMA's A operand from TMEM (128 rows = the TMEM
// lanes, widened x16 by the unpack warps), activation codes as its B operand
// from shared memory (256 tokens x 128 K, 128-byte swizzle), one int32
// accumulator of 256 columns.  What differs is the pipeline.  There a K
// step's activation tile and packed weight tile travel in one shared-memory
// stage, and the stage goes back to the producer only when the step's MMAs
// have completed, so every activation stage waits in its ring for the unpack
// of its weights: the ring's round trip holds TMA latency, the unpack and
// the MMAs.  Here the two streams have rings of their own:
//   activations  4 shared-memory stages of 32 KB, refilled when the MMAs of
//                the step 4 back have completed;
//   weights      4 shared-memory stages of 8 KB, refilled as soon as the
//                unpack warps have read them, and
//   widened A    8 TMEM stages of 32 columns (256 + 32 s; the accumulator
//                takes columns 0-255), rewritten when the MMAs of the step 8
//                back have completed,
// so the unpack runs up to 8 steps ahead of the MMAs and an activation
// stage's round trip is TMA latency and MMAs only, as for int8 weights.
//
// Warp roles (19 warps, one persistent CTA per SM, static tile list):
//   warp 0      activation producer (TMA)
//   warp 1      TMEM owner; one thread issues the MMAs (M 128, N 256, K 32)
//               and commits each step to the step's A-stage barrier
//   warps 2-9   weight unpack: warps 2-5 the even K steps, 6-9 the odd ones
//   warps 10-17 epilogue (as in gemm_tmem.cuh, one accumulator: two 32-token
//               chunks per TMEM read, handed back after the warp's last read)
//   warp 18     weight producer (TMA)
// One commit per step (a_empty[j % 8]) serves both rings: the activation
// producer waits for the one of step j - 4, the unpack for the one of step
// j - 8; neither barrier can complete again before the waiter moves on (its
// next completion needs the waiter's own stage), so the parities are exact.
#pragma once

#include "gemm_tmem.cuh"

namespace tint4 {

constexpr int kWdBN = 256;                 // tokens per tile (UMMA N)
constexpr int kWdActStages = 4;            // activation stages in shared memory
constexpr int kWdWStages = 4;              // packed-weight stages in shared memory
constexpr int kWdAStages = 8;              // widened-weight stages in TMEM
constexpr int kWdThreads = 608;            // 19 warps
constexpr int kWdAct = kWdBN * kTmBK;      // 32 KB of int8 codes per stage
constexpr int kWdOut = kWdBN * kTmBM * 2;  // 64 KB bf16 staging tile
constexpr int kWdBarBytes = 512;
constexpr int kWdSmem = kWdActStages * kWdAct + kWdWStages * kTmWBytes + kWdOut + kWdBarBytes +
                        kWdBN * 4 + 1024;
constexpr uint32_t kWdColA = kWdBN;        // A stage s at kWdColA + 32 s
static_assert(kWdColA + 32 * kWdAStages <= 512, "TMEM budget");
// each unpack chain takes every other K step, so a weight or A stage must
// belong to one chain (even stage counts): a chain then waits on its stages'
// phases in order and a parity wait cannot pass on a phase it skipped
static_assert(kWdWStages % 2 == 0 && kWdAStages % 2 == 0, "stages of one chain");
static_assert(kWdActStages <= kWdAStages, "the A-stage barriers also free the activation stages");
static_assert(kWdSmem <= 227 * 1024, "shared memory budget");
static_assert(kWdAct % 1024 == 0 && kTmWBytes % 1024 == 0, "swizzled stage alignment");

template <bool OUT_I32, bool EVOD>
__global__ void __launch_bounds__(kWdThreads, 1)
w4a8_wide_gemm_kernel(const __grid_constant__ CUtensorMap tmap_act,
                      const __grid_constant__ TmGroups grp,
                      const float* __restrict__ tok_scale, int M, int K, uint64_t wait_ns) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sAct = smem;
    uint8_t* sW = sAct + kWdActStages * kWdAct;
    uint8_t* sOut = sW + kWdWStages * kTmWBytes;
    uint64_t* act_full = reinterpret_cast<uint64_t*>(sOut + kWdOut);   // [4] landed (TMA)
    uint64_t* w_full = act_full + kWdActStages;    // [4] landed (TMA)
    uint64_t* w_empty = w_full + kWdWStages;       // [4] read by the 4 warps of a chain
    uint64_t* a_full = w_empty + kWdWStages;       // [8] TMEM A stage written (4 warps)
    uint64_t* a_empty = a_full + kWdAStages;       // [8] the step's MMAs completed (commit)
    uint64_t* acc_full = a_empty + kWdAStages;     // accumulator ready (commit)
    uint64_t* acc_empty = acc_full + 1;            // accumulator read (8 warps)
    uint64_t* final_bar = acc_empty + 1;           // all MMAs done (teardown)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;
    volatile uint32_t* epi_go = tmem_slot + 2;
    static_assert((2 * kWdActStages + 2 * kWdWStages + 2 * kWdAStages + 3) * 8 + 12 <= kWdBarBytes,
                  "barrier area");
    float* sTok = reinterpret_cast<float*>(sOut + kWdOut + kWdBarBytes);   // the tile's token scales

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int m_tiles = (M + kWdBN - 1) / kWdBN;
    const int n_work = grp.tile_end[grp.count - 1];
    const int KT = (K + kTmBK - 1) / kTmBK;
    const int my_tiles = (blockIdx.x < n_work) ? (n_work - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int total = my_tiles * KT;               // K steps this CTA runs
    struct TileAt {
        int g, m0, n0;
    };
    auto tile_at = [&](int tile) -> TileAt {
        int g = 0;
#pragma unroll
        for (int h = 0; h < kTmMaxGroups - 1; ++h)
            if (h + 1 < grp.count && tile >= grp.tile_end[h]) g = h + 1;
        const int t = tile - (g > 0 ? grp.tile_end[g - 1] : 0);
        return TileAt{g, (t % m_tiles) * kWdBN, (t / m_tiles) * kTmBM};
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kWdActStages; ++s) mbar_init(&act_full[s], 1);
        for (int s = 0; s < kWdWStages; ++s) {
            mbar_init(&w_full[s], 1);
            mbar_init(&w_empty[s], 4);
        }
        for (int s = 0; s < kWdAStages; ++s) {
            mbar_init(&a_full[s], 4);
            mbar_init(&a_empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 8);
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
        // ------------------------------------------------ activation producer
        if (lane == 0) {
            int j = 0, issued = 0;
            for (int i = 0; i < my_tiles && !*abort_flag; ++i) {
                const int m0 = tile_at(blockIdx.x + i * gridDim.x).m0;
                bool ok = true;
                for (int kt = 0; kt < KT; ++kt, ++j) {
                    // stage j % 4 is free once the MMAs of step j - 4 have completed
                    if (j >= kWdActStages &&
                        !mbar_wait_bounded(&a_empty[(j - kWdActStages) % kWdAStages],
                                           ((j - kWdActStages) / kWdAStages) & 1, abort_flag,
                                           wait_ns, kDevErrTimeoutProducer)) {
                        ok = false;
                        break;
                    }
                    const int s = j % kWdActStages;
                    mbar_arrive_expect_tx(&act_full[s], kWdAct);
                    tma_load_2d(&tmap_act, &act_full[s], sAct + s * kWdAct, kt * kTmBK, m0);
                    ++issued;
                }
                if (!ok) break;
            }
            if (*abort_flag) {
                // let the copies in flight land before the CTA leaves
                uint32_t never = 0u;
                for (int q = issued > kWdActStages ? issued - kWdActStages : 0; q < issued; ++q)
                    (void)mbar_wait_bounded(&act_full[q % kWdActStages], (q / kWdActStages) & 1,
                                            &never, wait_ns, 0u);
            }
        }
    } else if (warp == 18) {
        // ------------------------------------------------ weight producer
        if (lane == 0) {
            int j = 0, issued = 0;
            for (int i = 0; i < my_tiles && !*abort_flag; ++i) {
                const TileAt ta = tile_at(blockIdx.x + i * gridDim.x);
                const CUtensorMap* tmap_w = &grp.w[ta.g];
                bool ok = true;
                for (int kt = 0; kt < KT; ++kt, ++j) {
                    const int s = j % kWdWStages;
                    // stage s is free once the unpack of step j - 4 has read it
                    if (!mbar_wait_bounded(&w_empty[s], ((j / kWdWStages) & 1) ^ 1, abort_flag,
                                           wait_ns, kDevErrTimeoutProducer)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&w_full[s], kTmWBytes);
                    tma_load_2d(tmap_w, &w_full[s], sW + s * kTmWBytes, kt * (kTmBK / 2), ta.n0);
                    ++issued;
                }
                if (!ok) break;
            }
            if (*abort_flag) {
                uint32_t never = 0u;
                for (int q = issued > kWdWStages ? issued - kWdWStages : 0; q < issued; ++q)
                    (void)mbar_wait_bounded(&w_full[q % kWdWStages], (q / kWdWStages) & 1, &never,
                                            wait_ns, 0u);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_i8(kTmBM, kWdBN);
            // stage s of the activation ring starts (s * bytes) / 16 descriptor
            // units above stage 0 (the address field cannot carry)
            const uint64_t bdesc0 = umma_desc_sw128(smem_u32(sAct));
            static_assert(kTmBK == 4 * 32, "four MMAs per K step");
            int j = 0;
            bool ok = true;
            for (int i = 0; i < my_tiles && ok; ++i) {
                if (!mbar_wait_bounded(acc_empty, (i & 1) ^ 1, abort_flag, wait_ns,
                                       kDevErrTimeoutConsumer)) {
                    ok = false;
                    break;
                }
                tcgen05_fence_after();
                for (int kt = 0; kt < KT; ++kt, ++j) {
                    const int as = j % kWdAStages, s = j % kWdActStages;
                    // the widened weights (usually ready well ahead), then the codes
                    if (!mbar_wait_bounded(&a_full[as], (j / kWdAStages) & 1, abort_flag, wait_ns,
                                           kDevErrTimeoutConsumer) ||
                        !mbar_wait_bounded(&act_full[s], (j / kWdActStages) & 1, abort_flag,
                                           wait_ns, kDevErrTimeoutConsumer)) {
                        ok = false;
                        break;
                    }
                    tcgen05_fence_after();
                    umma_i8_ts_step(tmem_base, tmem_base + kWdColA + 32 * as,
                                    bdesc0 + static_cast<uint64_t>(s * (kWdAct >> 4)), idesc, kt);
                    umma_commit(&a_empty[as]);
                }
                if (ok) umma_commit(acc_full);
            }
            // everything issued lands before TMEM is released
            umma_commit(final_bar);
            uint32_t never = 0u;
            (void)mbar_wait_bounded(final_bar, 0, &never, wait_ns, 0u);
        }
        __syncwarp();
    } else if (warp < 10) {
        // ------------------------------------------------ weight unpack -> TMEM (warps 2-9)
        const int q = warp & 3;                 // TMEM lane quarter
        const int r = q * 32 + lane;            // weight row within the tile
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        // 64-byte swizzle of the TMA tile: chunk v of row r sits at chunk
        // v ^ ((r >> 1) & 3); 8 consecutive rows then hit 8 distinct bank groups
        const int sw = (r >> 1) & 3;
        for (int j = (warp < 6 ? 0 : 1); j < total; j += 2) {
            const int ws = j % kWdWStages, as = j % kWdAStages;
            if (!warp_wait(&w_full[ws], (j / kWdWStages) & 1, abort_flag, wait_ns,
                           kDevErrTimeoutConsumer))
                break;
            const uint8_t* row = sW + ws * kTmWBytes + r * 64;
            uint32_t a[32];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const uint4 p = lds128(row + 16 * (v ^ sw));
                const uint32_t w4[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if constexpr (EVOD)
                        unpack8_evod(w4[u], a[8 * v + 2 * u], a[8 * v + 2 * u + 1]);
                    else
                        unpack8_natural(w4[u], a[8 * v + 2 * u], a[8 * v + 2 * u + 1]);
                }
            }
            // the packed stage is in registers (the values above depend on every
            // load): the weight producer may refill it
            __syncwarp();
            if (lane == 0) mbar_arrive(&w_empty[ws]);
            // TMEM stage as is free once the MMAs of step j - 8 have completed
            if (j >= kWdAStages &&
                !warp_wait(&a_empty[as], ((j - kWdAStages) / kWdAStages) & 1, abort_flag, wait_ns,
                           kDevErrTimeoutConsumer))
                break;
            tcgen05_fence_after();
            tmem_st_32x32b_x32(tmem_base + lane_base + kWdColA + 32 * as, a);
            tmem_st_wait();
            tcgen05_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[as]);
        }
    } else if (warp < 18) {
        // ------------------------------------------------ epilogue (warps 10-17)
        const int e = warp - 10;                // 0..7
        const int q = warp & 3;                 // TMEM lane quarter
        const int half = e >> 2;                // tokens [128 half, 128 half + 128)
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
            // the tile's token scales into shared memory (0 beyond M) while its
            // MMAs run (the previous tile's readers passed the copy-out barrier)
            if (!OUT_I32)
                for (int t = e * 32 + lane; t < kWdBN; t += 256)
                    sTok[t] = (m0 + t < M) ? __ldcg(tok_scale + m0 + t) : 0.0f;
            // one thread waits for the accumulator; the named barrier hands the
            // decision to all 8 warps (and orders the previous tile's copy-out
            // before this tile's staging writes, the token scales before
            // their reads)
            if (leader) {
                const bool ok = mbar_wait_bounded(acc_full, i & 1, abort_flag, wait_ns,
                                                  kDevErrTimeoutEpilogue);
                *epi_go = ok ? 1u : 0u;
            }
            named_barrier_sync(1, 256);
            if (*epi_go == 0u) break;
            tcgen05_fence_after();
            const bool row_ok = n < N;
            // (16 acc) * s_tok * (s_row / 16) equals acc * s_tok * s_row in fp32
            const float sr16 = (row_ok && !OUT_I32) ? __ldcg(row_scale + n) * 0.0625f : 0.0f;
            const float b = (row_ok && !OUT_I32 && bias != nullptr) ? __bfloat162float(__ldcg(bias + n)) : 0.0f;
            // 32 tokens from registers: int32 sums, or scaled to bf16 into the
            // staging tile (row = token, 256 bytes; column = this thread's row),
            // two tokens at a time on packed fp32 pairs (rows beyond M are
            // written, never copied out)
            auto emit = [&](int c0, const uint32_t (&acc)[32]) {
                const int mb = m0 + c0;
                if (OUT_I32) {
                    if (!row_ok) return;
                    const int mcount = min(32, M - mb);
                    int32_t* o = static_cast<int32_t*>(out) + static_cast<size_t>(mb) * N + n;
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj)
                        if (jj < mcount) o[static_cast<size_t>(jj) * N] = static_cast<int32_t>(acc[jj]) >> 4;
                } else {
                    const float2* st2 = reinterpret_cast<const float2*>(sTok + c0);
                    const uint32_t dst = smem_u32(sOut + c0 * (kTmBM * 2) + r * 2);
                    const uint64_t sr2 = f2_pack(sr16, sr16), b2 = f2_pack(b, b);
#pragma unroll
                    for (int jj = 0; jj < 32; jj += 2) {
                        const uint64_t a2 = f2_pack(static_cast<float>(static_cast<int32_t>(acc[jj])),
                                                    static_cast<float>(static_cast<int32_t>(acc[jj + 1])));
                        const float2 tj = st2[jj / 2];
                        const uint32_t h2 = f2_to_bf16x2(f2_fma(f2_mul(a2, f2_pack(tj.x, tj.y)), sr2, b2));
                        asm volatile(
                            "{\n\t.reg .b16 l, h;\n\t"
                            "mov.b32 {l, h}, %2;\n\t"
                            "st.shared.b16 [%0], l;\n\t"
                            "st.shared.b16 [%1], h;\n\t}" ::"r"(dst + jj * (kTmBM * 2)),
                            "r"(dst + (jj + 1) * (kTmBM * 2)), "r"(h2)
                            : "memory");
                    }
                }
            };
            // two chunks per TMEM read; the accumulator goes back to the MMAs
            // after this warp's last read, before the math on it
            bool released = false;
            const int cend = (half + 1) * (kWdBN / 2);
#pragma unroll 1
            for (int c0 = half * (kWdBN / 2); c0 < cend; c0 += 64) {
                if (m0 + c0 >= M) break;   // warp-uniform
                const bool two = c0 + 32 < cend && m0 + c0 + 32 < M;   // warp-uniform
                uint32_t acc0[32], acc1[32];
                tmem_ld_32x32b_x32(tmem_base + lane_base + c0, acc0);
                if (two) tmem_ld_32x32b_x32(tmem_base + lane_base + c0 + 32, acc1);
                tmem_ld_wait();
                if (c0 + 64 >= cend || m0 + c0 + 64 >= M) {   // warp-uniform
                    tcgen05_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(acc_empty);
                    released = true;
                }
                emit(c0, acc0);
                if (two) emit(c0 + 32, acc1);
            }
            if (!released) {   // no token of this warp's half below M
                tcgen05_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty);
            }
            if (!OUT_I32) {
                // the staging tile is complete: the 8 warps copy it out, one
                // 16-byte piece of a token row per thread and step
                named_barrier_sync(1, 256);
                const int et = e * 32 + lane;
                __nv_bfloat16* yb = static_cast<__nv_bfloat16*>(out);
#pragma unroll 4
                for (int c = et; c < kWdBN * (kTmBM / 8); c += 256) {
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
