// w4a16_gemm.cuh -- W4A16 group-wise asymmetric linear for large M (prefill)
// on the tcgen05 tensor cores, dequantized weights in tensor memory.
//
//   y[m, n] = sum_k x[m, k] * bf16((q[n, k] - z[n, k/G]) * s[n, k/G])     (G = 128)
//
// "TINT4 v1.2 -- torchao INT4 for ComfyUI", "v1.1 新特性 > 5": the layer keeps
// _qdata / _scale / _zp (uint4 codes two per byte, a bf16 scale and a uint4
// zero point per 128-wide K group and row); "ComfyUI-INT-Crush", "Inference >
// INT4 > Triton backend": with rot_size == 0 the INT4 weights are widened to
// 16 bits and multiplied on the 16-bit tensor cores.  Widening means
// dequantizing: each weight becomes the bf16 number nearest to (q - z) * s,
// the value a bf16 dequantize-then-matmul computes, and the products
// accumulate in fp32.
//
// Shape on the tensor core: the weights are the MMA's M side (128 rows = the
// 128 TMEM lanes), the tokens its N side (256 per tile), as in the int8 GEMM
// (gemm_tmem.cuh).  Per 64-wide K step the TMA brings one token tile (256
// tokens x 64 bf16 = 128-byte rows, 128-byte swizzle: the MMA's B operand) and
// one packed weight tile (128 rows x 32 bytes).  Each of 128 dequant threads
// owns one weight row: it reads its 32 packed bytes, forms bf16(128 + q) for
// every nibble by OR-ing it into the mantissa of bf16 128 (exact), subtracts
// 128 + z (exact: small integers) and multiplies by s (one rounding), both on
// bf16 pairs, and writes the 64 K values of the step with one tcgen05.st into
// a TMEM A stage.  K order stays natural (the tokens come straight from
// memory), so a pair of weights is the two nibbles of one byte.
//
// K steps come in pairs inside a group (K % 128 == 0): warps 2-5 take the even
// steps, i.e. the first half of every group, warps 6-9 the odd ones; each
// loads the scale and zero point of its row for the group of its next step
// while it works on the current one.
//
// The pipeline is that of gemm_wide.cuh: the token tiles and the packed
// weights have rings of their own, and the dequantized weights a ring of 8
// TMEM stages, so the dequant (the kernel's critical path) runs up to 8 steps
// ahead of the MMAs and a token stage's round trip is TMA latency and MMAs.
// Warp roles (19 warps, one persistent CTA per SM, static tile list):
//   warp 0      token-tile producer (4 stages of 32 KB, refilled when the
//               MMAs of the step 4 back have completed)
//   warp 1      TMEM owner; one thread issues tcgen05.mma.kind::f16 (A bf16
//               from TMEM, B bf16 from shared memory, fp32 D; M 128, N 256,
//               K 16) and commits each step to its A stage's barrier
//   warps 2-9   dequant into the 8 TMEM A stages (32 columns each)
//   warps 10-17 epilogue: tcgen05.ld of the accumulator two 32-token chunks
//               at a time, handed back to the MMAs after the last read,
//               rounding to bf16 into a [256 tokens][128 columns] staging
//               tile, copied to y in 16-byte row pieces.
//   warp 18     packed-weight producer (4 stages of 4 KB, refilled once read)
// TMEM columns: one accumulator at 0 (256 columns), A stages at 256 + 32 s.
// (256 tokens per tile rather than 192 with two accumulators: the dequant
// work of a step then serves a third more tokens.)
#pragma once

#include "ptx.cuh"

namespace tint4 {

constexpr int kWgBM = 128;       // weight rows per tile (UMMA M, TMEM lanes)
constexpr int kWgBN = 256;       // tokens per tile (UMMA N)
constexpr int kWgBK = 64;        // K values per stage (bf16: 128-byte rows)
constexpr int kWgActStages = 4;  // token-tile stages in shared memory
constexpr int kWgWStages = 4;    // packed-weight stages in shared memory
constexpr int kWgAStages = 8;    // dequantized-weight stages in TMEM
constexpr int kWgThreads = 608;  // 19 warps
constexpr int kWgGroup = 128;    // quantization group along K
constexpr int kWgActBytes = kWgBN * kWgBK * 2;        // 32 KB token tile per stage
constexpr int kWgWBytes = kWgBM * kWgBK / 2;          // 4 KB packed weights per stage
constexpr int kWgOutBytes = kWgBN * kWgBM * 2;        // 64 KB bf16 staging tile
constexpr int kWgBarBytes = 512;
constexpr int kWgSmemBytes =
    kWgActStages * kWgActBytes + kWgWStages * kWgWBytes + kWgOutBytes + kWgBarBytes + 1024;
constexpr uint32_t kWgColD = 0;                       // the accumulator
constexpr uint32_t kWgColA = kWgBN;                   // A stage s at kWgColA + 32 s
static_assert(kWgColA + 32 * kWgAStages <= 512, "TMEM budget");
// each unpack chain takes every other K step, so a weight or A stage must
// belong to one chain (even stage counts): a chain then waits on its stages'
// phases in order and a parity wait cannot pass on a phase it skipped
static_assert(kWgWStages % 2 == 0 && kWgAStages % 2 == 0, "stages of one chain");
static_assert(kWgActStages <= kWgAStages, "the A-stage barriers also free the activation stages");
static_assert(kWgSmemBytes <= 227 * 1024, "shared memory budget");
static_assert(kWgActBytes % 1024 == 0 && kWgWBytes % 1024 == 0, "stage alignment");
static_assert(kWgGroup == 2 * kWgBK, "a group is two K steps");

// Instruction descriptor for kind::f16 with bf16 A and B, fp32 D, both
// operands K-major, shape M x N.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
    return (1u << 4)                                  // D format: f32
           | (1u << 7)                                // A: bf16
           | (1u << 10)                               // B: bf16
           | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);   // M / 16
}

__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t m, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(m), "r"(c));   // (a & m) | c
    return d;
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// 8 packed nibbles (K order, low nibble of each byte first) -> 4 bf16 pairs
// bf16((q - z) * s) in natural K order; zc = bf16x2(128 + z), s2 = bf16x2(s).
__device__ __forceinline__ void dequant8(uint32_t w, uint32_t zc, uint32_t s2, uint32_t (&o)[4]) {
    const uint32_t lo = w & 0x0F0F0F0Fu;          // q[2p]   in byte p
    const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;   // q[2p+1] in byte p
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        // byte 0 <- lo byte p, byte 2 <- hi byte p (bytes 1 and 3 are masked off)
        const uint32_t t = __byte_perm(lo, hi, static_cast<uint32_t>(p | (p << 4) | ((4 + p) << 8) | ((4 + p) << 12)));
        const uint32_t h = lop3_and_or(t, 0x000F000Fu, 0x43004300u);   // bf16(128 + q) x 2, exact
        o[p] = bf16x2_mul(bf16x2_sub(h, zc), s2);
    }
}

__global__ void __launch_bounds__(kWgThreads, 1)
w4a16_tmem_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x,
                       const __grid_constant__ CUtensorMap tmap_q,
                       const __nv_bfloat16* __restrict__ wscale,
                       const uint8_t* __restrict__ wzero, __nv_bfloat16* __restrict__ y, int M,
                       int N, int K, uint64_t wait_ns) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sAct = smem;
    uint8_t* sW = sAct + kWgActStages * kWgActBytes;
    uint8_t* sOut = sW + kWgWStages * kWgWBytes;
    uint64_t* act_full = reinterpret_cast<uint64_t*>(sOut + kWgOutBytes);   // [4] landed (TMA)
    uint64_t* w_full = act_full + kWgActStages;    // [4] landed (TMA)
    uint64_t* w_empty = w_full + kWgWStages;       // [4] read by the 4 warps of a chain
    uint64_t* a_full = w_empty + kWgWStages;       // [8] TMEM A stage written (4 warps)
    uint64_t* a_empty = a_full + kWgAStages;       // [8] the step's MMAs completed (commit)
    uint64_t* acc_full = a_empty + kWgAStages;     // accumulator ready (commit)
    uint64_t* acc_empty = acc_full + 1;            // accumulator read (8 warps)
    uint64_t* final_bar = acc_empty + 1;           // all MMAs done (teardown)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;
    volatile uint32_t* epi_go = tmem_slot + 2;
    static_assert((2 * kWgActStages + 2 * kWgWStages + 2 * kWgAStages + 3) * 8 + 12 <= kWgBarBytes,
                  "barrier area");

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int m_tiles = (M + kWgBN - 1) / kWgBN;
    const int n_tiles = (N + kWgBM - 1) / kWgBM;
    const int n_work = m_tiles * n_tiles;
    const int KT = K / kWgBK;                      // even: K % 128 == 0
    const int ngroups = K / kWgGroup;
    const int my_tiles = (blockIdx.x < n_work) ? (n_work - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int total = my_tiles * KT;               // K steps this CTA runs

    if (threadIdx.x == 0) {
        for (int s = 0; s < kWgActStages; ++s) mbar_init(&act_full[s], 1);
        for (int s = 0; s < kWgWStages; ++s) {
            mbar_init(&w_full[s], 1);
            mbar_init(&w_empty[s], 4);
        }
        for (int s = 0; s < kWgAStages; ++s) {
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
        prefetch_tensormap(&tmap_x);
        prefetch_tensormap(&tmap_q);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tcgen05_fence_before();
    __syncthreads();
    tcgen05_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // x (and the weights) may come from the grid launched just before
    grid_dependency_wait();

    if (warp == 0) {
        // ------------------------------------------------ token-tile producer
        if (lane == 0) {
            int j = 0, issued = 0;
            for (int i = 0; i < my_tiles && !*abort_flag; ++i) {
                const int m0 = ((blockIdx.x + i * gridDim.x) % m_tiles) * kWgBN;
                bool ok = true;
                for (int kt = 0; kt < KT; ++kt, ++j) {
                    // stage j % 4 is free once the MMAs of step j - 4 have completed
                    if (j >= kWgActStages &&
                        !mbar_wait_bounded(&a_empty[(j - kWgActStages) % kWgAStages],
                                           ((j - kWgActStages) / kWgAStages) & 1, abort_flag,
                                           wait_ns, kDevErrTimeoutProducer)) {
                        ok = false;
                        break;
                    }
                    const int s = j % kWgActStages;
                    mbar_arrive_expect_tx(&act_full[s], kWgActBytes);
                    tma_load_2d(&tmap_x, &act_full[s], sAct + s * kWgActBytes, kt * kWgBK, m0);
                    ++issued;
                }
                if (!ok) break;
            }
            if (*abort_flag) {
                uint32_t never = 0u;
                for (int q = issued > kWgActStages ? issued - kWgActStages : 0; q < issued; ++q)
                    (void)mbar_wait_bounded(&act_full[q % kWgActStages], (q / kWgActStages) & 1,
                                            &never, wait_ns, 0u);
            }
        }
    } else if (warp == 18) {
        // ------------------------------------------------ packed-weight producer
        if (lane == 0) {
            int j = 0, issued = 0;
            for (int i = 0; i < my_tiles && !*abort_flag; ++i) {
                const int n0 = ((blockIdx.x + i * gridDim.x) / m_tiles) * kWgBM;
                bool ok = true;
                for (int kt = 0; kt < KT; ++kt, ++j) {
                    const int s = j % kWgWStages;
                    // stage s is free once the dequant of step j - 4 has read it
                    if (!mbar_wait_bounded(&w_empty[s], ((j / kWgWStages) & 1) ^ 1, abort_flag,
                                           wait_ns, kDevErrTimeoutProducer)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&w_full[s], kWgWBytes);
                    tma_load_2d(&tmap_q, &w_full[s], sW + s * kWgWBytes, kt * (kWgBK / 2), n0);
                    ++issued;
                }
                if (!ok) break;
            }
            if (*abort_flag) {
                uint32_t never = 0u;
                for (int q = issued > kWgWStages ? issued - kWgWStages : 0; q < issued; ++q)
                    (void)mbar_wait_bounded(&w_full[q % kWgWStages], (q / kWgWStages) & 1, &never,
                                            wait_ns, 0u);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16(kWgBM, kWgBN);
            // B descriptors: stage s starts (s * bytes) / 16 units above stage 0,
            // MMA kk of a stage 32 bytes = 2 units further (the address field
            // cannot carry: shared addresses are below 2^18)
            const uint64_t bdesc0 = umma_desc_sw128(smem_u32(sAct));
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
                    const int as = j % kWgAStages, s = j % kWgActStages;
                    // the dequantized weights (usually ready well ahead), then the tokens
                    if (!mbar_wait_bounded(&a_full[as], (j / kWgAStages) & 1, abort_flag, wait_ns,
                                           kDevErrTimeoutConsumer) ||
                        !mbar_wait_bounded(&act_full[s], (j / kWgActStages) & 1, abort_flag,
                                           wait_ns, kDevErrTimeoutConsumer)) {
                        ok = false;
                        break;
                    }
                    tcgen05_fence_after();
                    const uint32_t a_tmem = tmem_base + kWgColA + 32 * as;
                    const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(s * (kWgActBytes >> 4));
#pragma unroll
                    for (int kk = 0; kk < kWgBK / 16; ++kk)
                        umma_bf16_ts(tmem_base + kWgColD, a_tmem + 8 * kk, bdesc + 2 * kk, idesc,
                                     (kt | kk) != 0);
                    umma_commit(&a_empty[as]);
                }
                if (ok) umma_commit(acc_full);
            }
            umma_commit(final_bar);
            uint32_t never = 0u;
            (void)mbar_wait_bounded(final_bar, 0, &never, wait_ns, 0u);
        }
        __syncwarp();
    } else if (warp < 10) {
        // ------------------------------------------------ dequant -> TMEM (warps 2-9)
        const int q = warp & 3;                 // TMEM lane quarter
        const int r = q * 32 + lane;            // weight row within the tile
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        // a row is 32 bytes (two 16-byte chunks), rows 32 bytes apart: lanes r
        // and r + 4 of a load phase take different chunks first, so the 8
        // lanes of a phase cover the 32 banks once
        const int c0 = (r >> 2) & 1;
        const int par = warp < 6 ? 0 : 1;       // K-step parity of this warp
        // scale and zero point of this row for the group of step j
        auto load_sz = [&](int j, uint32_t& zc, uint32_t& s2) {
            const int tile = blockIdx.x + (j / KT) * gridDim.x;
            const int n = (tile / m_tiles) * kWgBM + r;
            const int g = (j % KT) / 2;
            uint16_t sb = 0, zb = 0;
            if (n < N) {
                sb = __ldca(reinterpret_cast<const unsigned short*>(wscale) +
                            static_cast<size_t>(n) * ngroups + g);
                zb = __ldca(wzero + static_cast<size_t>(n) * ngroups + g);
            }
            const uint32_t zh = 0x4300u | zb;   // bf16(128 + z)
            zc = zh | (zh << 16);
            s2 = static_cast<uint32_t>(sb) | (static_cast<uint32_t>(sb) << 16);
        };
        uint32_t zc = 0, s2 = 0, zc_next = 0, s2_next = 0;
        if (par < total) load_sz(par, zc_next, s2_next);
        for (int j = par; j < total; j += 2) {
            zc = zc_next;
            s2 = s2_next;
            if (j + 2 < total) load_sz(j + 2, zc_next, s2_next);   // lands while this step runs
            const int ws = j % kWgWStages, as = j % kWgAStages;
            if (!warp_wait(&w_full[ws], (j / kWgWStages) & 1, abort_flag, wait_ns,
                              kDevErrTimeoutConsumer))
                break;
            const uint8_t* row = sW + ws * kWgWBytes + r * 32;
            const uint4 p0 = lds128(row + 16 * c0);
            const uint4 p1 = lds128(row + 16 * (c0 ^ 1));
            const uint4 lo = c0 ? p1 : p0, hi = c0 ? p0 : p1;   // K 0..31 / 32..63 of the step
            const uint32_t wv[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
            uint32_t a[32];
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                uint32_t o[4];
                dequant8(wv[v], zc, s2, o);
#pragma unroll
                for (int p = 0; p < 4; ++p) a[4 * v + p] = o[p];
            }
            // the packed stage is in registers (the values above depend on every
            // load): the weight producer may refill it
            __syncwarp();
            if (lane == 0) mbar_arrive(&w_empty[ws]);
            // TMEM stage as is free once the MMAs of step j - 8 have completed
            if (j >= kWgAStages &&
                !warp_wait(&a_empty[as], ((j - kWgAStages) / kWgAStages) & 1, abort_flag,
                              wait_ns, kDevErrTimeoutConsumer))
                break;
            tcgen05_fence_after();
            tmem_st_32x32b_x32(tmem_base + lane_base + kWgColA + 32 * as, a);
            tmem_st_wait();
            tcgen05_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[as]);
        }
    } else if (warp < 18) {
        // ------------------------------------------------ epilogue (warps 10-17)
        const int e = warp - 10;
        const int q = warp & 3;
        const int half = e >> 2;
        const int r = q * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        const bool leader = (e == 0 && lane == 0);
        for (int i = 0; i < my_tiles; ++i) {
            const int tile = blockIdx.x + i * gridDim.x;
            const int m0 = (tile % m_tiles) * kWgBN;
            const int n0 = (tile / m_tiles) * kWgBM;
            if (leader) {
                const bool ok = mbar_wait_bounded(acc_full, i & 1, abort_flag,
                                                  wait_ns, kDevErrTimeoutEpilogue);
                *epi_go = ok ? 1u : 0u;
            }
            named_barrier_sync(1, 256);
            if (*epi_go == 0u) break;
            tcgen05_fence_after();
            // 32 tokens from registers: fp32 sums rounded to bf16 (two at a time)
            // into the staging tile (row = token, 256 bytes; column = this
            // thread's row)
            auto emit = [&](int cc, const uint32_t (&acc)[32]) {
                const uint32_t dst = smem_u32(sOut + cc * (kWgBM * 2) + r * 2);
#pragma unroll
                for (int jj = 0; jj < 32; jj += 2) {
                    const uint32_t h2 =
                        f2_to_bf16x2(f2_pack(__uint_as_float(acc[jj]), __uint_as_float(acc[jj + 1])));
                    asm volatile(
                        "{\n\t.reg .b16 l, h;\n\t"
                        "mov.b32 {l, h}, %2;\n\t"
                        "st.shared.b16 [%0], l;\n\t"
                        "st.shared.b16 [%1], h;\n\t}" ::"r"(dst + jj * (kWgBM * 2)),
                        "r"(dst + (jj + 1) * (kWgBM * 2)), "r"(h2)
                        : "memory");
                }
            };
            // two chunks per TMEM read; the accumulator goes back to the MMAs
            // after this warp's last read, before the math on it
            bool released = false;
            const int cend = (half + 1) * (kWgBN / 2);
#pragma unroll 1
            for (int cc = half * (kWgBN / 2); cc < cend; cc += 64) {
                if (m0 + cc >= M) break;   // warp-uniform
                const bool two = cc + 32 < cend && m0 + cc + 32 < M;   // warp-uniform
                uint32_t acc0[32], acc1[32];
                tmem_ld_32x32b_x32(tmem_base + lane_base + kWgColD + cc, acc0);
                if (two) tmem_ld_32x32b_x32(tmem_base + lane_base + kWgColD + cc + 32, acc1);
                tmem_ld_wait();
                if (cc + 64 >= cend || m0 + cc + 64 >= M) {   // warp-uniform
                    tcgen05_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(acc_empty);
                    released = true;
                }
                emit(cc, acc0);
                if (two) emit(cc + 32, acc1);
            }
            if (!released) {   // no token of this warp's half below M
                tcgen05_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty);
            }
            named_barrier_sync(1, 256);
            const int et = e * 32 + lane;
#pragma unroll 4
            for (int c = et; c < kWgBN * (kWgBM / 8); c += 256) {
                const int tok = c >> 4, piece = c & 15;
                if (m0 + tok < M && n0 + piece * 8 < N)
                    *reinterpret_cast<uint4*>(y + static_cast<size_t>(m0 + tok) * N + n0 + piece * 8) =
                        lds128(sOut + tok * (kWgBM * 2) + piece * 16);
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
