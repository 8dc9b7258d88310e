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
// Warp roles (18 warps, one persistent CTA per SM, static tile list):
//   warp 0      TMA producer (4-deep ring of 32 KB token + 4 KB weight stages)
//   warp 1      TMEM owner; one thread issues tcgen05.mma.kind::f16 (A bf16
//               from TMEM, B bf16 from shared memory, fp32 D; M 128, N 256, K 16)
//   warps 2-9   dequant into the 4 TMEM A stages (32 columns each)
//   warps 10-17 epilogue: tcgen05.ld of the accumulator two 32-token chunks
//               at a time, handed back to the MMAs after the last read,
//               rounding to bf16 into a [256 tokens][128 columns] staging
//               tile, copied to y in 16-byte row pieces.
// TMEM columns: one accumulator at 0 (256 columns), A stages at 256 + 32 s.
// (256 tokens per tile rather than 192 with two accumulators: the dequant
// work of a step, the kernel's critical path, then serves a third more
// tokens.)
#pragma once

#include "ptx.cuh"

namespace tint4 {

constexpr int kWgBM = 128;       // weight rows per tile (UMMA M, TMEM lanes)
constexpr int kWgBN = 256;       // tokens per tile (UMMA N)
constexpr int kWgBK = 64;        // K values per stage (bf16: 128-byte rows)
constexpr int kWgStages = 4;     // shared-memory stages = TMEM A stages
constexpr int kWgThreads = 576;  // 18 warps
constexpr int kWgGroup = 128;    // quantization group along K
constexpr int kWgActBytes = kWgBN * kWgBK * 2;        // 32 KB token tile per stage
constexpr int kWgWBytes = kWgBM * kWgBK / 2;          // 4 KB packed weights per stage
constexpr int kWgOutBytes = kWgBN * kWgBM * 2;        // 64 KB bf16 staging tile
constexpr int kWgSmemBytes = kWgStages * (kWgActBytes + kWgWBytes) + kWgOutBytes + 256 + 1024;
constexpr uint32_t kWgColD = 0;                       // the accumulator
constexpr uint32_t kWgColA = kWgBN;                   // A stage s at kWgColA + 32 s
static_assert(kWgColA + 32 * kWgStages <= 512, "TMEM budget");
// warps 2-5 take the even K steps and 6-9 the odd ones, so a stage must belong
// to one chain (an even count): a chain then waits on its stages' phases in
// order and a parity wait cannot pass on a phase it skipped
static_assert(kWgStages % 2 == 0, "stages of one chain");
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
    uint8_t* sW = smem + kWgStages * kWgActBytes;
    uint8_t* sOut = sW + kWgStages * kWgWBytes;
    uint64_t* act_full = reinterpret_cast<uint64_t*>(sOut + kWgOutBytes);
    uint64_t* a_full = act_full + kWgStages;       // TMEM A stage written (one arrival per warp)
    uint64_t* empty = a_full + kWgStages;          // stage consumed by the MMAs (commit)
    uint64_t* acc_full = empty + kWgStages;        // accumulator ready (commit)
    uint64_t* acc_empty = acc_full + 2;            // accumulator read (8 warp arrivals)
    uint64_t* final_bar = acc_empty + 2;           // all MMAs done (teardown)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;
    volatile uint32_t* epi_go = tmem_slot + 2;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int m_tiles = (M + kWgBN - 1) / kWgBN;
    const int n_tiles = (N + kWgBM - 1) / kWgBM;
    const int n_work = m_tiles * n_tiles;
    const int KT = K / kWgBK;                      // even: K % 128 == 0
    const int ngroups = K / kWgGroup;
    const int my_tiles = (blockIdx.x < n_work) ? (n_work - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kWgStages; ++s) {
            mbar_init(&act_full[s], 1);
            mbar_init(&a_full[s], 4);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 8);
        }
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

    // x may come from the grid launched just before
    grid_dependency_wait();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t c = 0;
            int issued = 0;
            for (int i = 0; i < my_tiles && !*abort_flag; ++i) {
                const int tile = blockIdx.x + i * gridDim.x;
                const int m0 = (tile % m_tiles) * kWgBN;
                const int n0 = (tile / m_tiles) * kWgBM;
                for (int kt = 0; kt < KT; ++kt, ++c) {
                    const int s = c % kWgStages;
                    const uint32_t ph = (c / kWgStages) & 1;
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, wait_ns,
                                           kDevErrTimeoutProducer))
                        break;
                    mbar_arrive_expect_tx(&act_full[s], kWgActBytes + kWgWBytes);
                    tma_load_2d(&tmap_x, &act_full[s], sAct + s * kWgActBytes, kt * kWgBK, m0);
                    tma_load_2d(&tmap_q, &act_full[s], sW + s * kWgWBytes, kt * (kWgBK / 2), n0);
                    ++issued;
                }
            }
            if (*abort_flag) {
                uint32_t never = 0u;
                const int first = issued > kWgStages ? issued - kWgStages : 0;
                for (int j = first; j < issued; ++j)
                    (void)mbar_wait_bounded(&act_full[j % kWgStages], (j / kWgStages) & 1, &never,
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
            int s = 0;
            uint32_t ph = 0u;
            bool ok = true;
            for (int i = 0; i < my_tiles && ok; ++i) {
                const int buf = 0;
                const uint32_t aph = i & 1;
                if (!mbar_wait_bounded(&acc_empty[buf], aph ^ 1, abort_flag, wait_ns,
                                       kDevErrTimeoutConsumer)) {
                    ok = false;
                    break;
                }
                tcgen05_fence_after();
                const uint32_t d_tmem = tmem_base + kWgColD + buf * kWgBN;
                for (int kt = 0; kt < KT; ++kt) {
                    // a_full implies the stage has landed: the unpack warps arrive
                    // on it only after they have seen it (one wait per stage: the
                    // issuing thread's time per stage is the tensor pipe's budget)
                    if (!mbar_wait_bounded(&a_full[s], ph, abort_flag, wait_ns,
                                           kDevErrTimeoutConsumer)) {
                        ok = false;
                        break;
                    }
                    tcgen05_fence_after();
                    const uint32_t a_tmem = tmem_base + kWgColA + 32 * s;
                    const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(s * (kWgActBytes >> 4));
#pragma unroll
                    for (int kk = 0; kk < kWgBK / 16; ++kk)
                        umma_bf16_ts(d_tmem, a_tmem + 8 * kk, bdesc + 2 * kk, idesc, (kt | kk) != 0);
                    umma_commit(&empty[s]);
                    if (++s == kWgStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (ok) umma_commit(&acc_full[buf]);
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
        const int total = my_tiles * KT;
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
            const int s = j % kWgStages;
            const uint32_t ph = (j / kWgStages) & 1;
            if (!warp_wait(&act_full[s], ph, abort_flag, wait_ns, kDevErrTimeoutConsumer)) break;
            const uint8_t* row = sW + s * kWgWBytes + r * 32;
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
            // the TMEM A stage is free: its previous MMAs completed before the
            // producer refilled this stage (empty[s] -> act_full[s])
            tcgen05_fence_after();
            tmem_st_32x32b_x32(tmem_base + lane_base + kWgColA + 32 * s, a);
            tmem_st_wait();
            tcgen05_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[s]);
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
                const bool ok = mbar_wait_bounded(&acc_full[0], i & 1, abort_flag,
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
                for (int j = 0; j < 32; j += 2) {
                    const uint32_t h2 =
                        f2_to_bf16x2(f2_pack(__uint_as_float(acc[j]), __uint_as_float(acc[j + 1])));
                    asm volatile(
                        "{\n\t.reg .b16 l, h;\n\t"
                        "mov.b32 {l, h}, %2;\n\t"
                        "st.shared.b16 [%0], l;\n\t"
                        "st.shared.b16 [%1], h;\n\t}" ::"r"(dst + j * (kWgBM * 2)),
                        "r"(dst + (j + 1) * (kWgBM * 2)), "r"(h2)
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
                    if (lane == 0) mbar_arrive(&acc_empty[0]);
                    released = true;
                }
                emit(cc, acc0);
                if (two) emit(cc + 32, acc1);
            }
            if (!released) {   // no token of this warp's half below M
                tcgen05_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[0]);
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
