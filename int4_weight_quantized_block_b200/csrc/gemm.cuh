// gemm.cuh -- packed-INT4-weight integer GEMM on the sm_100a tensor cores.
//
//   acc[m, n] = sum_k qa[m, k] * qw[n, k]            (int32, exact)
//   y[m, n]   = bf16( acc * s_tok[m] * s_row[n] (+ bias[n]) )
//
// "ComfyUI-INT-Crush", "Inference > INT4 > CUDA backend": INT4 weights are
// unpacked to INT8 and fed to an INT8 GEMM with fused dequant; "Inference >
// INT4 > Triton backend": W4A8 = unpack + dynamically quantized activations +
// fused INT8 GEMM + dequant.  stable-diffusion.cpp "feat: packed int4 convrot
// model loading and dispatch", "Summary": the packed nibbles stream to the
// backend unconverted, about half a byte per weight.
//
// Here the packed weights are never widened in HBM.  Each CTA computes one
// 128 x BN output tile with four roles:
//   warp 0      TMA producer: per 128-wide K step, one tile of activation
//               codes (int8, or packed int4 for W4A4) and one tile of packed
//               weights (BN rows x 64 bytes) into a STAGES-deep ring.
//   warp 1      TMEM owner and single-thread UMMA issuer:
//               tcgen05.mma.cta_group::1.kind::i8, M = 128, N = BN, K = 32,
//               four per stage, int32 accumulators in TMEM.
//   warps 2-5   unpack: sign-extend every weight nibble to an int8 into the
//               128-byte-swizzled K-major layout the tensor core reads (and,
//               for W4A4, the activation nibbles too), then, after the last
//               K step, the epilogue: tcgen05.ld of the accumulator, the scale
//               product, bf16 rounding, stores.
//
// Nibble unpack without sign-extension arithmetic: a nibble moved to the high
// half of its byte, with the low half cleared, is the int8 value 16 * code.
// The tensor core therefore accumulates 16 * acc (W4A8) or 256 * acc (W4A4;
// both operands unpacked this way), which the epilogue shifts back exactly.
// |16 * acc| <= 16 * 127 * 7 * K stays inside int32 for K <= 65536.  For
// W4A4 the unpack leaves the K order inside each 8-value group permuted
// (even positions, then odd), identically for both operands, which leaves
// every dot product unchanged; for W4A8 a byte permute restores the natural
// K order so that the TMA-loaded int8 activations line up.
#pragma once

#include "ptx.cuh"

namespace tint4 {

constexpr int kGemmBM = 128;       // UMMA M (rows of activations per tile)
constexpr int kGemmBK = 128;       // K values per pipeline stage (128 bytes of int8)
constexpr int kGemmThreads = 192;  // 6 warps
constexpr int kGemmUnpackThreads = 128;

template <bool A_INT4, int BN, int STAGES>
struct GemmLayout {
    static constexpr int kABytes = kGemmBM * kGemmBK;              // int8 A tile, swizzled
    static constexpr int kApBytes = A_INT4 ? kGemmBM * kGemmBK / 2 : 0;  // packed A tile
    static constexpr int kWpBytes = BN * kGemmBK / 2;              // packed W tile
    static constexpr int kBBytes = BN * kGemmBK;                   // int8 W tile, swizzled
    static constexpr int kStageBytes = kABytes + kApBytes + kWpBytes + kBBytes;
    static constexpr int kOffA = 0;
    static constexpr int kOffB = kOffA + STAGES * kABytes;
    static constexpr int kOffWp = kOffB + STAGES * kBBytes;
    static constexpr int kOffAp = kOffWp + STAGES * kWpBytes;
    static constexpr int kOffBar = kOffAp + STAGES * kApBytes;
    static constexpr int kBarBytes = 256;
    // + 1024 so the kernel can round the dynamic smem base up to 1024 bytes
    static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;
    static constexpr uint32_t kTxBytes = (A_INT4 ? kApBytes : kABytes) + kWpBytes;
    static_assert(kABytes % 1024 == 0 && kBBytes % 1024 == 0, "swizzled tiles need 1 KB");
    static_assert(kWpBytes % 1024 == 0, "tile alignment");
    static_assert(3 * STAGES * 8 + 8 + 8 <= kBarBytes, "barrier area");
};

// 32 packed nibbles (K order, low nibble first) -> 32 int8 values x16 in
// natural K order (W4A8 weights).
__device__ __forceinline__ void unpack32_natural(const uint4 p, uint4& lo, uint4& hi) {
    const uint32_t w[4] = {p.x, p.y, p.z, p.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t L = (w[i] << 4) & 0xF0F0F0F0u;  // even-K nibbles, x16
        const uint32_t H = w[i] & 0xF0F0F0F0u;         // odd-K nibbles, x16
        o[2 * i] = __byte_perm(L, H, 0x5140);          // K 8i+0..3
        o[2 * i + 1] = __byte_perm(L, H, 0x7362);      // K 8i+4..7
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// 32 packed nibbles -> 32 int8 values x16 with the K order inside each word
// permuted to (0,2,4,6,1,3,5,7).  Used for both operands of W4A4.
__device__ __forceinline__ void unpack32_permuted(const uint4 p, uint4& lo, uint4& hi) {
    const uint32_t w[4] = {p.x, p.y, p.z, p.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        o[2 * i] = (w[i] << 4) & 0xF0F0F0F0u;
        o[2 * i + 1] = w[i] & 0xF0F0F0F0u;
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// Unpack `rows` rows of 64 packed bytes (one K stage) from `src` into the
// 128-byte swizzled K-major int8 layout at `dst`.  Thread t of the 128 unpack
// threads handles 16-byte pieces t, t + 128, ...; a piece is 32 K values of
// one row and becomes two swizzled 16-byte chunks.  Both the reads (8 lanes
// cover 128 contiguous bytes) and the writes (8 lanes hit 8 distinct chunk
// positions) are free of bank conflicts.
template <int ROWS, bool PERMUTED>
__device__ __forceinline__ void unpack_stage(const uint8_t* src, uint8_t* dst, int t) {
#pragma unroll 4
    for (int it = 0; it < ROWS * 4 / kGemmUnpackThreads; ++it) {
        const int piece = t + it * kGemmUnpackThreads;
        const int row = piece >> 2;
        const int c16 = piece & 3;
        const uint4 p = lds128(src + row * 64 + c16 * 16);
        uint4 lo, hi;
        if (PERMUTED) unpack32_permuted(p, lo, hi);
        else unpack32_natural(p, lo, hi);
        uint8_t* rowp = dst + (row >> 3) * 1024 + (row & 7) * 128;
        sts128(rowp + (((2 * c16) ^ (row & 7)) << 4), lo);
        sts128(rowp + (((2 * c16 + 1) ^ (row & 7)) << 4), hi);
    }
}

template <bool A_INT4, int BN, int STAGES, bool OUT_I32>
__global__ void __launch_bounds__(kGemmThreads, 1)
w4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
               const __grid_constant__ CUtensorMap tmap_w,
               const float* __restrict__ tok_scale, const float* __restrict__ row_scale,
               const __nv_bfloat16* __restrict__ bias, void* __restrict__ out, int M, int N,
               int K, uint64_t wait_ns) {
    using L = GemmLayout<A_INT4, BN, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem + L::kOffA;
    uint8_t* sB = smem + L::kOffB;
    uint8_t* sWp = smem + L::kOffWp;
    uint8_t* sAp = smem + L::kOffAp;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint64_t* unpacked = full + STAGES;
    uint64_t* empty = unpacked + STAGES;
    uint64_t* acc_full = empty + STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BN;
    const int m0 = blockIdx.y * kGemmBM;
    const int KT = (K + kGemmBK - 1) / kGemmBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&unpacked[s], kGemmUnpackThreads);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        *abort_flag = 0u;
        fence_mbarrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmap_a);
        prefetch_tensormap(&tmap_w);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, BN);
        tmem_relinquish();
    }
    tcgen05_fence_before();
    __syncthreads();
    tcgen05_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // The activation codes and token scales may come from the grid launched
    // just before this one (programmatic dependent launch).
    grid_dependency_wait();

    if (warp == 0) {
        if (lane == 0) {
            int issued = 0;
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % STAGES;
                const uint32_t ph = (kt / STAGES) & 1;
                if (!mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, wait_ns,
                                       kDevErrTimeoutProducer))
                    break;
                mbar_arrive_expect_tx(&full[s], L::kTxBytes);
                if (A_INT4) tma_load_2d(&tmap_a, &full[s], sAp + s * L::kApBytes, kt * 64, m0);
                else tma_load_2d(&tmap_a, &full[s], sA + s * L::kABytes, kt * kGemmBK, m0);
                tma_load_2d(&tmap_w, &full[s], sWp + s * L::kWpBytes, kt * 64, n0);
                ++issued;
            }
            if (*abort_flag) {
                // drain: do not leave bulk copies landing in a CTA that is gone
                uint32_t never = 0u;
                for (int j = (issued > STAGES ? issued - STAGES : 0); j < issued; ++j)
                    (void)mbar_wait_bounded(&full[j % STAGES], (j / STAGES) & 1, &never,
                                            wait_ns, 0u);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_i8(kGemmBM, BN);
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % STAGES;
                const uint32_t ph = (kt / STAGES) & 1;
                if (!mbar_wait_bounded(&full[s], ph, abort_flag, wait_ns, kDevErrTimeoutConsumer))
                    break;
                if (!mbar_wait_bounded(&unpacked[s], ph, abort_flag, wait_ns,
                                       kDevErrTimeoutConsumer))
                    break;
                tcgen05_fence_after();
                const uint32_t a_addr = smem_u32(sA + s * L::kABytes);
                const uint32_t b_addr = smem_u32(sB + s * L::kBBytes);
#pragma unroll
                for (int kk = 0; kk < kGemmBK / 32; ++kk) {
                    umma_i8_ss(tmem_base, umma_desc_sw128(a_addr + kk * 32),
                               umma_desc_sw128(b_addr + kk * 32), idesc, (kt | kk) != 0);
                }
                umma_commit(&empty[s]);
            }
            // every MMA issued so far lands before acc_full flips (also on abort,
            // so that the TMEM is quiet before it is freed)
            umma_commit(acc_full);
            uint32_t never = 0u;
            (void)mbar_wait_bounded(acc_full, 0, &never, wait_ns, 0u);
        }
        __syncwarp();   // lanes 1-31 park here instead of polling a barrier
    } else {
        const int t = threadIdx.x - 64;  // 0..127
        for (int kt = 0; kt < KT; ++kt) {
            const int s = kt % STAGES;
            const uint32_t ph = (kt / STAGES) & 1;
            if (!mbar_wait_bounded(&full[s], ph, abort_flag, wait_ns, kDevErrTimeoutConsumer))
                break;
            unpack_stage<BN, A_INT4>(sWp + s * L::kWpBytes, sB + s * L::kBBytes, t);
            if (A_INT4) unpack_stage<kGemmBM, true>(sAp + s * L::kApBytes, sA + s * L::kABytes, t);
            fence_proxy_async_smem();
            mbar_arrive(&unpacked[s]);
        }

        // ---- epilogue: TMEM -> registers -> scale -> bf16 -> global
        bool ok = mbar_wait_bounded(acc_full, 0, abort_flag, wait_ns, kDevErrTimeoutEpilogue);
        // tcgen05.ld is warp-collective: the whole warp takes the same branch
        ok = __all_sync(0xFFFFFFFFu, ok && !*abort_flag);
        if (ok) {
            tcgen05_fence_after();
            const int q = warp & 3;  // TMEM lane quarter this warp may access
            const int row = m0 + q * 32 + lane;
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
            const float st = (row < M) ? __ldg(tok_scale + row) : 0.0f;
            constexpr int shift = A_INT4 ? 8 : 4;
            for (int c0 = 0; c0 < BN; c0 += 32) {
                if (n0 + c0 >= N) break;  // warp-uniform
                uint32_t r[32];
                tmem_ld_32x32b_x32(taddr + c0, r);
                tmem_ld_wait();
                if (row >= M) continue;
                const int nb = n0 + c0;
                const bool full_chunk = nb + 32 <= N;
                if (OUT_I32) {
                    int32_t* o = static_cast<int32_t*>(out) + static_cast<size_t>(row) * N + nb;
                    if (full_chunk) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            int4 v = make_int4(static_cast<int32_t>(r[j]) >> shift,
                                               static_cast<int32_t>(r[j + 1]) >> shift,
                                               static_cast<int32_t>(r[j + 2]) >> shift,
                                               static_cast<int32_t>(r[j + 3]) >> shift);
                            *reinterpret_cast<int4*>(o + j) = v;
                        }
                    } else {
                        for (int j = 0; j < 32 && nb + j < N; ++j)
                            o[j] = static_cast<int32_t>(r[j]) >> shift;
                    }
                } else {
                    float sr[32];
                    if (full_chunk) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            const float4 v = __ldg(reinterpret_cast<const float4*>(row_scale + nb + j));
                            sr[j] = v.x; sr[j + 1] = v.y; sr[j + 2] = v.z; sr[j + 3] = v.w;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) sr[j] = (nb + j < N) ? __ldg(row_scale + nb + j) : 0.0f;
                    }
                    uint32_t packed[16];
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        float y0 = static_cast<float>(static_cast<int32_t>(r[j]) >> shift) * st * sr[j];
                        float y1 = static_cast<float>(static_cast<int32_t>(r[j + 1]) >> shift) * st * sr[j + 1];
                        if (bias != nullptr) {
                            if (nb + j < N) y0 += __bfloat162float(bias[nb + j]);
                            if (nb + j + 1 < N) y1 += __bfloat162float(bias[nb + j + 1]);
                        }
                        const __nv_bfloat162 h = __floats2bfloat162_rn(y0, y1);
                        packed[j / 2] = *reinterpret_cast<const uint32_t*>(&h);
                    }
                    __nv_bfloat16* o =
                        static_cast<__nv_bfloat16*>(out) + static_cast<size_t>(row) * N + nb;
                    if (full_chunk) {
#pragma unroll
                        for (int j = 0; j < 16; j += 4)
                            *reinterpret_cast<uint4*>(o + 2 * j) =
                                make_uint4(packed[j], packed[j + 1], packed[j + 2], packed[j + 3]);
                    } else {
                        for (int j = 0; j < 32 && nb + j < N; ++j) {
                            const uint32_t w = packed[j / 2];
                            const uint16_t b = (j & 1) ? static_cast<uint16_t>(w >> 16)
                                                       : static_cast<uint16_t>(w & 0xFFFF);
                            reinterpret_cast<uint16_t*>(o)[j] = b;
                        }
                    }
                }
            }
        }
    }

    // ---- teardown: the accumulator is quiet (warp 1 waited on acc_full,
    // also on abort) before TMEM is released
    tcgen05_fence_before();
    __syncthreads();
    if (warp == 1) {
        tcgen05_fence_after();
        tmem_dealloc(tmem_base, BN);
    }
}

}  // namespace tint4
