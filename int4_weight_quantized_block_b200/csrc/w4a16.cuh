// w4a16.cuh -- W4A16 group-wise asymmetric linear for small M (decode).
//
//   y[m, n] = sum_k x[m, k] * (q[n, k] - z[n, k/G]) * s[n, k/G]
//
// "TINT4 v1.2 -- torchao INT4 for ComfyUI", "v1.1 新特性 > 5": the layer
// keeps _qdata / _scale / _zp; "参数选择指南": group_size 128 standard.
// "ComfyUI-INT-Crush", "Inference > INT4 > Triton backend": W4A16 is the
// rot_size == 0 path (INT4 -> 16-bit unpack + 16-bit GEMM).
//
// The cost is streaming the packed weights from HBM (0.5 byte per weight plus
// 3 bytes of scale and zero point per 128 weights); every weight is used by
// at most 32 tokens.  Per group the sum is
//   s * sum_k x_k * (q_k - z)
// with q_k - z formed exactly in bf16: 0x4300 | q is bf16(128 + q), one
// shift + AND/OR per two nibbles from the packed bytes, and subtracting
// bf16(128 + z) leaves the small integer q - z.  The products run on the
// warp-level bf16 MMA (m16n8k16, fp32 accumulation): at M = 16 the 805 M
// multiply-adds of the 4096 x 12288 layer would take several times the HBM
// time on the fp32 CUDA cores.  Weights are the MMA's A operand straight from
// registers (16 rows x 128 K per warp step, one 16-byte load per lane and
// row), tokens the B operand (n = 8 per block).  The K order inside an MMA is
// permuted so that each lane's 32 packed nibbles map onto its own fragment
// slots; x is gathered in the same order, which leaves each dot product
// unchanged.
//
// Work split: a persistent grid of one (M <= 8: two) CTAs per SM; CTA c owns
// a contiguous run of 16-row blocks (at most MB).  A producer warp streams,
// two K groups at a time, the packed weights of those rows (one 16-row x
// 128-byte TMA box per block: whole 128-byte lines of every row, which DRAM
// serves best) and the matching x tile into an 8-deep shared-memory ring;
// consumer warp w takes stages w, w + 8, ... (ring slot w), reads its x
// fragments once per group and uses them for all of the CTA's row blocks, two
// blocks at a time so that independent MMA chains overlap.  The 8 partial
// sums of each output meet in shared memory at the end.
//
// The weight boxes use the 128-byte swizzle (16-byte chunk c of smem row r at
// c ^ (r & 7)).  The two rows an 8-lane phase reads would hit the same banks,
// so MMA row m holds weight row pi(m) = 4 (m & 1) + (m >> 1) (m < 8; +8 above),
// which puts them 4 rows apart and onto disjoint chunk sets: conflict-free.
#pragma once

#include "ptx.cuh"

namespace tint4 {

constexpr int kW16Warps = 8;
constexpr int kW16Threads = kW16Warps * 32;
constexpr int kW16Group = 128;       // K values per quantization group

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               const uint32_t b0, const uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// nibbles (i, i + 4) of a packed word -> bf16x2 (128 + q_i, 128 + q_{i+4})
__device__ __forceinline__ uint32_t nib_pair_bf16(uint32_t w, int i) {
    return ((w >> (4 * i)) & 0x000F000Fu) | 0x43004300u;
}

// elementwise a - b of two bf16 pairs (exact here: small integers)
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// x values 8w .. 8w + 7 of a lane's slice (one 16-byte word q, bf16) to the
// B fragments of k steps 2w (f0) and 2w + 1 (f1): k step 2w + h takes the
// values (2h, 2h + 4) and (2h + 1, 2h + 5), matching the nibble pairing of
// the weights
__device__ __forceinline__ void x_frag(const uint4& q, uint32_t (&f0)[2], uint32_t (&f1)[2]) {
    f0[0] = __byte_perm(q.x, q.z, 0x5410);
    f0[1] = __byte_perm(q.x, q.z, 0x7632);
    f1[0] = __byte_perm(q.y, q.w, 0x5410);
    f1[1] = __byte_perm(q.y, q.w, 0x7632);
}

constexpr int kW16Stages = 8;        // = consumer warps: warp w owns ring slot w
constexpr int kW16Threads9 = (kW16Warps + 1) * 32;   // + the TMA producer warp
constexpr int kW16GPS = 2;           // K groups per stage (128 packed bytes per row)
constexpr int kW16MaxK = 16384;      // scales / zero points of a CTA's rows stay in shared memory

// MMA row m (0..15) of a block holds weight row w16_perm(m) of the block
__host__ __device__ constexpr int w16_perm(int m) {
    return (m & 8) | ((m & 1) << 2) | ((m >> 1) & 3);
}

template <int NB, int MB>
struct W16Layout {
    static constexpr int kBoxBytes = 16 * 128;                          // one block, two groups
    static constexpr int kWBytes = MB * kBoxBytes;
    static constexpr int kXBytes = 8 * NB * kW16GPS * kW16Group * 2;     // x tile, two groups
    static constexpr int kStage = kWBytes + kXBytes;
    static constexpr int kRedBytes = kW16Warps * MB * NB * 32 * 16;
    static constexpr int kBarOff = kW16Stages * kStage > kRedBytes ? kW16Stages * kStage : kRedBytes;
    static constexpr int kSzOff = kBarOff + (2 * kW16Stages + 1) * 8 + 120;
    // the CTA's rows of scale (bf16) and zero point (uint8), all groups, as
    // they lie in global memory
    __host__ __device__ static constexpr int smem(int ngroups) {
        return kSzOff + MB * 16 * ngroups * 3 + 16 + 1024;   // + 1024: base alignment
    }
    static_assert(kStage % 1024 == 0, "swizzled boxes need 1 KB alignment");
};

// NB = number of 8-token blocks (M <= 8 * NB); MB = 16-row blocks per CTA at most.
template <int NB, int MB>
__global__ void __launch_bounds__(kW16Threads9, 1)
w4a16_mma_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                 const __nv_bfloat16* __restrict__ wscale, const uint8_t* __restrict__ wzero,
                 __nv_bfloat16* __restrict__ y, int M, int N, int K, uint64_t wait_ns) {
    using L = W16Layout<NB, MB>;
    extern __shared__ uint8_t w16_smem_raw[];
    uint8_t* w16_smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(w16_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(w16_smem + L::kBarOff);
    uint64_t* empty = full + kW16Stages;
    uint64_t* sz_full = empty + kW16Stages;        // scales + zero points landed
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sz_full + 1);
    float* red = reinterpret_cast<float*>(w16_smem);   // reused after the main loop

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2;   // MMA group id: MMA rows g / g + 8, token column g
    const int t = lane & 3;    // thread in group: which 32-value slice of a K group
    const int ngroups = K / kW16Group;
    const int nstages = (ngroups + kW16GPS - 1) / kW16GPS;
    const int nblk = (N + 15) / 16;
    // contiguous run of row blocks of this CTA
    const int b0 = static_cast<int>((static_cast<long long>(blockIdx.x) * nblk) / gridDim.x);
    const int b1 = static_cast<int>((static_cast<long long>(blockIdx.x + 1) * nblk) / gridDim.x);
    const int nb_here = b1 - b0;   // 1..MB (the host sizes the grid)
    const int rA = w16_perm(g), rB = w16_perm(g + 8);   // weight rows of MMA rows g, g + 8
    const int swz = rA & 7;                              // = rB & 7

    const __nv_bfloat16* sScale = reinterpret_cast<const __nv_bfloat16*>(w16_smem + L::kSzOff);
    const uint8_t* sZero = w16_smem + L::kSzOff + MB * 16 * ngroups * 2;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kW16Stages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(sz_full, 1);
        *abort_flag = 0u;
        fence_mbarrier_init();
    }
    __syncthreads();

    float total[MB][NB][4];
#pragma unroll
    for (int rb = 0; rb < MB; ++rb)
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int j = 0; j < 4; ++j) total[rb][b][j] = 0.0f;

    if (warp == kW16Warps) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tmap_w);
            prefetch_tensormap(&tmap_x);
            // this CTA's rows of scales and zero points are one contiguous,
            // 16-byte aligned range each (row starts are multiples of 16)
            const uint32_t sbytes = nb_here * 16 * ngroups * 2, zbytes = nb_here * 16 * ngroups;
            mbar_arrive_expect_tx(sz_full, sbytes + zbytes);
            bulk_load_1d(w16_smem + L::kSzOff, wscale + static_cast<size_t>(b0) * 16 * ngroups,
                         sbytes, sz_full);
            bulk_load_1d(w16_smem + L::kSzOff + MB * 16 * ngroups * 2,
                         wzero + static_cast<size_t>(b0) * 16 * ngroups, zbytes, sz_full);
            const uint32_t bytes = nb_here * L::kBoxBytes + L::kXBytes;
            int issued = 0;
            for (int j = 0; j < nstages; ++j) {
                const int s = j % kW16Stages;
                const uint32_t ph = (j / kW16Stages) & 1;
                if (!mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, wait_ns, kDevErrTimeoutProducer))
                    break;
                uint8_t* st = w16_smem + s * L::kStage;
                mbar_arrive_expect_tx(&full[s], bytes);
                for (int rb = 0; rb < nb_here; ++rb)
                    tma_load_2d(&tmap_w, &full[s], st + rb * L::kBoxBytes, j * 128, (b0 + rb) * 16);
                tma_load_2d(&tmap_x, &full[s], st + L::kWBytes, j * kW16GPS * kW16Group, 0);
                ++issued;
            }
            uint32_t never = 0u;
            if (*abort_flag) {
                // let the copies in flight land before the ring is reused or freed
                (void)mbar_wait_bounded(sz_full, 0, &never, wait_ns, 0u);
                for (int j = (issued > kW16Stages ? issued - kW16Stages : 0); j < issued; ++j)
                    (void)mbar_wait_bounded(&full[j % kW16Stages], (j / kW16Stages) & 1, &never,
                                            wait_ns, 0u);
            }
        }
    } else {
        // ------------------------------------------------ consumers
        int szok = 0;
        if (lane == 0) szok = mbar_wait_bounded(sz_full, 0, abort_flag, wait_ns, kDevErrTimeoutConsumer);
        if (__shfl_sync(0xFFFFFFFFu, szok, 0) == 0) goto consumers_done;
        for (int j = warp; j < nstages; j += kW16Warps) {
            const int s = j % kW16Stages;
            const uint32_t ph = (j / kW16Stages) & 1;
            int ok = 0;
            if (lane == 0) ok = mbar_wait_bounded(&full[s], ph, abort_flag, wait_ns, kDevErrTimeoutConsumer);
            if (__shfl_sync(0xFFFFFFFFu, ok, 0) == 0) break;
            const uint8_t* st = w16_smem + s * L::kStage;
#pragma unroll 1
            for (int gi = 0; gi < kW16GPS; ++gi) {
                const int G = j * kW16GPS + gi;
                if (G >= ngroups) break;   // warp-uniform
                // x fragments: token 8b + g, values 32t .. 32t + 31 of group G,
                // regrouped into the MMA's B layout
                // (with 4 token blocks the fragments of all 8 k steps would not
                // fit next to the sums: then they are re-read per row pair)
                constexpr bool kXReload = NB >= 4;
                const uint8_t* xg = st + L::kWBytes + g * (kW16GPS * kW16Group * 2) + gi * (kW16Group * 2) + 64 * t;
                uint32_t bfr[kXReload ? 1 : NB][kXReload ? 1 : 8][2];
                if constexpr (!kXReload) {
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        const uint8_t* xr = xg + 8 * b * (kW16GPS * kW16Group * 2);
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            const uint4 q = lds128(xr + 16 * w);
                            x_frag(q, bfr[b][2 * w], bfr[b][2 * w + 1]);
                        }
                    }
                }
                // this lane's 16-byte chunk of group G in rows rA / rB (swizzled)
                const int chunk_off = ((4 * gi + t) ^ swz) << 4;
                // row blocks in pairs: two independent dequant + MMA chains per
                // k step keep the tensor pipe and the ALUs busy together
#pragma unroll
                for (int rp = 0; rp < MB; rp += 2) {
                    if (rp >= nb_here) break;   // CTA-uniform
                    uint32_t wa[2][4], wb[2][4], zA[2], zB[2];
                    float sA[2], sB[2];
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        // a missing second block (odd count) reads a stale box;
                        // its sums are dropped below
                        const int rb = min(rp + p, MB - 1);
                        const uint8_t* box = st + rb * L::kBoxBytes;
                        const uint4 pa = lds128(box + rA * 128 + chunk_off);
                        const uint4 pb = lds128(box + rB * 128 + chunk_off);
                        wa[p][0] = pa.x; wa[p][1] = pa.y; wa[p][2] = pa.z; wa[p][3] = pa.w;
                        wb[p][0] = pb.x; wb[p][1] = pb.y; wb[p][2] = pb.z; wb[p][3] = pb.w;
                        sA[p] = __bfloat162float(sScale[(rb * 16 + rA) * ngroups + G]);
                        sB[p] = __bfloat162float(sScale[(rb * 16 + rB) * ngroups + G]);
                        // bf16x2 (128 + z, 128 + z): subtracting it from (128 + q) leaves q - z exactly
                        zA[p] = 0x43004300u | (0x00010001u * sZero[(rb * 16 + rA) * ngroups + G]);
                        zB[p] = 0x43004300u | (0x00010001u * sZero[(rb * 16 + rB) * ngroups + G]);
                    }
                    float acc[2][NB][4];
#pragma unroll
                    for (int p = 0; p < 2; ++p)
#pragma unroll
                        for (int b = 0; b < NB; ++b)
#pragma unroll
                            for (int q = 0; q < 4; ++q) acc[p][b][q] = 0.0f;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int w = k >> 1;          // packed word of this lane's 16 bytes
                        const int i0 = 2 * (k & 1);    // nibble pairs (i0, i0+4) and (i0+1, i0+5)
                        uint32_t bk[NB][2];
                        if constexpr (kXReload) {
                            uint32_t unused[2];
#pragma unroll
                            for (int b = 0; b < NB; ++b) {
                                const uint4 q = lds128(xg + 8 * b * (kW16GPS * kW16Group * 2) + 16 * w);
                                if (k & 1) x_frag(q, unused, bk[b]);
                                else x_frag(q, bk[b], unused);
                            }
                        } else {
#pragma unroll
                            for (int b = 0; b < NB; ++b) { bk[b][0] = bfr[b][k][0]; bk[b][1] = bfr[b][k][1]; }
                        }
#pragma unroll
                        for (int p = 0; p < 2; ++p) {
                            uint32_t a[4];
                            a[0] = bf16x2_sub(nib_pair_bf16(wa[p][w], i0), zA[p]);       // MMA row g,   k 2t, 2t+1
                            a[1] = bf16x2_sub(nib_pair_bf16(wb[p][w], i0), zB[p]);       // MMA row g+8, k 2t, 2t+1
                            a[2] = bf16x2_sub(nib_pair_bf16(wa[p][w], i0 + 1), zA[p]);   // MMA row g,   k 2t+8, 2t+9
                            a[3] = bf16x2_sub(nib_pair_bf16(wb[p][w], i0 + 1), zB[p]);   // MMA row g+8, k 2t+8, 2t+9
#pragma unroll
                            for (int b = 0; b < NB; ++b)
                                mma_bf16_16816(acc[p][b], a, bk[b][0], bk[b][1]);
                        }
                    }
                    // acc: [0] MMA row g / token 8b+2t, [1] row g / 8b+2t+1,
                    //      [2] MMA row g+8 / 8b+2t,     [3] row g+8 / 8b+2t+1
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        if (rp + p >= MB || rp + p >= nb_here) break;
#pragma unroll
                        for (int b = 0; b < NB; ++b) {
                            total[rp + p][b][0] = fmaf(sA[p], acc[p][b][0], total[rp + p][b][0]);
                            total[rp + p][b][1] = fmaf(sA[p], acc[p][b][1], total[rp + p][b][1]);
                            total[rp + p][b][2] = fmaf(sB[p], acc[p][b][2], total[rp + p][b][2]);
                            total[rp + p][b][3] = fmaf(sB[p], acc[p][b][3], total[rp + p][b][3]);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    consumers_done:;
    }

    // ---- the 8 consumer warps' partial sums meet in shared memory (the ring
    // is idle once every warp is here: each stage was released after use)
    __syncthreads();
    if (warp < kW16Warps) {
#pragma unroll
        for (int rb = 0; rb < MB; ++rb)
#pragma unroll
            for (int b = 0; b < NB; ++b)
                *reinterpret_cast<float4*>(red + (((warp * MB + rb) * NB + b) * 32 + lane) * 4) =
                    make_float4(total[rb][b][0], total[rb][b][1], total[rb][b][2], total[rb][b][3]);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < nb_here * NB * 32; e += kW16Threads9) {
        const int ln = e & 31;
        const int b = (e >> 5) % NB;
        const int rb = (e >> 5) / NB;
        float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int w = 0; w < kW16Warps; ++w) {
            const float4 p = *reinterpret_cast<const float4*>(red + (((w * MB + rb) * NB + b) * 32 + ln) * 4);
            v[0] += p.x; v[1] += p.y; v[2] += p.z; v[3] += p.w;
        }
        const int gg = ln >> 2, tt = ln & 3;
        const int tok0 = 8 * b + 2 * tt;
        const int r0 = (b0 + rb) * 16 + w16_perm(gg), r1 = (b0 + rb) * 16 + w16_perm(gg + 8);
        if (tok0 < M) {
            if (r0 < N) y[static_cast<size_t>(tok0) * N + r0] = __float2bfloat16_rn(v[0]);
            if (r1 < N) y[static_cast<size_t>(tok0) * N + r1] = __float2bfloat16_rn(v[2]);
        }
        if (tok0 + 1 < M) {
            if (r0 < N) y[static_cast<size_t>(tok0 + 1) * N + r0] = __float2bfloat16_rn(v[1]);
            if (r1 < N) y[static_cast<size_t>(tok0 + 1) * N + r1] = __float2bfloat16_rn(v[3]);
        }
    }
}

}  // namespace tint4
