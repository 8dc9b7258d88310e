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
// Work split: a persistent grid of one CTA per SM; CTA c owns a contiguous
// run of 16-row blocks (at most MB).  A producer warp streams, for every K
// group, the packed weights of those rows (one 16-row TMA box per block) and
// the matching x tile (all tokens) into an 8-deep shared-memory ring; consumer
// warp w takes groups w, w + 8, ... (ring slot w), reads its x fragments once
// and uses them for all of the CTA's row blocks.  The TMA keeps up to 8
// groups of weights in flight per SM whatever the warps are doing, which is
// what an HBM-bound stream needs.  The 8 partial sums of each output meet in
// shared memory at the end.
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

constexpr int kW16Stages = 8;        // = consumer warps: warp w owns ring slot w
constexpr int kW16Threads9 = (kW16Warps + 1) * 32;   // + the TMA producer warp

constexpr int kW16MaxK = 16384;   // scales / zero points of a CTA's rows stay in shared memory

template <int NB, int MB>
struct W16Layout {
    static constexpr int kWBytes = MB * 16 * 64;           // packed weights of one group
    static constexpr int kXBytes = 8 * NB * kW16Group * 2;  // x tile of one group (bf16)
    static constexpr int kStage = kWBytes + kXBytes;
    static constexpr int kRedBytes = kW16Warps * MB * NB * 32 * 16;
    static constexpr int kBarOff = kW16Stages * kStage > kRedBytes ? kW16Stages * kStage : kRedBytes;
    static constexpr int kSzOff = kBarOff + (2 * kW16Stages + 1) * 8 + 120;
    // the CTA's rows of scale (bf16) and zero point (uint8), all groups, as
    // they lie in global memory
    __host__ __device__ static constexpr int smem(int ngroups) { return kSzOff + MB * 16 * ngroups * 3 + 16; }
};

// NB = number of 8-token blocks (M <= 8 * NB); MB = 16-row blocks per CTA at most.
template <int NB, int MB>
__global__ void __launch_bounds__(kW16Threads9, 1)
w4a16_mma_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                 const __nv_bfloat16* __restrict__ wscale, const uint8_t* __restrict__ wzero,
                 __nv_bfloat16* __restrict__ y, int M, int N, int K, uint64_t wait_ns) {
    using L = W16Layout<NB, MB>;
    extern __shared__ __align__(128) uint8_t w16_smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(w16_smem + L::kBarOff);
    uint64_t* empty = full + kW16Stages;
    uint64_t* sz_full = empty + kW16Stages;        // scales + zero points landed
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sz_full + 1);
    float* red = reinterpret_cast<float*>(w16_smem);   // reused after the main loop

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2;   // MMA group id: weight row g / g + 8, token column g
    const int t = lane & 3;    // thread in group: which 32-value slice of a K group
    const int ngroups = K / kW16Group;
    const int nblk = (N + 15) / 16;
    // contiguous run of row blocks of this CTA
    const int b0 = static_cast<int>((static_cast<long long>(blockIdx.x) * nblk) / gridDim.x);
    const int b1 = static_cast<int>((static_cast<long long>(blockIdx.x + 1) * nblk) / gridDim.x);
    const int nb_here = b1 - b0;   // 1..MB (the host sizes the grid)

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
            const uint32_t bytes = nb_here * 1024 + L::kXBytes;
            int issued = 0;
            for (int G = 0; G < ngroups; ++G) {
                const int s = G % kW16Stages;
                const uint32_t ph = (G / kW16Stages) & 1;
                if (!mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, wait_ns, kDevErrTimeoutProducer))
                    break;
                uint8_t* st = w16_smem + s * L::kStage;
                mbar_arrive_expect_tx(&full[s], bytes);
                for (int rb = 0; rb < nb_here; ++rb)
                    tma_load_2d(&tmap_w, &full[s], st + rb * 1024, G * 64, (b0 + rb) * 16);
                tma_load_2d(&tmap_x, &full[s], st + L::kWBytes, G * kW16Group, 0);
                ++issued;
            }
            if (*abort_flag) {
                // let the copies in flight land before the ring is reused or freed
                uint32_t never = 0u;
                (void)mbar_wait_bounded(sz_full, 0, &never, wait_ns, 0u);
                for (int G = (issued > kW16Stages ? issued - kW16Stages : 0); G < issued; ++G)
                    (void)mbar_wait_bounded(&full[G % kW16Stages], (G / kW16Stages) & 1, &never,
                                            wait_ns, 0u);
            }
        }
    } else {
        // ------------------------------------------------ consumers
        int szok = 0;
        if (lane == 0) szok = mbar_wait_bounded(sz_full, 0, abort_flag, wait_ns, kDevErrTimeoutConsumer);
        if (__shfl_sync(0xFFFFFFFFu, szok, 0) == 0) goto consumers_done;
        for (int G = warp; G < ngroups; G += kW16Warps) {
            const int s = G % kW16Stages;
            const uint32_t ph = (G / kW16Stages) & 1;
            int ok = 0;
            if (lane == 0) ok = mbar_wait_bounded(&full[s], ph, abort_flag, wait_ns, kDevErrTimeoutConsumer);
            if (__shfl_sync(0xFFFFFFFFu, ok, 0) == 0) break;
            const uint8_t* st = w16_smem + s * L::kStage;
            // x fragments: token 8b + g, values 32t .. 32t + 31 of the group,
            // regrouped into the MMA's B layout
            uint32_t bfr[NB][8][2];
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                const uint8_t* xr = st + L::kWBytes + (8 * b + g) * (kW16Group * 2) + 64 * t;
                uint32_t xw[16];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint4 q = lds128(xr + 16 * v);
                    xw[4 * v] = q.x; xw[4 * v + 1] = q.y; xw[4 * v + 2] = q.z; xw[4 * v + 3] = q.w;
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int w = j >> 1;
                    const int i0 = 2 * (j & 1);
                    const uint32_t X0 = xw[4 * w + (i0 >> 1)];       // x[8w+i0],   x[8w+i0+1]
                    const uint32_t X2 = xw[4 * w + 2 + (i0 >> 1)];   // x[8w+i0+4], x[8w+i0+5]
                    bfr[b][j][0] = __byte_perm(X0, X2, 0x5410);      // (x[i0],   x[i0+4])
                    bfr[b][j][1] = __byte_perm(X0, X2, 0x7632);      // (x[i0+1], x[i0+5])
                }
            }
#pragma unroll
            for (int rb = 0; rb < MB; ++rb) {
                if (rb >= nb_here) break;   // CTA-uniform
                const float sA = __bfloat162float(sScale[(rb * 16 + g) * ngroups + G]);
                const float sB = __bfloat162float(sScale[(rb * 16 + g + 8) * ngroups + G]);
                // bf16x2 (128 + z, 128 + z): subtracting it from (128 + q) leaves q - z exactly
                const uint32_t zA = 0x43004300u | (0x00010001u * sZero[(rb * 16 + g) * ngroups + G]);
                const uint32_t zB = 0x43004300u | (0x00010001u * sZero[(rb * 16 + g + 8) * ngroups + G]);
                const uint4 pa = lds128(st + rb * 1024 + g * 64 + t * 16);
                const uint4 pb = lds128(st + rb * 1024 + (g + 8) * 64 + t * 16);
                const uint32_t wa[4] = {pa.x, pa.y, pa.z, pa.w};
                const uint32_t wb[4] = {pb.x, pb.y, pb.z, pb.w};
                float acc[NB][4];
#pragma unroll
                for (int b = 0; b < NB; ++b)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[b][j] = 0.0f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int w = j >> 1;          // packed word of this lane's 16 bytes
                    const int i0 = 2 * (j & 1);    // nibble pairs (i0, i0+4) and (i0+1, i0+5)
                    uint32_t a[4];
                    a[0] = bf16x2_sub(nib_pair_bf16(wa[w], i0), zA);       // row g,   k 2t, 2t+1
                    a[1] = bf16x2_sub(nib_pair_bf16(wb[w], i0), zB);       // row g+8, k 2t, 2t+1
                    a[2] = bf16x2_sub(nib_pair_bf16(wa[w], i0 + 1), zA);   // row g,   k 2t+8, 2t+9
                    a[3] = bf16x2_sub(nib_pair_bf16(wb[w], i0 + 1), zB);   // row g+8, k 2t+8, 2t+9
#pragma unroll
                    for (int b = 0; b < NB; ++b) mma_bf16_16816(acc[b], a, bfr[b][j][0], bfr[b][j][1]);
                }
                // acc: [0] row g / token 8b+2t, [1] row g / 8b+2t+1,
                //      [2] row g+8 / 8b+2t,     [3] row g+8 / 8b+2t+1
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    total[rb][b][0] = fmaf(sA, acc[b][0], total[rb][b][0]);
                    total[rb][b][1] = fmaf(sA, acc[b][1], total[rb][b][1]);
                    total[rb][b][2] = fmaf(sB, acc[b][2], total[rb][b][2]);
                    total[rb][b][3] = fmaf(sB, acc[b][3], total[rb][b][3]);
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
        const int r0 = (b0 + rb) * 16 + gg, r1 = r0 + 8;
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
