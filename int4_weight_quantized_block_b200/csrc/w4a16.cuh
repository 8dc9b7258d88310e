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
// 3 bytes of scale and zero point per 128 weights).  Per group the sum is
//   s * sum_k x_k * (q_k - z)
// with q_k - z formed exactly in bf16: 0x4300 | q is bf16(128 + q), one
// AND/OR per two nibbles from the packed bytes, and subtracting bf16(128 + z)
// leaves the small integer q - z, exact.  The products run on the warp-level
// bf16 tensor-core MMA (m16n8k16, fp32 accumulation): at M = 16 the 805 M
// multiply-adds of the 4096 x 12288 layer would take several times the HBM
// time on the fp32 CUDA cores.  Weights form the MMA's A operand straight
// from registers (16 rows x 128 K per warp step, one 16-byte load per lane
// and row), tokens the B operand (n = 8 per block).  The K order inside an
// MMA is permuted so that each lane's 32 packed nibbles map onto its own
// fragment slots; x is gathered in the same order, which leaves each dot
// product unchanged.
//
// CTA = 4 warps on the same 16 weight rows; warp w takes the K groups w,
// w + 4, ...; the 4 partial results meet in shared memory.
#pragma once

#include "ptx.cuh"

namespace tint4 {

constexpr int kW16Warps = 4;
constexpr int kW16Threads = kW16Warps * 32;
constexpr int kW16Rows = 16;       // weight rows per CTA
constexpr int kW16Group = 128;     // K values per quantization group
constexpr int kW16Unroll = 4;      // groups whose weight loads are in flight at once

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

// NB = number of 8-token blocks (M <= 8 * NB).
template <int NB>
__global__ void __launch_bounds__(kW16Threads)
w4a16_mma_kernel(const __nv_bfloat16* __restrict__ x, const uint8_t* __restrict__ wq,
                 const __nv_bfloat16* __restrict__ wscale, const uint8_t* __restrict__ wzero,
                 __nv_bfloat16* __restrict__ y, int M, int N, int K) {
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2;   // MMA group id: weight row g / g + 8, token column g
    const int t = lane & 3;    // thread in group: which 32-value slice of a K group
    const int n0 = blockIdx.x * kW16Rows;
    const int ngroups = K / kW16Group;
    const int Kh = K / 2;

    const int rowA = min(n0 + g, N - 1);       // clamped rows: loads stay in bounds,
    const int rowB = min(n0 + g + 8, N - 1);   // results of padded rows are not stored
    const uint8_t* wA = wq + static_cast<size_t>(rowA) * Kh + t * 16;
    const uint8_t* wB = wq + static_cast<size_t>(rowB) * Kh + t * 16;

    float total[NB][4];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int j = 0; j < 4; ++j) total[b][j] = 0.0f;

    for (int gb = warp; gb < ngroups; gb += kW16Warps * kW16Unroll) {
        // issue the weight loads of up to kW16Unroll groups before any math
        uint4 pa[kW16Unroll], pb[kW16Unroll];
#pragma unroll
        for (int u = 0; u < kW16Unroll; ++u) {
            const int G = gb + u * kW16Warps;
            if (G < ngroups) {
                pa[u] = __ldg(reinterpret_cast<const uint4*>(wA + G * 64));
                pb[u] = __ldg(reinterpret_cast<const uint4*>(wB + G * 64));
            } else {
                pa[u] = make_uint4(0, 0, 0, 0);
                pb[u] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int u = 0; u < kW16Unroll; ++u) {
            const int G = gb + u * kW16Warps;
            if (G >= ngroups) break;  // warp-uniform
            const float sA = __bfloat162float(wscale[static_cast<size_t>(rowA) * ngroups + G]);
            const float sB = __bfloat162float(wscale[static_cast<size_t>(rowB) * ngroups + G]);
            // bf16x2 (128 + z, 128 + z): subtracting it from (128 + q) leaves q - z exactly
            const uint32_t zA = 0x43004300u | (0x00010001u * wzero[static_cast<size_t>(rowA) * ngroups + G]);
            const uint32_t zB = 0x43004300u | (0x00010001u * wzero[static_cast<size_t>(rowB) * ngroups + G]);
            const uint32_t wa[4] = {pa[u].x, pa[u].y, pa[u].z, pa[u].w};
            const uint32_t wb[4] = {pb[u].x, pb[u].y, pb[u].z, pb[u].w};
            // dequantized A fragments (q - z in bf16), shared by every token block
            uint32_t afr[8][4];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int w = j >> 1;          // packed word of this lane's 16 bytes
                const int i0 = 2 * (j & 1);    // nibble pairs (i0, i0+4) and (i0+1, i0+5)
                afr[j][0] = bf16x2_sub(nib_pair_bf16(wa[w], i0), zA);      // row g,   k 2t, 2t+1
                afr[j][1] = bf16x2_sub(nib_pair_bf16(wb[w], i0), zB);      // row g+8, k 2t, 2t+1
                afr[j][2] = bf16x2_sub(nib_pair_bf16(wa[w], i0 + 1), zA);  // row g,   k 2t+8, 2t+9
                afr[j][3] = bf16x2_sub(nib_pair_bf16(wb[w], i0 + 1), zB);  // row g+8, k 2t+8, 2t+9
            }
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                // x[token 8b + g][G*128 + 32t .. +31]
                const int tok = 8 * b + g;
                uint32_t xw[16];
                if (tok < M) {
                    const uint4* xp = reinterpret_cast<const uint4*>(
                        x + static_cast<size_t>(tok) * K + G * kW16Group + 32 * t);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const uint4 q = __ldg(xp + v);
                        xw[4 * v] = q.x; xw[4 * v + 1] = q.y; xw[4 * v + 2] = q.z; xw[4 * v + 3] = q.w;
                    }
                } else {
#pragma unroll
                    for (int v = 0; v < 16; ++v) xw[v] = 0u;
                }
                float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int w = j >> 1;
                    const int i0 = 2 * (j & 1);
                    // x values 8w + (0..7) of this lane's slice, paired like the nibbles
                    const uint32_t X0 = xw[4 * w + (i0 >> 1)];       // x[8w+i0],   x[8w+i0+1]
                    const uint32_t X2 = xw[4 * w + 2 + (i0 >> 1)];   // x[8w+i0+4], x[8w+i0+5]
                    const uint32_t b0 = __byte_perm(X0, X2, 0x5410);  // (x[i0],   x[i0+4])
                    const uint32_t b1 = __byte_perm(X0, X2, 0x7632);  // (x[i0+1], x[i0+5])
                    mma_bf16_16816(acc, afr[j], b0, b1);
                }
                // acc: [0] row g / token 8b+2t, [1] row g / 8b+2t+1,
                //      [2] row g+8 / 8b+2t,     [3] row g+8 / 8b+2t+1
                total[b][0] = fmaf(sA, acc[0], total[b][0]);
                total[b][1] = fmaf(sA, acc[1], total[b][1]);
                total[b][2] = fmaf(sB, acc[2], total[b][2]);
                total[b][3] = fmaf(sB, acc[3], total[b][3]);
            }
        }
    }

    // reduce the 4 warps' partial sums, then store
    __shared__ float red[kW16Warps][NB][32][4];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int j = 0; j < 4; ++j) red[warp][b][lane][j] = total[b][j];
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            float v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                v[j] = red[0][b][lane][j] + red[1][b][lane][j] + red[2][b][lane][j] +
                       red[3][b][lane][j];
            const int tok0 = 8 * b + 2 * t;
            const int r0 = n0 + g, r1 = n0 + g + 8;
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
}

}  // namespace tint4
