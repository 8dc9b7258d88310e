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
// at most 16 tokens of one launch.  Per group the sum is written
//   s * (sum_k x_k * (128 + q_k)  -  (128 + z) * sum_k x_k)
// which is the same number: 128 + q_k is exact in bf16 (OR a nibble into the
// mantissa of bf16 128), so the dequantization is one bit operation per two
// weights plus a shift, and the zero point leaves the inner loop.  The sums
// of x per group come from the same MMA with an all-ones weight tile.  The products run on the
// warp-level bf16 MMA (m16n8k16, fp32 accumulation): at M = 16 the 805 M
// multiply-adds of the 4096 x 12288 layer would take several times the HBM
// time on the fp32 CUDA cores.  Weights are the MMA's A operand straight from
// registers (16 rows x 16 K per MMA, one 16-byte load per lane and row and
// group), tokens the B operand (n = 8 per token block).  The K order inside
// an MMA is permuted so that each lane's 32 packed nibbles of a group map onto
// its own fragment slots; x is gathered in the same order, which leaves each
// dot product unchanged.
//
// Work split: one CTA per SM owns a contiguous run of 16-row blocks (at most
// kW16MB).  A unit of work is one K group pair x one block pair: a 32-row x
// 128-byte TMA box (4 KB; smaller boxes leave the copy engine, not DRAM, as
// the limit).  The run's units, in pair-major order, are split into equal
// contiguous ranges, one per warp, so a warp mostly stays on one group pair.  Every warp is
// its own producer: its lane 0 keeps the warp's next units in flight in a
// private ring, so no warp waits for another until the end.  A warp keeps the
// x fragments of its current group pair in registers for all blocks of the
// run, and its running sums in registers; the partial sums of the warps meet
// in shared memory once at the end.  Scales and zero points of the run's rows
// are copied to shared memory once, by two bulk copies issued ahead of the
// weight boxes.
//
// The weight boxes use the 128-byte swizzle (16-byte chunk c of smem row r at
// c ^ (r & 7)).  The two rows an 8-lane phase reads would share banks, so MMA
// row m holds weight row pi(m) = 4 (m & 1) + (m >> 1) (m < 8; +8 above), which
// puts them 4 rows apart and onto disjoint chunk sets: conflict-free.
//
// Launched with programmatic dependent launch: the CTA sets up its barriers
// while the previous kernel of the stream drains, and waits for it before
// the first read of any input.
#pragma once

#include "ptx.cuh"

namespace tint4 {

constexpr int kW16Group = 128;      // K values per quantization group
constexpr int kW16Box = 32 * 128;   // one unit: 2 row blocks x 2 groups of packed bytes
constexpr int kW16Ring = 128 * 1024;  // all warps' rings
constexpr int kW16MB = 6;           // 16-row blocks per CTA at most
constexpr int kW16Rows = kW16MB * 16;
constexpr int kW16MaxK = 16384;
constexpr int kW16MaxM = 16;        // tokens per launch (the host splits larger batches)

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               const uint32_t b0, const uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Constants of the nibble unpack, passed as a kernel parameter: the compiler
// then takes them as constant-bank operands instead of rebuilding them in
// registers around every use (two bit operations per pair instead of one).
struct W16Consts {
    uint32_t mask;    // 0x000F000F: the low nibble of each 16-bit half
    uint32_t base;    // 0x43004300: bf16x2 (128, 128)
};

__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t m, uint32_t o) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(m), "r"(o));   // (a & m) | o
    return d;
}

// One packed word (nibbles q0..q7, q_i at bits 4i) to the four bf16x2 pairs
// (128 + q0, 128 + q4), (128 + q1, 128 + q5), (128 + q2, 128 + q6),
// (128 + q3, 128 + q7), all exact: a nibble OR-ed into the low mantissa bits
// of bf16 128 (0x4300) adds its value (the 7-bit mantissa has room for 4 bits
// only at the bottom, so the upper nibbles are shifted down first).  Seven
// ALU instructions per 8 weights: this is what bounds the kernel's math.
__device__ __forceinline__ void unpack_word(uint32_t w, const W16Consts& c, uint32_t (&p)[4]) {
    p[0] = and_or(w, c.mask, c.base);
    p[1] = and_or(w >> 4, c.mask, c.base);
    p[2] = and_or(w >> 8, c.mask, c.base);
    p[3] = and_or(w >> 12, c.mask, c.base);
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

// MMA row m (0..15) of a block holds weight row w16_perm(m) of the block
__host__ __device__ constexpr int w16_perm(int m) {
    return (m & 8) | ((m & 1) << 2) | ((m >> 1) & 3);
}

// NB 8-token blocks with WARPS warps: the running sums (kW16MB blocks x NB x 4
// floats) and the x fragments of a group pair (NB x 32 words) stay in
// registers, so NB = 2 runs 8 warps (255 registers each), NB = 1 16 warps.
// The ring takes what shared memory the scales and zero points leave: every
// warp's units are in flight at once for the decode shapes.
template <int NB>
struct W16Cfg {
    static constexpr int WARPS = NB == 1 ? 16 : 8;
    static constexpr int THREADS = WARPS * 32;
    static constexpr int kMaxSlots = 2;
    static constexpr int kBarBytes = WARPS * kMaxSlots * 8 + 16;   // + scale/zero barrier, abort flag
    static constexpr int kRedBytes = WARPS * kW16MB * NB * 32 * 16;   // reuses the ring
    static constexpr int kSmemMax = 227 * 1024;
    // boxes in flight per warp for a K of ngroups groups
    __host__ __device__ static constexpr int slots(int ngroups) {
        return (kSmemMax - 1024 - kBarBytes - ngroups * kW16Rows * 3) / (WARPS * kW16Box) < kMaxSlots
                   ? (kSmemMax - 1024 - kBarBytes - ngroups * kW16Rows * 3) / (WARPS * kW16Box)
                   : kMaxSlots;
    }
    __host__ __device__ static constexpr int ring_bytes(int ngroups) {
        return slots(ngroups) * WARPS * kW16Box;
    }
    // ring | barriers | scales (bf16) and zero points (uint8) of up to kW16Rows rows, as in global memory
    __host__ __device__ static constexpr int smem(int ngroups) {
        return ring_bytes(ngroups) + kBarBytes + ngroups * kW16Rows * 3 + 1024;   // + 1024: alignment
    }
    static_assert(kRedBytes <= 2 * WARPS * kW16Box, "the reduction reuses the ring");
    static_assert((kSmemMax - 1024 - kBarBytes - (kW16MaxK / kW16Group) * kW16Rows * 3) /
                          (WARPS * kW16Box) >= 2,
                  "double buffering at least, at the largest K");
};

// NB = number of 8-token blocks (M <= 8 * NB <= 16).
template <int NB>
__global__ void __launch_bounds__(W16Cfg<NB>::THREADS, 1)
w4a16_mma_kernel(const __grid_constant__ CUtensorMap tmap_w, const __nv_bfloat16* __restrict__ x,
                 const __nv_bfloat16* __restrict__ wscale, const uint8_t* __restrict__ wzero,
                 __nv_bfloat16* __restrict__ y, int M, int N, int K, const W16Consts kc,
                 int early_weights, uint64_t wait_ns) {
    using C = W16Cfg<NB>;
    constexpr int WARPS = C::WARPS;
    extern __shared__ uint8_t w16_smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(w16_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int ngroups = K / kW16Group;
    const int SLOTS = C::slots(ngroups);
    const int ring_bytes = SLOTS * WARPS * kW16Box;
    uint64_t* full_all = reinterpret_cast<uint64_t*>(sm + ring_bytes);
    uint64_t* sz_full = full_all + WARPS * C::kMaxSlots;   // scales + zero points landed
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sz_full + 1);
    float* red = reinterpret_cast<float*>(sm);   // reused after the main loop

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2;   // MMA group id: MMA rows g / g + 8, token column g
    const int t = lane & 3;    // which 32-value slice of a group
    const int npairs = (ngroups + 1) / 2;
    const int nblk = N / 16;
    int b0, b1;   // this CTA's run of blocks (32-bit arithmetic: 64-bit division is a long
    even_split(nblk, gridDim.x, blockIdx.x, b0, b1);   // software routine on the prologue's path)
    const int nb = b1 - b0;             // 1..kW16MB (the host sizes the grid)
    const int nbp = (nb + 1) / 2;       // block pairs (an odd run's last box reads 16 rows it skips)
    const int rA = w16_perm(g), rB = w16_perm(g + 8);   // weight rows of MMA rows g, g + 8
    const int swz = rA & 7;                              // = rB & 7

    // the run's rows of scale (bf16 bits) and zero point, [row][group] as in global memory
    const uint16_t* sScale = reinterpret_cast<const uint16_t*>(sm + ring_bytes + C::kBarBytes);
    const uint8_t* sZero = sm + ring_bytes + C::kBarBytes + ngroups * kW16Rows * 2;

    // the run's units in pair-major order, u = P * nbp + bp; this warp takes
    // the contiguous, balanced range [u0, u1)
    const int ntot = npairs * nbp;
    int u0, u1;
    even_split(ntot, WARPS, warp, u0, u1);
    const int nunits = u1 - u0;
    uint64_t* full = full_all + warp * SLOTS;
    uint8_t* ring = sm + warp * SLOTS * kW16Box;

    if (lane == 0) {
        for (int i = 0; i < SLOTS; ++i) mbar_init(&full[i], 1);
        if (warp == 0) {
            *abort_flag = 0u;
            mbar_init(sz_full, 1);
        }
        fence_mbarrier_init();
        prefetch_tensormap(&tmap_w);
    }
    __syncthreads();

    int issued = 0;
    bool nunits_ok = true;
    auto issue = [&](int i) {
        const int slot = i % SLOTS;
        const int P = (u0 + i) / nbp;
        const int bp = (u0 + i) % nbp;
        mbar_arrive_expect_tx(&full[slot], kW16Box);
        tma_load_2d(&tmap_w, &full[slot], ring + slot * kW16Box, P * 128, (b0 + 2 * bp) * 16);
    };
    // The run's scales and zero points (two contiguous, 16-byte aligned
    // ranges) go out first, as two bulk copies: behind tens of MB of weight
    // boxes they would hold up every warp's first unit.  Then the weight
    // boxes.  All of it may start before the previous kernel of the stream
    // has finished only when the caller said the weights are not written by
    // it (tint4_set_decode_weight_prefetch); x is read after the wait.
    auto issue_weights = [&]() {
        if (threadIdx.x == 0) {
            const uint32_t sbytes = nb * 16 * ngroups * 2, zbytes = nb * 16 * ngroups;
            const size_t base = static_cast<size_t>(b0) * 16 * ngroups;
            mbar_arrive_expect_tx(sz_full, sbytes + zbytes);
            bulk_load_1d(sm + ring_bytes + C::kBarBytes, wscale + base, sbytes, sz_full);
            bulk_load_1d(sm + ring_bytes + C::kBarBytes + ngroups * kW16Rows * 2, wzero + base, zbytes, sz_full);
        }
        __syncwarp();
        // one box per warp now, the rest once the scales have landed: every
        // warp's first box then reaches the front of the memory queues
        if (lane == 0 && issued < nunits) issue(issued++);
    };
    if (early_weights) issue_weights();
    grid_dependency_wait();
    grid_launch_dependents();
    if (!early_weights) issue_weights();
    {
        if (!warp_wait(sz_full, 0, abort_flag, wait_ns, kDevErrTimeoutConsumer)) nunits_ok = false;
        if (lane == 0)
            for (; issued < SLOTS && issued < nunits; ++issued) issue(issued);
    }

    float total[kW16MB][NB][4];
#pragma unroll
    for (int j = 0; j < kW16MB; ++j)
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int q = 0; q < 4; ++q) total[j][b][q] = 0.0f;

    int consumed = 0, cslot = 0;
    uint32_t cphase = 0u;
    bool aborted = !nunits_ok;
    const int P0 = u0 / nbp, P1 = nunits > 0 ? (u1 - 1) / nbp : P0 - 1;
    for (int P = P0; P <= P1 && !aborted; ++P) {
        const int bp_lo = P == P0 ? u0 % nbp : 0;                 // this warp's block pairs of pair P
        const int bp_hi = P == P1 ? (u1 - 1) % nbp + 1 : nbp;
        const bool two = 2 * P + 1 < ngroups;   // an odd group count's last pair has one
        // (a missing second group gets x = 0: its sums vanish, whatever its box holds)
        // x fragments of groups 2P, 2P + 1: token 8b + g, values 32t .. 32t + 31,
        // in the MMA's B layout (zeros for tokens >= M and for a missing group)
        uint32_t bfr[2][NB][8][2];
#pragma unroll
        for (int gi = 0; gi < 2; ++gi)
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                const int tok = 8 * b + g;
                if (tok < M && (gi == 0 || two)) {
                    const uint4* xr = reinterpret_cast<const uint4*>(
                        x + static_cast<size_t>(tok) * K + (2 * P + gi) * kW16Group + 32 * t);
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const uint4 q = __ldcg(xr + w);
                        x_frag(q, bfr[gi][b][2 * w], bfr[gi][b][2 * w + 1]);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k) bfr[gi][b][k][0] = bfr[gi][b][k][1] = 0u;
                }
            }
        // per-group sums of x (tokens 8b + 2t, 8b + 2t + 1 in [0], [1]: the MMA's
        // accumulator layout) from an all-ones weight tile
        float xs[2][NB][4];
        {
            const uint32_t ones[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};
#pragma unroll
            for (int gi = 0; gi < 2; ++gi)
#pragma unroll
                for (int b = 0; b < NB; ++b) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) xs[gi][b][q] = 0.0f;
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_bf16_16816(xs[gi][b], ones, bfr[gi][b][k][0], bfr[gi][b][k][1]);
                }
        }
#pragma unroll
        for (int bp = 0; bp < kW16MB / 2; ++bp) {
            if (bp >= bp_hi) break;   // warp-uniform
            if (bp < bp_lo) continue;
            const int slot = cslot;
            if (!warp_wait(&full[slot], cphase, abort_flag, wait_ns, kDevErrTimeoutConsumer)) {
                aborted = true;
                break;
            }
            const uint8_t* box = ring + slot * kW16Box;
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
                const int j = 2 * bp + hb;         // block of the run
                if (j >= nb) break;                // CTA-uniform
                const uint8_t* bbox = box + hb * 16 * 128;
#pragma unroll
                for (int gi = 0; gi < 2; ++gi) {
                    // this lane's 16-byte chunk of group 2P + gi in rows rA / rB (swizzled)
                    const int coff = ((4 * gi + t) ^ swz) << 4;
                    const uint4 pa = *reinterpret_cast<const uint4*>(bbox + rA * 128 + coff);
                    const uint4 pb = *reinterpret_cast<const uint4*>(bbox + rB * 128 + coff);
                    const int G = min(2 * P + gi, ngroups - 1);   // a missing group has x = 0
                    const int r = j * 16;
                    const float sA = __uint_as_float(static_cast<uint32_t>(sScale[(r + rA) * ngroups + G]) << 16);
                    const float sB = __uint_as_float(static_cast<uint32_t>(sScale[(r + rB) * ngroups + G]) << 16);
                    // -(128 + z) exactly: (2^23 - 128) - (2^23 + z)
                    const float cA = 8388480.0f - __uint_as_float(0x4B000000u | sZero[(r + rA) * ngroups + G]);
                    const float cB = 8388480.0f - __uint_as_float(0x4B000000u | sZero[(r + rB) * ngroups + G]);
                    const uint32_t wa[4] = {pa.x, pa.y, pa.z, pa.w};
                    const uint32_t wb[4] = {pb.x, pb.y, pb.z, pb.w};
                    float acc[NB][4];
#pragma unroll
                    for (int b = 0; b < NB; ++b)
#pragma unroll
                        for (int q = 0; q < 4; ++q) acc[b][q] = 0.0f;
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        // packed word w of rows rA / rB: k steps 2w (pairs (0,4), (1,5))
                        // and 2w + 1 (pairs (2,6), (3,7))
                        uint32_t da[4], db[4];
                        unpack_word(wa[w], kc, da);
                        unpack_word(wb[w], kc, db);
                        const uint32_t a0[4] = {da[0], db[0], da[1], db[1]};   // rows g, g+8 x k 2t.., 2t+8..
                        const uint32_t a1[4] = {da[2], db[2], da[3], db[3]};
#pragma unroll
                        for (int b = 0; b < NB; ++b) {
                            mma_bf16_16816(acc[b], a0, bfr[gi][b][2 * w][0], bfr[gi][b][2 * w][1]);
                            mma_bf16_16816(acc[b], a1, bfr[gi][b][2 * w + 1][0], bfr[gi][b][2 * w + 1][1]);
                        }
                    }
                    // acc: [0] MMA row g / token 8b+2t, [1] row g / 8b+2t+1,
                    //      [2] MMA row g+8 / 8b+2t,     [3] row g+8 / 8b+2t+1
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        total[j][b][0] = fmaf(sA, fmaf(cA, xs[gi][b][0], acc[b][0]), total[j][b][0]);
                        total[j][b][1] = fmaf(sA, fmaf(cA, xs[gi][b][1], acc[b][1]), total[j][b][1]);
                        total[j][b][2] = fmaf(sB, fmaf(cB, xs[gi][b][0], acc[b][2]), total[j][b][2]);
                        total[j][b][3] = fmaf(sB, fmaf(cB, xs[gi][b][1], acc[b][3]), total[j][b][3]);
                    }
                }
            }
            ++consumed;
            if (++cslot == SLOTS) { cslot = 0; cphase ^= 1u; }
            // the slot is free again: refill it with this warp's unit SLOTS ahead
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
        if (warp == 0) (void)mbar_wait_bounded(sz_full, 0, &never, wait_ns, 0u);
        for (int i = consumed; i < issued; ++i)
            (void)mbar_wait_bounded(&full[i % SLOTS], (i / SLOTS) & 1, &never, wait_ns, 0u);
    }

    // ---- the warps' partial sums meet in shared memory
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kW16MB; ++j) {
        if (j >= nb) break;
#pragma unroll
        for (int b = 0; b < NB; ++b)
            *reinterpret_cast<float4*>(red + (((warp * kW16MB + j) * NB + b) * 32 + lane) * 4) =
                make_float4(total[j][b][0], total[j][b][1], total[j][b][2], total[j][b][3]);
    }
    __syncthreads();
    if (*abort_flag) return;   // the device error word says why; y is left as it was
    for (int e = threadIdx.x; e < nb * NB * 32; e += C::THREADS) {
        const int ln = e & 31;
        const int b = (e >> 5) % NB;
        const int j = (e >> 5) / NB;
        float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int w = 0; w < WARPS; ++w) {
            const float4 p = *reinterpret_cast<const float4*>(red + (((w * kW16MB + j) * NB + b) * 32 + ln) * 4);
            v[0] += p.x; v[1] += p.y; v[2] += p.z; v[3] += p.w;
        }
        const int gg = ln >> 2, tt = ln & 3;
        const int tok0 = 8 * b + 2 * tt;
        const int r0 = (b0 + j) * 16 + w16_perm(gg), r1 = (b0 + j) * 16 + w16_perm(gg + 8);
        if (tok0 < M) {
            y[static_cast<size_t>(tok0) * N + r0] = __float2bfloat16_rn(v[0]);
            y[static_cast<size_t>(tok0) * N + r1] = __float2bfloat16_rn(v[2]);
        }
        if (tok0 + 1 < M) {
            y[static_cast<size_t>(tok0 + 1) * N + r0] = __float2bfloat16_rn(v[1]);
            y[static_cast<size_t>(tok0 + 1) * N + r1] = __float2bfloat16_rn(v[3]);
        }
    }
}

}  // namespace tint4
