// tint4_abi.cu -- the C ABI of include/tint4.h: argument checks, tensor maps,
// launch configuration.  Every operation runs in the kernels of quantize.cuh,
// gemm_tmem.cuh, w4a8_small.cuh and w4a16.cuh; nothing here touches tensor
// data.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <mutex>

#include "../../include/tint4.h"
#include "gemm_tmem.cuh"
#include "gemm_tmem_gw.cuh"
#include "gemm_wide.cuh"
#include "pack_groupwise.cuh"
#include "ptx.cuh"
#include "quantize.cuh"
#include "w4a16.cuh"
#include "w4a16_gemm.cuh"
#include "w4a8_small.cuh"

namespace {

using namespace tint4;

constexpr int kAbiVersion = 1;
constexpr int kMaxDevices = 64;
constexpr int kMaxTokens = 65535 * 128;   // M limit of the GEMM entry points
constexpr int kW16SmallMaxM = 32;         // W4A16: up to here the streaming kernel, above the GEMM

std::atomic<uint64_t> g_wait_limit_ns{4000000000ull};
std::atomic<int> g_decode_prefetch{0};   // tint4_set_decode_weight_prefetch

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ------------------------------------------------------------------ device check

tint4_status check_device(int* dev_out = nullptr) {
    static std::atomic<int> cache[kMaxDevices];  // 0 unknown, 1 ok, 2 unsupported
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return TINT4_ERR_NO_DEVICE;
    }
    if (dev_out) *dev_out = dev;
    if (dev < 0 || dev >= kMaxDevices) return TINT4_ERR_NO_DEVICE;
    int c = cache[dev].load(std::memory_order_relaxed);
    if (c == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
            cudaGetLastError();
            return TINT4_ERR_NO_DEVICE;
        }
        c = (major == 10 && minor == 0) ? 1 : 2;
        cache[dev].store(c, std::memory_order_relaxed);
    }
    return c == 1 ? TINT4_OK : TINT4_ERR_NO_DEVICE;
}

tint4_status last_launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TINT4_OK : TINT4_ERR_CUDA;
}

// ------------------------------------------------------------------ tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// 2-D tensor [outer, inner] of `dtype` with row pitch `pitch` bytes; box
// [box_outer, box_inner]; out-of-range elements read as zero and are not
// written by stores.
bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                 uint64_t outer, uint64_t pitch, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle swizzle) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {pitch};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_map_u8(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                 uint64_t pitch, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle swizzle) {
    return make_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, inner, outer, pitch, box_inner,
                       box_outer, swizzle);
}

// ------------------------------------------------------------------ shape rules

tint4_status check_mnk(int M, int N, int K) {
    if (M < 0 || N < 0 || K < 0) return TINT4_ERR_INVALID_ARG;
    if (N < 16 || N % 16 != 0) return TINT4_ERR_UNSUPPORTED_SHAPE;
    if (K < 32 || K % 32 != 0 || K > 65536) return TINT4_ERR_UNSUPPORTED_SHAPE;
    if (M > kMaxTokens) return TINT4_ERR_UNSUPPORTED_SHAPE;
    return TINT4_OK;
}

bool valid_group(int g) { return g == 0 || g == 16 || g == 64 || g == 256; }

// ------------------------------------------------------------------ rotate + quantize

// Q = 127 or 7; PACKED: int4 codes two per byte, else one code per int8.
// One row per pass of a CTA (rq_team_rows): CPL chunks of 8 values per lane
// and as many warps as cover K.
int num_sms(int dev);

struct RqShape {
    int cpl, warps;
};

RqShape rq_shape(int K) {
    const int nc = K / 8;
    const int cpl = nc <= 32 ? 1 : (nc <= 64 ? 2 : 4);
    return RqShape{cpl, (nc + 32 * cpl - 1) / (32 * cpl)};
}

// persistent grid: as many CTAs as fit on the GPU at once (per block size,
// looked up once per device), at most one per row
template <typename InT, int G, int Q, bool PACKED, bool EVOD, int CPL, bool S16 = false>
void launch_rq_persistent(const InT* in, int rows, int K, void* codes, void* scales, int threads,
                          cudaStream_t st) {
    auto kern = rotate_quantize_rows_kernel<InT, G, Q, PACKED, EVOD, CPL, S16>;
    int dev = 0;
    cudaGetDevice(&dev);
    static std::atomic<int> per_sm[kMaxDevices][kQuantMaxWarps + 1];
    const int nw = threads / 32;
    int occ = per_sm[dev][nw].load(std::memory_order_relaxed);
    if (occ == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, 0) != cudaSuccess ||
            occ < 1) {
            cudaGetLastError();
            occ = 1;
        }
        per_sm[dev][nw].store(occ, std::memory_order_relaxed);
    }
    const int grid = std::min(rows, occ * num_sms(dev));
    kern<<<grid, threads, 0, st>>>(in, rows, K, codes, scales);
}

template <typename InT, int G, int Q, bool PACKED, bool EVOD = false, bool S16 = false>
void launch_rq_ch(const InT* in, int rows, int K, void* codes, void* scales, cudaStream_t st) {
    const RqShape sh = rq_shape(K);
    const int threads = sh.warps * 32;
    if (sh.cpl == 1)
        launch_rq_persistent<InT, G, Q, PACKED, EVOD, 1, S16>(in, rows, K, codes, scales, threads, st);
    else if (sh.cpl == 2)
        launch_rq_persistent<InT, G, Q, PACKED, EVOD, 2, S16>(in, rows, K, codes, scales, threads, st);
    else
        launch_rq_persistent<InT, G, Q, PACKED, EVOD, 4, S16>(in, rows, K, codes, scales, threads, st);
}

template <typename InT, int Q, bool PACKED, bool EVOD = false, bool S16 = false>
void launch_rq_g(const InT* in, int rows, int K, int g, void* codes, void* scales,
                 cudaStream_t st) {
    switch (g) {
        case 0: launch_rq_ch<InT, 0, Q, PACKED, EVOD, S16>(in, rows, K, codes, scales, st); break;
        case 16: launch_rq_ch<InT, 16, Q, PACKED, EVOD, S16>(in, rows, K, codes, scales, st); break;
        case 64: launch_rq_ch<InT, 64, Q, PACKED, EVOD, S16>(in, rows, K, codes, scales, st); break;
        default: launch_rq_ch<InT, 256, Q, PACKED, EVOD, S16>(in, rows, K, codes, scales, st); break;
    }
}

tint4_status check_rq_shape(int rows, int K, int g) {
    if (rows < 0 || K < 0) return TINT4_ERR_INVALID_ARG;
    if (!valid_group(g)) return TINT4_ERR_INVALID_ARG;
    if (K < 32 || K % 32 != 0 || K > kQuantMaxK) return TINT4_ERR_UNSUPPORTED_SHAPE;
    if (g != 0 && K % g != 0) return TINT4_ERR_UNSUPPORTED_SHAPE;
    return TINT4_OK;
}

// ------------------------------------------------------------------ GEMM

int num_sms(int dev) {
    static std::atomic<int> cache[kMaxDevices];
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            v = 148;
        }
        cache[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

cudaLaunchAttribute pdl_attr() {
    cudaLaunchAttribute a;
    a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a.val.programmaticStreamSerializationAllowed = 1;
    return a;
}

// Int8 activation codes x packed int4 weights: the kernel with decoupled
// weight and activation rings (gemm_wide.cuh), 256-token tiles.
template <bool OUT_I32, bool EVOD>
tint4_status launch_gemm_wide(const void* a, const float* st, TmGroups& grp,
                              const uint8_t* const* w, int M, int K, cudaStream_t stream,
                              bool pdl) {
    auto kern = w4a8_wide_gemm_kernel<OUT_I32, EVOD>;
    CUtensorMap ta;
    bool ok = make_map_u8(&ta, a, K, M, K, kTmBK, kWdBN, CU_TENSOR_MAP_SWIZZLE_128B);
    const int m_tiles = (M + kWdBN - 1) / kWdBN;
    int tiles = 0;
    for (int g = 0; g < grp.count; ++g) {
        ok = ok && make_map_u8(&grp.w[g], w[g], K / 2, grp.N[g], K / 2, kTmBK / 2, kTmBM,
                               CU_TENSOR_MAP_SWIZZLE_64B);
        tiles += m_tiles * ((grp.N[g] + kTmBM - 1) / kTmBM);
        grp.tile_end[g] = tiles;
    }
    if (!ok) return TINT4_ERR_CUDA;
    int dev = 0;
    cudaGetDevice(&dev);
    static std::atomic<bool> attr_done[kMaxDevices];
    if (!attr_done[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kWdSmem) !=
            cudaSuccess) {
            cudaGetLastError();
            return TINT4_ERR_CUDA;
        }
        attr_done[dev].store(true, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(std::min(tiles, num_sms(dev)), 1, 1);
    cfg.blockDim = dim3(kWdThreads, 1, 1);
    cfg.dynamicSmemBytes = kWdSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    if (pdl) {
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    const uint64_t wait_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
    if (cudaLaunchKernelEx(&cfg, kern, ta, grp, st, M, K, wait_ns) != cudaSuccess) {
        cudaGetLastError();
        return TINT4_ERR_CUDA;
    }
    return TINT4_OK;
}

// The shared-stage kernel (gemm_tmem.cuh): packed int4 activation codes
// widened in shared memory (A_INT4), or int8 weights (W8).  `grp` holds 1 to
// kTmMaxGroups weight matrices sharing the activation codes (the tensor maps
// and the tile list are filled in here).
template <bool OUT_I32, bool A_INT4, bool W8, bool EVOD, bool S16>
tint4_status launch_gemm_shared_stage(const void* a, const float* st, TmGroups& grp,
                                      const uint8_t* const* w, int M, int K,
                                      cudaStream_t stream, bool pdl) {
    auto kern = w4a8_tmem_gemm_kernel<OUT_I32, A_INT4, W8, EVOD, S16>;
    using C = TmCfg<A_INT4, W8>;
    constexpr int smem_bytes = C::SMEM;
    CUtensorMap ta;
    bool ok = A_INT4 ? make_map_u8(&ta, a, K / 2, M, K / 2, kTmBK / 2, C::BN, CU_TENSOR_MAP_SWIZZLE_NONE)
                     : make_map_u8(&ta, a, K, M, K, kTmBK, C::BN, CU_TENSOR_MAP_SWIZZLE_128B);
    const int m_tiles = (M + C::BN - 1) / C::BN;
    int tiles = 0;
    for (int g = 0; g < grp.count; ++g) {
        ok = ok && (W8 ? make_map_u8(&grp.w[g], w[g], K, grp.N[g], K, kTmBK, kTmBM,
                                     CU_TENSOR_MAP_SWIZZLE_128B)
                       : make_map_u8(&grp.w[g], w[g], K / 2, grp.N[g], K / 2, kTmBK / 2, kTmBM,
                                     CU_TENSOR_MAP_SWIZZLE_64B));
        tiles += m_tiles * ((grp.N[g] + kTmBM - 1) / kTmBM);
        grp.tile_end[g] = tiles;
    }
    if (!ok) return TINT4_ERR_CUDA;
    int dev = 0;
    cudaGetDevice(&dev);
    static std::atomic<bool> attr_done[kMaxDevices];
    if (!attr_done[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem_bytes) != cudaSuccess) {
            cudaGetLastError();
            return TINT4_ERR_CUDA;
        }
        attr_done[dev].store(true, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(std::min(tiles, num_sms(dev)), 1, 1);
    cfg.blockDim = dim3(kTmThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    if (pdl) {
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    const uint64_t wait_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
    if (cudaLaunchKernelEx(&cfg, kern, ta, grp, st, M, K, wait_ns) != cudaSuccess) {
        cudaGetLastError();
        return TINT4_ERR_CUDA;
    }
    return TINT4_OK;
}

// The tensor-core GEMM of every large-M entry point: int8 activation codes x
// packed int4 weights run the kernel with decoupled rings (gemm_wide.cuh),
// the other forms the shared-stage one.
template <bool OUT_I32, bool A_INT4, bool W8 = false, bool EVOD = false, bool S16 = false>
tint4_status launch_gemm_tmem(const void* a, const float* st, TmGroups& grp,
                              const uint8_t* const* w, int M, int K, cudaStream_t stream,
                              bool pdl) {
    if constexpr (!A_INT4 && !W8)
        return launch_gemm_wide<OUT_I32, EVOD>(a, st, grp, w, M, K, stream, pdl);
    else
        return launch_gemm_shared_stage<OUT_I32, A_INT4, W8, EVOD, S16>(a, st, grp, w, M, K, stream,
                                                                          pdl);
}


// Small M (<= kS8MaxM tokens): the warp-MMA kernel that streams the packed
// weights once (w4a8_small.cuh).
template <int NB, bool A_INT4, bool OUT_I32>
tint4_status launch_gemm_small(const void* a, const uint8_t* w, const float* st, const float* sr,
                               const __nv_bfloat16* bias, void* out, int M, int N, int K,
                               cudaStream_t stream, bool pdl) {
    auto kern = w4a8_small_kernel<NB, A_INT4, OUT_I32>;
    CUtensorMap tw;
    if (!make_map_u8(&tw, w, K / 2, N, K / 2, 128, 32, CU_TENSOR_MAP_SWIZZLE_128B))
        return TINT4_ERR_CUDA;
    int dev = 0;
    cudaGetDevice(&dev);
    static std::atomic<bool> attr_done[kMaxDevices];
    if (!attr_done[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 S8Cfg<NB>::SMEM) != cudaSuccess) {
            cudaGetLastError();
            return TINT4_ERR_CUDA;
        }
        attr_done[dev].store(true, std::memory_order_release);
    }
    const int nblk = N / 16;
    // one CTA per SM unless that would give a CTA more than kS8MB blocks
    const int sms = num_sms(dev);
    const int grid = nblk <= kS8MB * sms ? std::min(sms, nblk) : (nblk + kS8MB - 1) / kS8MB;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(S8Cfg<NB>::THREADS, 1, 1);
    cfg.dynamicSmemBytes = S8Cfg<NB>::SMEM;
    cfg.stream = stream;
    // always programmatic: the kernel waits for the previous grid before it
    // reads anything that grid may have written
    (void)pdl;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tw, static_cast<const uint8_t*>(a), st, sr, bias, out, M,
                           N, K, 0xF0F0F0F0u, g_decode_prefetch.load(std::memory_order_relaxed),
                           g_wait_limit_ns.load(std::memory_order_relaxed),
                           static_cast<const uint8_t*>(nullptr)) != cudaSuccess) {
        cudaGetLastError();
        return TINT4_ERR_CUDA;
    }
    return last_launch_status();
}

// The fused linear at M <= kFuseMaxRows, K <= kS8FuseMaxK: one launch of the
// small-M kernel that rotates and quantizes x itself (group G, codes in
// [-Q, Q]) while its first weight boxes are in flight.
template <int G, int Q>
tint4_status launch_linear_small_fused(const __nv_bfloat16* x, const uint8_t* w, const float* sr,
                                       const __nv_bfloat16* bias, __nv_bfloat16* y, int M, int N,
                                       int K, cudaStream_t stream) {
    auto kern = w4a8_small_kernel<1, false, false, G, Q>;
    constexpr int smem = S8Cfg<1>::SMEM + kS8FuseBytes;
    CUtensorMap tw;
    if (!make_map_u8(&tw, w, K / 2, N, K / 2, 128, 32, CU_TENSOR_MAP_SWIZZLE_128B))
        return TINT4_ERR_CUDA;
    int dev = 0;
    cudaGetDevice(&dev);
    static std::atomic<bool> attr_done[kMaxDevices];
    if (!attr_done[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess) {
            cudaGetLastError();
            return TINT4_ERR_CUDA;
        }
        attr_done[dev].store(true, std::memory_order_release);
    }
    const int nblk = N / 16;
    const int sms = num_sms(dev);
    const int grid = nblk <= kS8MB * sms ? std::min(sms, nblk) : (nblk + kS8MB - 1) / kS8MB;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(S8Cfg<1>::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tw, reinterpret_cast<const uint8_t*>(x),
                           static_cast<const float*>(nullptr), sr, bias, static_cast<void*>(y), M,
                           N, K, 0xF0F0F0F0u, g_decode_prefetch.load(std::memory_order_relaxed),
                           g_wait_limit_ns.load(std::memory_order_relaxed),
                           static_cast<const uint8_t*>(nullptr)) != cudaSuccess) {
        cudaGetLastError();
        return TINT4_ERR_CUDA;
    }
    return last_launch_status();
}

template <int Q>
tint4_status launch_linear_small_fused_g(const __nv_bfloat16* x, const uint8_t* w, const float* sr,
                                         const __nv_bfloat16* bias, __nv_bfloat16* y, int M, int N,
                                         int K, int g, cudaStream_t stream) {
    switch (g) {
        case 0: return launch_linear_small_fused<0, Q>(x, w, sr, bias, y, M, N, K, stream);
        case 16: return launch_linear_small_fused<16, Q>(x, w, sr, bias, y, M, N, K, stream);
        case 64: return launch_linear_small_fused<64, Q>(x, w, sr, bias, y, M, N, K, stream);
        default: return launch_linear_small_fused<256, Q>(x, w, sr, bias, y, M, N, K, stream);
    }
}

// The fused linears keep their int8 codes in the tensor-core GEMM's
// even/odd K order whenever that GEMM runs them (past the small-M kernel).
bool linear_codes_evod(int M) { return M > kS8MaxM; }

// Rotation + int8 codes of x (codes in [-Q, Q]) for a fused linear, in the
// order linear_codes_evod picks.
template <int Q>
void launch_linear_codes(const tint4_bf16* x, int M, int K, int group, void* codes,
                         float* tok_scale, cudaStream_t st) {
    const auto* xb = reinterpret_cast<const __nv_bfloat16*>(x);
    if (linear_codes_evod(M))
        launch_rq_g<__nv_bfloat16, Q, false, true>(xb, M, K, group, codes, tok_scale, st);
    else
        launch_rq_g<__nv_bfloat16, Q, false>(xb, M, K, group, codes, tok_scale, st);
}

// A_INT4: activation codes packed two per byte (else int8, one per byte).
// EVOD: int8 codes in the even/odd K order (only where linear_codes_evod(M)).
template <bool A_INT4, bool OUT_I32, bool EVOD = false>
tint4_status launch_gemm(const void* a, const uint8_t* w, const float* st, const float* sr,
                         const __nv_bfloat16* bias, void* out, int M, int N, int K,
                         cudaStream_t stream, bool pdl) {
    static_assert(!(EVOD && A_INT4), "packed codes are widened in the kernel");
    if (EVOD && !linear_codes_evod(M)) return TINT4_ERR_INVALID_ARG;
    if (M <= 8)
        return launch_gemm_small<1, A_INT4, OUT_I32>(a, w, st, sr, bias, out, M, N, K, stream, pdl);
    if (M <= kS8MaxM)
        return launch_gemm_small<2, A_INT4, OUT_I32>(a, w, st, sr, bias, out, M, N, K, stream, pdl);
    TmGroups grp{};
    grp.row_scale[0] = sr;
    grp.bias[0] = bias;
    grp.out[0] = out;
    grp.N[0] = N;
    grp.count = 1;
    return launch_gemm_tmem<OUT_I32, A_INT4, false, EVOD>(a, st, grp, &w, M, K, stream, pdl);
}

// The fused linears' workspace: the activation codes (one byte per code) and
// the token scales, each part 256-byte aligned.
struct LinearWs {
    uint8_t* codes;
    float* tok_scale;
};

LinearWs linear_ws(void* ws, int M, int K) {
    uint8_t* b = static_cast<uint8_t*>(ws);
    return LinearWs{b, reinterpret_cast<float*>(b + align_up(static_cast<size_t>(M) * K, 256))};
}

tint4_status gemm_entry(bool a_int4, const void* a, const float* tok_scale, const uint8_t* w,
                        const float* row_scale, const tint4_bf16* bias, tint4_bf16* y, int M,
                        int N, int K, void* stream) {
    tint4_status s = check_mnk(M, N, K);
    if (s != TINT4_OK) return s;
    if (M > 0 && (!a || !tok_scale || !w || !row_scale || !y)) return TINT4_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(tok_scale) || !aligned16(w) || !aligned16(row_scale) ||
        !aligned16(y) || !aligned16(bias))
        return TINT4_ERR_MISALIGNED;
    if ((s = check_device()) != TINT4_OK) return s;
    if (M == 0) return TINT4_OK;
    const auto* b = reinterpret_cast<const __nv_bfloat16*>(bias);
    return a_int4 ? launch_gemm<true, false>(a, w, tok_scale, row_scale, b, y, M, N, K,
                                             as_stream(stream), false)
                  : launch_gemm<false, false>(a, w, tok_scale, row_scale, b, y, M, N, K,
                                              as_stream(stream), false);
}

// The fused linear after its checks (M > 0; ws: a workspace of at least
// convrot_linear_workspace_size bytes, 256-byte aligned).
tint4_status linear_run(int bits, const tint4_bf16* x, const uint8_t* w_packed,
                        const float* row_scale, const tint4_bf16* bias, tint4_bf16* y, int M,
                        int N, int K, int group, void* ws, cudaStream_t st) {
    const auto* b = reinterpret_cast<const __nv_bfloat16*>(bias);
    if (M <= kFuseMaxRows && K <= kS8FuseMaxK) {
        // decode: one launch, the codes never leave the CTA
        const auto* xb = reinterpret_cast<const __nv_bfloat16*>(x);
        auto* yb = reinterpret_cast<__nv_bfloat16*>(y);
        return bits == 8 ? launch_linear_small_fused_g<127>(xb, w_packed, row_scale, b, yb, M, N, K,
                                                            group, st)
                         : launch_linear_small_fused_g<7>(xb, w_packed, row_scale, b, yb, M, N, K,
                                                          group, st);
    }
    // one int8 per code for both widths: the W4A4 codes (in [-7, 7]) are kept
    // one per byte in the workspace and run through the W4A8 kernel, whose
    // int32 sums are the same numbers
    const LinearWs w = linear_ws(ws, M, K);
    if (bits == 8) launch_linear_codes<127>(x, M, K, group, w.codes, w.tok_scale, st);
    else launch_linear_codes<7>(x, M, K, group, w.codes, w.tok_scale, st);
    tint4_status s = last_launch_status();
    if (s != TINT4_OK) return s;
    return linear_codes_evod(M)
               ? launch_gemm<false, false, true>(w.codes, w_packed, w.tok_scale, row_scale, b, y, M,
                                                 N, K, st, true)
               : launch_gemm<false, false>(w.codes, w_packed, w.tok_scale, row_scale, b, y, M, N, K,
                                           st, true);
}

tint4_status linear_entry(int bits, const tint4_bf16* x, const uint8_t* w_packed,
                          const float* row_scale, const tint4_bf16* bias, tint4_bf16* y, int M,
                          int N, int K, int group, void* workspace, size_t workspace_bytes,
                          void* stream) {
    tint4_status s = check_mnk(M, N, K);
    if (s != TINT4_OK) return s;
    if ((s = check_rq_shape(M, K, group)) != TINT4_OK) return s;
    if (M > 0 && (!x || !w_packed || !row_scale || !y)) return TINT4_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_packed) || !aligned16(row_scale) || !aligned16(y) ||
        !aligned16(bias))
        return TINT4_ERR_MISALIGNED;
    if (M > 0 && (!workspace || workspace_bytes < convrot_linear_workspace_size(M, K, bits)))
        return TINT4_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TINT4_ERR_MISALIGNED;
    if ((s = check_device()) != TINT4_OK) return s;
    if (M == 0) return TINT4_OK;
    return linear_run(bits, x, w_packed, row_scale, bias, y, M, N, K, group, workspace,
                      as_stream(stream));
}

// ------------------------------------------------------------------ W4A16

// Large M: the tcgen05 GEMM with the weights dequantized into TMEM
// (w4a16_gemm.cuh).
tint4_status launch_w4a16_gemm(const __nv_bfloat16* x, const uint8_t* q, const __nv_bfloat16* s,
                               const uint8_t* z, __nv_bfloat16* y, int M, int N, int K,
                               cudaStream_t st) {
    auto kern = w4a16_tmem_gemm_kernel;
    CUtensorMap tx, tq;
    bool ok = make_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, M,
                          static_cast<uint64_t>(K) * 2, kWgBK, kWgBN, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map_u8(&tq, q, K / 2, N, K / 2, kWgBK / 2, kWgBM, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return TINT4_ERR_CUDA;
    int dev = 0;
    cudaGetDevice(&dev);
    static std::atomic<bool> attr_done[kMaxDevices];
    if (!attr_done[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kWgSmemBytes) != cudaSuccess) {
            cudaGetLastError();
            return TINT4_ERR_CUDA;
        }
        attr_done[dev].store(true, std::memory_order_release);
    }
    const int tiles = ((M + kWgBN - 1) / kWgBN) * ((N + kWgBM - 1) / kWgBM);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(std::min(tiles, num_sms(dev)), 1, 1);
    cfg.blockDim = dim3(kWgThreads, 1, 1);
    cfg.dynamicSmemBytes = kWgSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tx, tq, s, z, y, M, N, K,
                           g_wait_limit_ns.load(std::memory_order_relaxed)) != cudaSuccess) {
        cudaGetLastError();
        return TINT4_ERR_CUDA;
    }
    return last_launch_status();
}

template <int NB>
tint4_status launch_w4a16(const __nv_bfloat16* x, const uint8_t* q, const __nv_bfloat16* s,
                          const uint8_t* z, __nv_bfloat16* y, int M, int N, int K,
                          cudaStream_t st) {
    using C = W16Cfg<NB>;
    auto kern = w4a16_mma_kernel<NB>;
    CUtensorMap tw;
    if (!make_map_u8(&tw, q, K / 2, N, K / 2, 128, 32, CU_TENSOR_MAP_SWIZZLE_128B))
        return TINT4_ERR_CUDA;
    int dev = 0;
    cudaGetDevice(&dev);
    static std::atomic<bool> attr_done[kMaxDevices];
    if (!attr_done[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::kSmemMax) != cudaSuccess) {
            cudaGetLastError();
            return TINT4_ERR_CUDA;
        }
        attr_done[dev].store(true, std::memory_order_release);
    }
    const int nblk = N / 16;
    // one CTA per SM unless that would give a CTA more than kW16MB blocks
    const int sms = num_sms(dev);
    const int grid = nblk <= kW16MB * sms ? std::min(sms, nblk) : (nblk + kW16MB - 1) / kW16MB;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::smem(K / kW16Group);
    cfg.stream = st;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const W16Consts kc{0x000F000Fu, 0x43004300u};
    if (cudaLaunchKernelEx(&cfg, kern, tw, x, s, z, y, M, N, K, kc,
                           g_decode_prefetch.load(std::memory_order_relaxed),
                           g_wait_limit_ns.load(std::memory_order_relaxed)) != cudaSuccess) {
        cudaGetLastError();
        return TINT4_ERR_CUDA;
    }
    return last_launch_status();
}

// ------------------------------------------------------------------ bounded-wait test

__global__ void bounded_wait_test_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ uint32_t abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0u;
        fence_mbarrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // nobody arrives on `bar`: the wait must run out and report
        mbar_wait_bounded(&bar, 0, &abort_flag, limit_ns, kDevErrTimeoutTest);
    }
}

// ------------------------------------------------------------------ allocation-free fused linear
//
// For callers that cannot allocate device memory: the scratch of the fused
// W4A8 linear (activation codes + token scales) lives in one fixed device
// array that every device holds from the moment it loads this library until
// the process exits.  Host code must not hand the array's name to a kernel
// (on the host it is only a stand-in for the symbol); its device address is
// looked up once per device with cudaGetSymbolAddress.

constexpr size_t kStaticScratchBytes = size_t(16) << 20;   // 16 MiB
static __device__ __align__(256) uint8_t g_static_linear_scratch[kStaticScratchBytes];

std::mutex g_static_scratch_mu;
void* g_static_scratch_ptr[kMaxDevices];
void* g_static_scratch_ctx[kMaxDevices];   // the context the address belongs to

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// Device address of the scratch array on `dev` (the current device), looked
// up on the first call and again whenever the device's context has changed
// since (a context rebuilt after cudaDeviceReset loads the module anew, and
// the array may move).  nullptr on failure.
void* static_scratch_address(int dev) {
    std::lock_guard<std::mutex> lock(g_static_scratch_mu);
    CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    if (get_ctx == nullptr) return nullptr;
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) ctx = nullptr;
    if (ctx == nullptr || g_static_scratch_ptr[dev] == nullptr || g_static_scratch_ctx[dev] != ctx) {
        // (the lookup also makes the device's primary context current)
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_linear_scratch) != cudaSuccess ||
            get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) {
            cudaGetLastError();
            return nullptr;
        }
        g_static_scratch_ptr[dev] = p;
        g_static_scratch_ctx[dev] = ctx;
    }
    return g_static_scratch_ptr[dev];
}

static_assert(TINT4_MAX_GROUPS == kTmMaxGroups, "group limit of the ABI and the kernel");

// Shape, pointer and alignment rules of a grouped call (nothing launched).
tint4_status check_groups(const tint4_weight_group* groups, int num_groups, int M, int K) {
    if (groups == nullptr || num_groups < 1) return TINT4_ERR_INVALID_ARG;
    if (num_groups > TINT4_MAX_GROUPS) return TINT4_ERR_UNSUPPORTED_SHAPE;
    for (int g = 0; g < num_groups; ++g) {
        const tint4_weight_group& w = groups[g];
        tint4_status s = check_mnk(M, w.N, K);
        if (s != TINT4_OK) return s;
        if (M > 0 && (!w.w_packed || !w.row_scale || !w.y)) return TINT4_ERR_INVALID_ARG;
        if (!aligned16(w.w_packed) || !aligned16(w.row_scale) || !aligned16(w.bias) ||
            !aligned16(w.y))
            return TINT4_ERR_MISALIGNED;
    }
    return TINT4_OK;
}

// EVOD: int8 codes in the even/odd K order (only where linear_codes_evod(M)).
template <bool EVOD = false>
tint4_status launch_gemm_grouped(const int8_t* codes, const float* tok_scale,
                                 const tint4_weight_group* groups, int num_groups, int M, int K,
                                 cudaStream_t st, bool pdl) {
    if (EVOD && !linear_codes_evod(M)) return TINT4_ERR_INVALID_ARG;
    if (M <= kS8MaxM) {
        // every weight is read once per launch anyway: one small-M launch per group
        for (int g = 0; g < num_groups; ++g) {
            const tint4_weight_group& w = groups[g];
            const tint4_status s = launch_gemm<false, false>(
                codes, w.w_packed, tok_scale, w.row_scale,
                reinterpret_cast<const __nv_bfloat16*>(w.bias), w.y, M, w.N, K, st,
                pdl || g > 0);
            if (s != TINT4_OK) return s;
        }
        return TINT4_OK;
    }
    TmGroups grp{};
    const uint8_t* w[kTmMaxGroups] = {};
    for (int g = 0; g < num_groups; ++g) {
        w[g] = groups[g].w_packed;
        grp.row_scale[g] = groups[g].row_scale;
        grp.bias[g] = reinterpret_cast<const __nv_bfloat16*>(groups[g].bias);
        grp.out[g] = groups[g].y;
        grp.N[g] = groups[g].N;
    }
    grp.count = num_groups;
    return launch_gemm_tmem<false, false, false, EVOD>(codes, tok_scale, grp, w, M, K, st, pdl);
}

// W8A8: int8 codes x int8 weights, one tensor-core launch at every M; S16:
// fp16 row scales.
template <bool S16 = false>
tint4_status launch_w8a8(const int8_t* codes, const float* st, const int8_t* w, const void* sr,
                         const __nv_bfloat16* bias, __nv_bfloat16* y, int M, int N, int K,
                         cudaStream_t stream, bool pdl) {
    TmGroups grp{};
    grp.row_scale[0] = static_cast<const float*>(sr);   // fp16 bits when S16
    grp.bias[0] = bias;
    grp.out[0] = y;
    grp.N[0] = N;
    grp.count = 1;
    const uint8_t* wp = reinterpret_cast<const uint8_t*>(w);
    return launch_gemm_tmem<false, false, true, false, S16>(codes, st, grp, &wp, M, K, stream, pdl);
}

// ------------------------------------------------------------------ group-wise W4A8

static_assert(TINT4_WEIGHT_GROUP == kWeightGroup, "weight group of the ABI and the kernels");

// Shape rules of the group-wise GEMM: the W4A8 rules plus K a multiple of
// the weight group.
tint4_status check_gw_mnk(int M, int N, int K) {
    tint4_status s = check_mnk(M, N, K);
    if (s != TINT4_OK) return s;
    if (K % kWeightGroup != 0) return TINT4_ERR_UNSUPPORTED_SHAPE;
    return TINT4_OK;
}

template <int G, bool S16 = false>
void launch_pack_gw(const float* W, int N, int K, int asym, uint8_t* packed, void* scale,
                    uint8_t* zero, cudaStream_t st) {
    const long warps = static_cast<long>(N) * ((K + kQuantChunk - 1) / kQuantChunk);
    int dev = 0;
    cudaGetDevice(&dev);
    const long grid = std::min<long>((warps + 7) / 8, 8L * num_sms(dev));
    pack_weights_groupwise_kernel<G, S16><<<static_cast<int>(grid), 256, 0, st>>>(W, N, K, asym,
                                                                                 packed, scale, zero);
}

// The tensor-core GEMM with group-wise scales at every M (gemm_tmem_gw.cuh).
template <bool ASYM, bool EVOD, bool S16 = false>
tint4_status launch_gemm_gw(const int8_t* codes, const float* tok_scale, const uint8_t* w,
                            const void* wscale, const uint8_t* wzero, const __nv_bfloat16* bias,
                            __nv_bfloat16* y, int M, int N, int K, cudaStream_t stream, bool pdl) {
    auto kern = w4a8_gw_tmem_gemm_kernel<ASYM, EVOD, S16>;
    CUtensorMap ta, tw, ty;
    bool ok = make_map_u8(&ta, codes, K, M, K, kGwBK, kGwBN, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map_u8(&tw, w, K / 2, N, K / 2, kGwBK / 2, kGwBM, CU_TENSOR_MAP_SWIZZLE_64B);
    ok = ok && make_map_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M,
                           static_cast<uint64_t>(N) * 2, kGwBM, kGwBN, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return TINT4_ERR_CUDA;
    int dev = 0;
    cudaGetDevice(&dev);
    static std::atomic<bool> attr_done[kMaxDevices];
    if (!attr_done[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kGwSmemBytes) != cudaSuccess) {
            cudaGetLastError();
            return TINT4_ERR_CUDA;
        }
        attr_done[dev].store(true, std::memory_order_release);
    }
    const int tiles = ((M + kGwBN - 1) / kGwBN) * ((N + kGwBM - 1) / kGwBM);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(std::min(tiles, num_sms(dev)), 1, 1);
    cfg.blockDim = dim3(kGwThreads, 1, 1);
    cfg.dynamicSmemBytes = kGwSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    if (pdl) {
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    const uint64_t wait_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
    if (cudaLaunchKernelEx(&cfg, kern, ta, tw, ty, tok_scale, wscale, wzero, bias, M, N, K,
                           wait_ns) != cudaSuccess) {
        cudaGetLastError();
        return TINT4_ERR_CUDA;
    }
    return TINT4_OK;
}

// Small M (<= kS8MaxM tokens, natural-order codes, K <= 128 kS8GwMaxGroups):
// the streaming kernel with group-wise scales (w4a8_small.cuh, GW = 1
// symmetric / 2 asymmetric); else the tensor-core kernel.
bool gw_streaming(int M, int K) { return M <= kS8MaxM && K <= 128 * kS8GwMaxGroups; }

template <int NB, int GW, bool S16 = false>
tint4_status launch_gemm_small_gw(const int8_t* a, const uint8_t* w, const float* st,
                                  const void* wscale, const uint8_t* wzero,
                                  const __nv_bfloat16* bias, __nv_bfloat16* y, int M, int N, int K,
                                  cudaStream_t stream, bool pdl) {
    auto kern = w4a8_small_kernel<NB, false, false, 0, 0, GW, S16>;
    constexpr int smem = S8Cfg<NB>::FUSE_OFF + kS8GwBytes + 1024;
    static_assert(smem <= 227 * 1024, "shared memory budget");
    CUtensorMap tw;
    if (!make_map_u8(&tw, w, K / 2, N, K / 2, 128, 32, CU_TENSOR_MAP_SWIZZLE_128B))
        return TINT4_ERR_CUDA;
    int dev = 0;
    cudaGetDevice(&dev);
    static std::atomic<bool> attr_done[kMaxDevices];
    if (!attr_done[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess) {
            cudaGetLastError();
            return TINT4_ERR_CUDA;
        }
        attr_done[dev].store(true, std::memory_order_release);
    }
    const int nblk = N / 16;
    const int sms = num_sms(dev);
    const int grid = nblk <= kS8MB * sms ? std::min(sms, nblk) : (nblk + kS8MB - 1) / kS8MB;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(S8Cfg<NB>::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    (void)pdl;   // always programmatic, as launch_gemm_small
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tw, reinterpret_cast<const uint8_t*>(a), st,
                           static_cast<const float*>(wscale), bias, static_cast<void*>(y), M, N, K,
                           0xF0F0F0F0u,
                           g_decode_prefetch.load(std::memory_order_relaxed),
                           g_wait_limit_ns.load(std::memory_order_relaxed), wzero) != cudaSuccess) {
        cudaGetLastError();
        return TINT4_ERR_CUDA;
    }
    return last_launch_status();
}

template <bool EVOD, bool S16 = false>
tint4_status launch_gemm_gw_any(const int8_t* codes, const float* tok_scale, const uint8_t* w,
                                const void* wscale, const uint8_t* wzero, const tint4_bf16* bias,
                                tint4_bf16* y, int M, int N, int K, cudaStream_t st, bool pdl) {
    const auto* b = reinterpret_cast<const __nv_bfloat16*>(bias);
    auto* yb = reinterpret_cast<__nv_bfloat16*>(y);
    if (gw_streaming(M, K)) {
        if (EVOD) return TINT4_ERR_INVALID_ARG;   // the streaming kernel reads natural-order codes
        if (M <= 8)
            return wzero ? launch_gemm_small_gw<1, 2, S16>(codes, w, tok_scale, wscale, wzero, b, yb,
                                                           M, N, K, st, pdl)
                         : launch_gemm_small_gw<1, 1, S16>(codes, w, tok_scale, wscale, nullptr, b,
                                                           yb, M, N, K, st, pdl);
        return wzero ? launch_gemm_small_gw<2, 2, S16>(codes, w, tok_scale, wscale, wzero, b, yb, M,
                                                       N, K, st, pdl)
                     : launch_gemm_small_gw<2, 1, S16>(codes, w, tok_scale, wscale, nullptr, b, yb,
                                                       M, N, K, st, pdl);
    }
    return wzero ? launch_gemm_gw<true, EVOD, S16>(codes, tok_scale, w, wscale, wzero, b, yb, M, N,
                                                   K, st, pdl)
                 : launch_gemm_gw<false, EVOD, S16>(codes, tok_scale, w, wscale, nullptr, b, yb, M,
                                                    N, K, st, pdl);
}

// ------------------------------------------------------------------ fp32 / fp16 weight scales
//
// The group-wise and W8A8 entry points with S16 = false take fp32 scales,
// with S16 = true IEEE fp16 scales (the stored format of "ComfyUI-INT-Crush",
// "Weight Format").

template <bool S16>
tint4_status pack_weights_groupwise_impl(const float* W, int N, int K, int group, int asym,
                                         uint8_t* w_packed, void* w_scale, uint8_t* w_zero,
                                         void* stream) {
    if (asym != 0 && asym != 1) return TINT4_ERR_INVALID_ARG;
    tint4_status s = check_rq_shape(N, K, group);
    if (s != TINT4_OK) return s;
    if (K % kWeightGroup != 0) return TINT4_ERR_UNSUPPORTED_SHAPE;
    if (N > 0 && (!W || !w_packed || !w_scale || (asym && !w_zero))) return TINT4_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(w_packed) || !aligned16(w_scale) || !aligned16(w_zero))
        return TINT4_ERR_MISALIGNED;
    if ((s = check_device()) != TINT4_OK) return s;
    if (N == 0) return TINT4_OK;
    cudaStream_t st = as_stream(stream);
    switch (group) {
        case 0: launch_pack_gw<0, S16>(W, N, K, asym, w_packed, w_scale, w_zero, st); break;
        case 16: launch_pack_gw<16, S16>(W, N, K, asym, w_packed, w_scale, w_zero, st); break;
        case 64: launch_pack_gw<64, S16>(W, N, K, asym, w_packed, w_scale, w_zero, st); break;
        default: launch_pack_gw<256, S16>(W, N, K, asym, w_packed, w_scale, w_zero, st); break;
    }
    return last_launch_status();
}

template <bool S16>
tint4_status gemm_groupwise_impl(const int8_t* a, const float* tok_scale, const uint8_t* w_packed,
                                 const void* w_scale, const uint8_t* w_zero, const tint4_bf16* bias,
                                 tint4_bf16* y, int M, int N, int K, void* stream) {
    tint4_status s = check_gw_mnk(M, N, K);
    if (s != TINT4_OK) return s;
    if (M > 0 && (!a || !tok_scale || !w_packed || !w_scale || !y)) return TINT4_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(tok_scale) || !aligned16(w_packed) || !aligned16(w_scale) ||
        !aligned16(w_zero) || !aligned16(bias) || !aligned16(y))
        return TINT4_ERR_MISALIGNED;
    if ((s = check_device()) != TINT4_OK) return s;
    if (M == 0) return TINT4_OK;
    return launch_gemm_gw_any<false, S16>(a, tok_scale, w_packed, w_scale, w_zero, bias, y, M, N, K,
                                          as_stream(stream), false);
}

template <bool S16>
tint4_status linear_groupwise_impl(const tint4_bf16* x, const uint8_t* w_packed, const void* w_scale,
                                   const uint8_t* w_zero, const tint4_bf16* bias, tint4_bf16* y,
                                   int M, int N, int K, int group, void* workspace,
                                   size_t workspace_bytes, void* stream) {
    tint4_status s = check_gw_mnk(M, N, K);
    if (s != TINT4_OK) return s;
    if ((s = check_rq_shape(M, K, group)) != TINT4_OK) return s;
    if (M > 0 && (!x || !w_packed || !w_scale || !y)) return TINT4_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_packed) || !aligned16(w_scale) || !aligned16(w_zero) ||
        !aligned16(bias) || !aligned16(y))
        return TINT4_ERR_MISALIGNED;
    if (M > 0 && (!workspace || workspace_bytes < convrot_linear_workspace_size(M, K, 8)))
        return TINT4_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TINT4_ERR_MISALIGNED;
    if ((s = check_device()) != TINT4_OK) return s;
    if (M == 0) return TINT4_OK;
    int8_t* codes = static_cast<int8_t*>(workspace);
    float* tok_scale = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                                align_up(static_cast<size_t>(M) * K, 256));
    cudaStream_t st = as_stream(stream);
    // even/odd codes whenever the tensor-core kernel runs them
    const auto* xb = reinterpret_cast<const __nv_bfloat16*>(x);
    if (gw_streaming(M, K))
        launch_rq_g<__nv_bfloat16, 127, false>(xb, M, K, group, codes, tok_scale, st);
    else
        launch_rq_g<__nv_bfloat16, 127, false, true>(xb, M, K, group, codes, tok_scale, st);
    if ((s = last_launch_status()) != TINT4_OK) return s;
    return !gw_streaming(M, K)
               ? launch_gemm_gw_any<true, S16>(codes, tok_scale, w_packed, w_scale, w_zero, bias, y,
                                               M, N, K, st, true)
               : launch_gemm_gw_any<false, S16>(codes, tok_scale, w_packed, w_scale, w_zero, bias,
                                                y, M, N, K, st, true);
}

template <bool S16>
tint4_status quantize_weights_int8_impl(const float* W, int N, int K, int group, int8_t* w_int8,
                                        void* row_scale, void* stream) {
    tint4_status s = check_rq_shape(N, K, group);
    if (s != TINT4_OK) return s;
    if (N > 0 && (!W || !w_int8 || !row_scale)) return TINT4_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(w_int8) || !aligned16(row_scale)) return TINT4_ERR_MISALIGNED;
    if ((s = check_device()) != TINT4_OK) return s;
    if (N == 0) return TINT4_OK;
    launch_rq_g<float, 127, false, false, S16>(W, N, K, group, w_int8, row_scale, as_stream(stream));
    return last_launch_status();
}

template <bool S16>
tint4_status w8a8_gemm_impl(const int8_t* codes, const float* tok_scale, const int8_t* w_int8,
                            const void* row_scale, const tint4_bf16* bias, tint4_bf16* y, int M,
                            int N, int K, void* stream) {
    tint4_status s = check_mnk(M, N, K);
    if (s != TINT4_OK) return s;
    if (M > 0 && (!codes || !tok_scale || !w_int8 || !row_scale || !y))
        return TINT4_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(tok_scale) || !aligned16(w_int8) ||
        !aligned16(row_scale) || !aligned16(y) || !aligned16(bias))
        return TINT4_ERR_MISALIGNED;
    if ((s = check_device()) != TINT4_OK) return s;
    if (M == 0) return TINT4_OK;
    return launch_w8a8<S16>(codes, tok_scale, w_int8, row_scale,
                            reinterpret_cast<const __nv_bfloat16*>(bias),
                            reinterpret_cast<__nv_bfloat16*>(y), M, N, K, as_stream(stream), false);
}

template <bool S16>
tint4_status w8a8_linear_impl(const tint4_bf16* x, const int8_t* w_int8, const void* row_scale,
                              const tint4_bf16* bias, tint4_bf16* y, int M, int N, int K, int group,
                              void* workspace, size_t workspace_bytes, void* stream) {
    tint4_status s = check_mnk(M, N, K);
    if (s != TINT4_OK) return s;
    if ((s = check_rq_shape(M, K, group)) != TINT4_OK) return s;
    if (M > 0 && (!x || !w_int8 || !row_scale || !y)) return TINT4_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_int8) || !aligned16(row_scale) || !aligned16(y) ||
        !aligned16(bias))
        return TINT4_ERR_MISALIGNED;
    if (M > 0 && (!workspace || workspace_bytes < convrot_linear_workspace_size(M, K, 8)))
        return TINT4_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TINT4_ERR_MISALIGNED;
    if ((s = check_device()) != TINT4_OK) return s;
    if (M == 0) return TINT4_OK;
    int8_t* codes = static_cast<int8_t*>(workspace);
    float* tok_scale = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                                align_up(static_cast<size_t>(M) * K, 256));
    cudaStream_t st = as_stream(stream);
    launch_rq_g<__nv_bfloat16, 127, false>(reinterpret_cast<const __nv_bfloat16*>(x), M, K, group,
                                           codes, tok_scale, st);
    if ((s = last_launch_status()) != TINT4_OK) return s;
    return launch_w8a8<S16>(codes, tok_scale, w_int8, row_scale,
                            reinterpret_cast<const __nv_bfloat16*>(bias),
                            reinterpret_cast<__nv_bfloat16*>(y), M, N, K, st, true);
}

}  // namespace

// ====================================================================== C ABI

extern "C" {

int tint4_abi_version(void) { return kAbiVersion; }

const char* tint4_status_string(tint4_status status) {
    switch (status) {
        case TINT4_OK: return "ok";
        case TINT4_ERR_INVALID_ARG: return "invalid argument";
        case TINT4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case TINT4_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case TINT4_ERR_CUDA: return "CUDA error";
        case TINT4_ERR_TIMEOUT: return "device-side wait timed out";
        case TINT4_ERR_WORKSPACE: return "workspace missing or too small";
        case TINT4_ERR_NO_DEVICE: return "current device is not an sm_100 GPU";
    }
    return "unknown status";
}

tint4_status tint4_pack_weights(const float* W, int N, int K, int group, uint8_t* w_packed,
                                float* row_scale, void* stream) {
    tint4_status s = check_rq_shape(N, K, group);
    if (s != TINT4_OK) return s;
    if (N > 0 && (!W || !w_packed || !row_scale)) return TINT4_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(w_packed) || !aligned16(row_scale)) return TINT4_ERR_MISALIGNED;
    if ((s = check_device()) != TINT4_OK) return s;
    if (N == 0) return TINT4_OK;
    launch_rq_g<float, 7, true>(W, N, K, group, w_packed, row_scale, as_stream(stream));
    return last_launch_status();
}

tint4_status convrot_quantize_act(const tint4_bf16* x, int M, int K, int group, int bits,
                                  void* codes, float* tok_scale, void* stream) {
    if (bits != 8 && bits != 4) return TINT4_ERR_INVALID_ARG;
    tint4_status s = check_rq_shape(M, K, group);
    if (s != TINT4_OK) return s;
    if (M > 0 && (!x || !codes || !tok_scale)) return TINT4_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(tok_scale)) return TINT4_ERR_MISALIGNED;
    if ((s = check_device()) != TINT4_OK) return s;
    if (M == 0) return TINT4_OK;
    const auto* xb = reinterpret_cast<const __nv_bfloat16*>(x);
    if (bits == 8)
        launch_rq_g<__nv_bfloat16, 127, false>(xb, M, K, group, codes, tok_scale, as_stream(stream));
    else
        launch_rq_g<__nv_bfloat16, 7, true>(xb, M, K, group, codes, tok_scale, as_stream(stream));
    return last_launch_status();
}

tint4_status w4a8_gemm(const int8_t* a, const float* tok_scale, const uint8_t* w_packed,
                       const float* row_scale, const tint4_bf16* bias, tint4_bf16* y, int M,
                       int N, int K, void* stream) {
    return gemm_entry(false, a, tok_scale, w_packed, row_scale, bias, y, M, N, K, stream);
}

tint4_status w4a4_gemm(const uint8_t* a_packed, const float* tok_scale, const uint8_t* w_packed,
                       const float* row_scale, const tint4_bf16* bias, tint4_bf16* y, int M,
                       int N, int K, void* stream) {
    return gemm_entry(true, a_packed, tok_scale, w_packed, row_scale, bias, y, M, N, K, stream);
}

tint4_status w4a4_gemm_widened(const uint8_t* a_packed, const float* tok_scale,
                               const uint8_t* w_packed, const float* row_scale,
                               const tint4_bf16* bias, tint4_bf16* y, int M, int N, int K,
                               void* workspace, size_t workspace_bytes, void* stream) {
    tint4_status s = check_mnk(M, N, K);
    if (s != TINT4_OK) return s;
    if (M > 0 && (!a_packed || !tok_scale || !w_packed || !row_scale || !y))
        return TINT4_ERR_INVALID_ARG;
    if (!aligned16(a_packed) || !aligned16(tok_scale) || !aligned16(w_packed) ||
        !aligned16(row_scale) || !aligned16(y) || !aligned16(bias))
        return TINT4_ERR_MISALIGNED;
    if (!linear_codes_evod(M))   // the streaming kernel reads packed codes itself
        return gemm_entry(true, a_packed, tok_scale, w_packed, row_scale, bias, y, M, N, K, stream);
    if (!workspace || workspace_bytes < convrot_linear_workspace_size(M, K, 4))
        return TINT4_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TINT4_ERR_MISALIGNED;
    int dev = 0;
    if ((s = check_device(&dev)) != TINT4_OK) return s;
    cudaStream_t st = as_stream(stream);
    int8_t* codes = static_cast<int8_t*>(workspace);
    const long pieces = static_cast<long>(M) * K / 32;
    const int grid = static_cast<int>(std::min<long>((pieces + 255) / 256, 8L * num_sms(dev)));
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, widen_int4_codes_kernel, a_packed, codes, pieces) != cudaSuccess) {
        cudaGetLastError();
        return TINT4_ERR_CUDA;
    }
    return launch_gemm<false, false, true>(codes, w_packed, tok_scale, row_scale,
                                           reinterpret_cast<const __nv_bfloat16*>(bias), y, M, N,
                                           K, st, true);
}

size_t convrot_w4a8_linear_workspace(int M, int K) {
    return convrot_linear_workspace_size(M, K, 8);
}

size_t convrot_linear_workspace_size(int M, int K, int bits) {
    if (M < 0 || K < 0 || (bits != 8 && bits != 4)) return 0;
    const size_t code_bytes = static_cast<size_t>(M) * K;   // one byte per code, both widths
    return align_up(code_bytes, 256) + align_up(static_cast<size_t>(M) * sizeof(float), 256);
}

tint4_status convrot_w4a8_linear(const tint4_bf16* x, const uint8_t* w_packed,
                                 const float* row_scale, const tint4_bf16* bias, tint4_bf16* y,
                                 int M, int N, int K, int group, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    return linear_entry(8, x, w_packed, row_scale, bias, y, M, N, K, group, workspace,
                        workspace_bytes, stream);
}

tint4_status convrot_w4a4_linear(const tint4_bf16* x, const uint8_t* w_packed,
                                 const float* row_scale, const tint4_bf16* bias, tint4_bf16* y,
                                 int M, int N, int K, int group, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    return linear_entry(4, x, w_packed, row_scale, bias, y, M, N, K, group, workspace,
                        workspace_bytes, stream);
}

tint4_status w4a8_gemm_grouped(const int8_t* codes, const float* tok_scale,
                                          const tint4_weight_group* groups, int num_groups, int M,
                                          int K, void* stream) {
    tint4_status s = check_groups(groups, num_groups, M, K);
    if (s != TINT4_OK) return s;
    if (M > 0 && (!codes || !tok_scale)) return TINT4_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(tok_scale)) return TINT4_ERR_MISALIGNED;
    if ((s = check_device()) != TINT4_OK) return s;
    if (M == 0) return TINT4_OK;
    return launch_gemm_grouped(codes, tok_scale, groups, num_groups, M, K, as_stream(stream),
                               false);
}

tint4_status convrot_w4a8_linear_grouped(const tint4_bf16* x,
                                                    const tint4_weight_group* groups,
                                                    int num_groups, int M, int K, int group,
                                                    void* workspace, size_t workspace_bytes,
                                                    void* stream) {
    tint4_status s = check_groups(groups, num_groups, M, K);
    if (s != TINT4_OK) return s;
    if ((s = check_rq_shape(M, K, group)) != TINT4_OK) return s;
    if (M > 0 && !x) return TINT4_ERR_INVALID_ARG;
    if (!aligned16(x)) return TINT4_ERR_MISALIGNED;
    if (M > 0 && (!workspace || workspace_bytes < convrot_linear_workspace_size(M, K, 8)))
        return TINT4_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TINT4_ERR_MISALIGNED;
    if ((s = check_device()) != TINT4_OK) return s;
    if (M == 0) return TINT4_OK;
    const LinearWs w = linear_ws(workspace, M, K);
    int8_t* codes = reinterpret_cast<int8_t*>(w.codes);
    cudaStream_t st = as_stream(stream);
    launch_linear_codes<127>(x, M, K, group, codes, w.tok_scale, st);
    if ((s = last_launch_status()) != TINT4_OK) return s;
    return linear_codes_evod(M)
               ? launch_gemm_grouped<true>(codes, w.tok_scale, groups, num_groups, M, K, st, true)
               : launch_gemm_grouped(codes, w.tok_scale, groups, num_groups, M, K, st, true);
}

tint4_status tint4_pack_weights_groupwise(const float* W, int N, int K, int group, int asym,
                                          uint8_t* w_packed, float* w_scale, uint8_t* w_zero,
                                          void* stream) {
    return pack_weights_groupwise_impl<false>(W, N, K, group, asym, w_packed, w_scale, w_zero, stream);
}

tint4_status tint4_pack_weights_groupwise_f16(const float* W, int N, int K, int group, int asym,
                                              uint8_t* w_packed, tint4_f16* w_scale,
                                              uint8_t* w_zero, void* stream) {
    return pack_weights_groupwise_impl<true>(W, N, K, group, asym, w_packed, w_scale, w_zero, stream);
}

tint4_status w4a8_gemm_groupwise(const int8_t* a, const float* tok_scale,
                                 const uint8_t* w_packed, const float* w_scale,
                                 const uint8_t* w_zero, const tint4_bf16* bias, tint4_bf16* y,
                                 int M, int N, int K, void* stream) {
    return gemm_groupwise_impl<false>(a, tok_scale, w_packed, w_scale, w_zero, bias, y, M, N, K,
                                      stream);
}

tint4_status w4a8_gemm_groupwise_f16(const int8_t* a, const float* tok_scale,
                                     const uint8_t* w_packed, const tint4_f16* w_scale,
                                     const uint8_t* w_zero, const tint4_bf16* bias, tint4_bf16* y,
                                     int M, int N, int K, void* stream) {
    return gemm_groupwise_impl<true>(a, tok_scale, w_packed, w_scale, w_zero, bias, y, M, N, K,
                                     stream);
}

tint4_status convrot_w4a8_linear_groupwise(const tint4_bf16* x, const uint8_t* w_packed,
                                           const float* w_scale, const uint8_t* w_zero,
                                           const tint4_bf16* bias, tint4_bf16* y, int M, int N,
                                           int K, int group, void* workspace,
                                           size_t workspace_bytes, void* stream) {
    return linear_groupwise_impl<false>(x, w_packed, w_scale, w_zero, bias, y, M, N, K, group,
                                        workspace, workspace_bytes, stream);
}

tint4_status convrot_w4a8_linear_groupwise_f16(const tint4_bf16* x, const uint8_t* w_packed,
                                               const tint4_f16* w_scale, const uint8_t* w_zero,
                                               const tint4_bf16* bias, tint4_bf16* y, int M, int N,
                                               int K, int group, void* workspace,
                                               size_t workspace_bytes, void* stream) {
    return linear_groupwise_impl<true>(x, w_packed, w_scale, w_zero, bias, y, M, N, K, group,
                                       workspace, workspace_bytes, stream);
}

tint4_status tint4_quantize_weights_int8(const float* W, int N, int K, int group,
                                         int8_t* w_int8, float* row_scale, void* stream) {
    return quantize_weights_int8_impl<false>(W, N, K, group, w_int8, row_scale, stream);
}

tint4_status tint4_quantize_weights_int8_f16(const float* W, int N, int K, int group,
                                             int8_t* w_int8, tint4_f16* row_scale, void* stream) {
    return quantize_weights_int8_impl<true>(W, N, K, group, w_int8, row_scale, stream);
}

tint4_status w8a8_gemm(const int8_t* codes, const float* tok_scale, const int8_t* w_int8,
                       const float* row_scale, const tint4_bf16* bias, tint4_bf16* y, int M,
                       int N, int K, void* stream) {
    return w8a8_gemm_impl<false>(codes, tok_scale, w_int8, row_scale, bias, y, M, N, K, stream);
}

tint4_status w8a8_gemm_f16(const int8_t* codes, const float* tok_scale, const int8_t* w_int8,
                           const tint4_f16* row_scale, const tint4_bf16* bias, tint4_bf16* y, int M,
                           int N, int K, void* stream) {
    return w8a8_gemm_impl<true>(codes, tok_scale, w_int8, row_scale, bias, y, M, N, K, stream);
}

tint4_status convrot_w8a8_linear(const tint4_bf16* x, const int8_t* w_int8,
                                 const float* row_scale, const tint4_bf16* bias, tint4_bf16* y,
                                 int M, int N, int K, int group, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    return w8a8_linear_impl<false>(x, w_int8, row_scale, bias, y, M, N, K, group, workspace,
                                   workspace_bytes, stream);
}

tint4_status convrot_w8a8_linear_f16(const tint4_bf16* x, const int8_t* w_int8,
                                     const tint4_f16* row_scale, const tint4_bf16* bias,
                                     tint4_bf16* y, int M, int N, int K, int group, void* workspace,
                                     size_t workspace_bytes, void* stream) {
    return w8a8_linear_impl<true>(x, w_int8, row_scale, bias, y, M, N, K, group, workspace,
                                  workspace_bytes, stream);
}

tint4_status convrot_w4a8_linear_noalloc(const tint4_bf16* x, const uint8_t* w_packed,
                                         const float* row_scale, const tint4_bf16* bias,
                                         tint4_bf16* y, int M, int N, int K, int group,
                                         void* stream) {
    tint4_status s = check_mnk(M, N, K);
    if (s != TINT4_OK) return s;
    if ((s = check_rq_shape(M, K, group)) != TINT4_OK) return s;
    if (M > 0 && (!x || !w_packed || !row_scale || !y)) return TINT4_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_packed) || !aligned16(row_scale) || !aligned16(y) ||
        !aligned16(bias))
        return TINT4_ERR_MISALIGNED;
    if (convrot_linear_workspace_size(M, K, 8) > kStaticScratchBytes) return TINT4_ERR_WORKSPACE;
    int dev = 0;
    if ((s = check_device(&dev)) != TINT4_OK) return s;
    if (M == 0) return TINT4_OK;
    void* scratch = static_scratch_address(dev);
    if (scratch == nullptr) return TINT4_ERR_CUDA;
    return linear_run(8, x, w_packed, row_scale, bias, y, M, N, K, group, scratch,
                      as_stream(stream));
}

tint4_status w4a16_gemv_gemm(const tint4_bf16* x, const uint8_t* w_q, const tint4_bf16* scale,
                             const uint8_t* zero, int group, tint4_bf16* y, int M, int N, int K,
                             void* stream) {
    if (M < 0 || N < 0 || K < 0) return TINT4_ERR_INVALID_ARG;
    if (group != kW16Group) return TINT4_ERR_UNSUPPORTED_SHAPE;
    const bool small = M <= kW16SmallMaxM;
    if (M < 1 || M > kMaxTokens || N < 16 || N % 16 != 0 || K < kW16Group ||
        K % kW16Group != 0 || K > (small ? kW16MaxK : 65536))
        return TINT4_ERR_UNSUPPORTED_SHAPE;
    if (!x || !w_q || !scale || !zero || !y) return TINT4_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_q) || !aligned16(scale) || !aligned16(zero) ||
        !aligned16(y))
        return TINT4_ERR_MISALIGNED;
    tint4_status s = check_device();
    if (s != TINT4_OK) return s;
    const auto* xb = reinterpret_cast<const __nv_bfloat16*>(x);
    const auto* sb = reinterpret_cast<const __nv_bfloat16*>(scale);
    auto* yb = reinterpret_cast<__nv_bfloat16*>(y);
    cudaStream_t st = as_stream(stream);
    if (!small) return launch_w4a16_gemm(xb, w_q, sb, zero, yb, M, N, K, st);
    // 16 tokens per launch: a 17..32-token batch streams the weights twice
    for (int m0 = 0; m0 < M; m0 += kW16MaxM) {
        const int mc = std::min(kW16MaxM, M - m0);
        const __nv_bfloat16* xs = xb + static_cast<size_t>(m0) * K;
        __nv_bfloat16* ys = yb + static_cast<size_t>(m0) * N;
        s = mc <= 8 ? launch_w4a16<1>(xs, w_q, sb, zero, ys, mc, N, K, st)
                    : launch_w4a16<2>(xs, w_q, sb, zero, ys, mc, N, K, st);
        if (s != TINT4_OK) return s;
    }
    return TINT4_OK;
}

tint4_status tint4_debug_int32_gemm(const void* a, int act_bits, const uint8_t* w_packed,
                                    int32_t* acc, int M, int N, int K, void* stream) {
    if (act_bits != 8 && act_bits != 4) return TINT4_ERR_INVALID_ARG;
    tint4_status s = check_mnk(M, N, K);
    if (s != TINT4_OK) return s;
    if (M > 0 && (!a || !w_packed || !acc)) return TINT4_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(w_packed) || !aligned16(acc)) return TINT4_ERR_MISALIGNED;
    if ((s = check_device()) != TINT4_OK) return s;
    if (M == 0) return TINT4_OK;
    return act_bits == 4 ? launch_gemm<true, true>(a, w_packed, nullptr, nullptr, nullptr, acc, M,
                                                   N, K, as_stream(stream), false)
                         : launch_gemm<false, true>(a, w_packed, nullptr, nullptr, nullptr, acc,
                                                    M, N, K, as_stream(stream), false);
}

tint4_status tint4_debug_w4a8_gemm_even_odd(const int8_t* a_even_odd, const float* tok_scale,
                                            const uint8_t* w_packed, const float* row_scale,
                                            const tint4_bf16* bias, tint4_bf16* y, int M, int N,
                                            int K, void* stream) {
    tint4_status s = check_mnk(M, N, K);
    if (s != TINT4_OK) return s;
    if (!linear_codes_evod(M)) return TINT4_ERR_UNSUPPORTED_SHAPE;
    if (!a_even_odd || !tok_scale || !w_packed || !row_scale || !y) return TINT4_ERR_INVALID_ARG;
    if (!aligned16(a_even_odd) || !aligned16(tok_scale) || !aligned16(w_packed) ||
        !aligned16(row_scale) || !aligned16(y) || !aligned16(bias))
        return TINT4_ERR_MISALIGNED;
    if ((s = check_device()) != TINT4_OK) return s;
    return launch_gemm<false, false, true>(a_even_odd, w_packed, tok_scale, row_scale,
                                           reinterpret_cast<const __nv_bfloat16*>(bias), y, M, N,
                                           K, as_stream(stream), false);
}

tint4_status tint4_debug_bounded_wait(uint64_t limit_ns, void* stream) {
    if (limit_ns < 1000ull || limit_ns > 10000000000ull) return TINT4_ERR_INVALID_ARG;
    tint4_status s = check_device();
    if (s != TINT4_OK) return s;
    bounded_wait_test_kernel<<<1, 32, 0, as_stream(stream)>>>(limit_ns);
    return last_launch_status();
}

tint4_status tint4_get_device_error(void* stream) {
    tint4_status s = check_device();
    if (s != TINT4_OK) return s;
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) {
        cudaGetLastError();
        return TINT4_ERR_CUDA;
    }
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) {
        cudaGetLastError();
        return TINT4_ERR_CUDA;
    }
    if (v != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) {
            cudaGetLastError();
            return TINT4_ERR_CUDA;
        }
        return TINT4_ERR_TIMEOUT;
    }
    return TINT4_OK;
}

tint4_status tint4_set_wait_limit_ns(uint64_t limit_ns) {
    if (limit_ns < 1000ull || limit_ns > 60000000000ull) return TINT4_ERR_INVALID_ARG;
    g_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
    return TINT4_OK;
}

tint4_status tint4_set_decode_weight_prefetch(int enable) {
    if (enable != 0 && enable != 1) return TINT4_ERR_INVALID_ARG;
    g_decode_prefetch.store(enable, std::memory_order_relaxed);
    return TINT4_OK;
}

}  // extern "C"
