// mx_api.cu -- the C ABI of libmx.so (declared in include/mx.h): host-side
// argument checks, TMA descriptor encoding and kernel launches.  The kernels
// themselves live in quantize.cuh and gemm_sm100.cuh; this file is the single
// translation unit of the library.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <set>
#include <utility>

#include "mx.h"
#include "mx_common.cuh"
#include "quantize.cuh"
#include "rotate.cuh"
#include "gemm_sm100.cuh"
#include "gemm_pair_sm100.cuh"
#include "gemm_mbs_sm100.cuh"

namespace {

using namespace mx;

std::atomic<uint64_t> g_wait_limit_ns{1000000000ull};
std::atomic<int> g_skip_producer{0};
std::atomic<int> g_pair_enabled{1};
std::atomic<int> g_pdl_enabled{1};
std::atomic<int> g_max_gemm_ctas{0};  // 0: one CTA (or CTA pair) per SM pair of the device
std::atomic<int> g_fused_mode{MX_FUSED_PIPELINED};  // how mx_gemm_fused_act runs (MX_DEBUG_FUSED_MODE)
std::atomic<int> g_ksplit_mode{0};  // MX_DEBUG_K_SPLIT: 0 auto, 1 never, 2 whenever possible

// Launch attributes shared by the kernels that may overlap the previous kernel
// in the stream (they call griddep_wait() before reading any input).
int pdl_attr(cudaLaunchAttribute *a) {
    if (!g_pdl_enabled.load()) return 0;
    a->id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a->val.programmaticStreamSerializationAllowed = 1;
    return 1;
}

bool valid_fmt(int fmt) { return fmt >= 0 && fmt <= 5; }
int fmt_block(int fmt) { return (fmt == MX_NVFP4 || fmt == MX_MXFP4_MBS) ? 16 : 32; }
int fmt_bits(int fmt) {
    return (fmt == MX_MXFP4 || fmt == MX_NVFP4 || fmt == MX_MXFP4_MBS) ? 4 : (fmt == MX_MXFP6_E3M2 ? 6 : 8);
}
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
// Blocking granularity a format needs along K (MXFP4-MBS: its 128-element macro blocks).
int fmt_k_multiple(int fmt) { return fmt == MX_MXFP4_MBS ? 128 : fmt_block(fmt); }
// Scale tiles, and for MXFP4-MBS the macro mantissas after them ([rows][cols/128], padded to 16).
size_t tile_bytes(int fmt, int64_t rows, int64_t cols) {
    return (size_t)(cdiv(rows, 128) * 128 * cdiv(cols / fmt_block(fmt), 4) * 4);
}
size_t scales_bytes(int fmt, int64_t rows, int64_t cols) {
    size_t t = tile_bytes(fmt, rows, cols);
    if (fmt == MX_MXFP4_MBS) t += (size_t)(cdiv(rows * (cols / 128), 16) * 16);
    return t;
}
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mx_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MX_OK : MX_ERR_CUDA; }

mx_status last_launch() {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        fprintf(stderr, "libmx: launch failed: %s\n", cudaGetErrorString(e));
        return MX_ERR_CUDA;
    }
    return MX_OK;
}

// --- cuTensorMapEncodeTiled through the runtime's driver entry point ---------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2D uint8 tensor [rows x row_bytes] (row pitch = row_bytes), box 128 bytes x box_rows, 128-byte swizzle.
bool make_tmap_u8(CUtensorMap *m, const void *base, int64_t rows, int64_t row_bytes, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Codes of a kind::mxf8f6f4 operand as a 2D tensor of K elements per row, box
// 128 elements x box_rows, 128-byte swizzle.  Every type lands in shared memory
// as 128 bytes per row: FP8 bytes as they are; FP6 (16 codes in 12 bytes) and
// FP4 (16 codes in 8 bytes) unpacked by the copy to one 16-byte group per 16
// codes, the layout the MMA reads for these types.  The sub-byte types need a
// 32-byte aligned base, row pitches that are multiples of 32 bytes and K a
// multiple of 128 (the caller checks).
bool make_tmap_codes_f8f6f4(CUtensorMap *m, int fmt, const void *base, int64_t rows, int64_t K, int box_rows) {
    if (fmt_bits(fmt) == 8) return make_tmap_u8(m, base, rows, K, box_rows);
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const CUtensorMapDataType dt =
        fmt_bits(fmt) == 6 ? CU_TENSOR_MAP_DATA_TYPE_16U6_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(K * fmt_bits(fmt) / 8)};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) fprintf(stderr, "libmx: tensor map for format %d codes failed (%d)\n", fmt, (int)r);
    return r == CUDA_SUCCESS;
}

// Formats that kind::mxf8f6f4 multiplies (E8M0 scales on 32-element blocks),
// and their element-type codes in its instruction descriptor.
bool f8f6f4_fmt(int fmt) {
    return fmt == MX_MXFP8_E4M3 || fmt == MX_MXFP8_E5M2 || fmt == MX_MXFP4 || fmt == MX_MXFP6_E3M2;
}
uint32_t f8f6f4_type(int fmt) {
    switch (fmt) {
    case MX_MXFP8_E4M3: return kTypeE4M3;
    case MX_MXFP8_E5M2: return kTypeE5M2;
    case MX_MXFP6_E3M2: return kTypeE3M2;
    default: return kTypeE2M1;
    }
}
// Can A and B be multiplied, and on which kernel: the format's own (same
// format, 0..3) or the run-time-typed kind::mxf8f6f4 one.
bool gemm_pair_ok(int fa, int fb) {
    return (fa == fb && (fa <= MX_NVFP4 || fa == MX_MXFP4_MBS)) || (f8f6f4_fmt(fa) && f8f6f4_fmt(fb));
}
bool gemm_runtime_types(int fa, int fb) { return !(fa == fb && (fa <= MX_NVFP4 || fa == MX_MXFP4_MBS)); }
bool aligned32(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// --- quantize ------------------------------------------------------------
template <int FMT, int RULE = RULE_OCP>
mx_status launch_quantize(const uint16_t *src, int64_t M, int64_t K, int64_t ld, const mx_tensor *dst,
                          const float *g_in, float *g_out, cudaStream_t st, int g_from_amax = 0,
                          uint32_t *band_ready = nullptr, uint32_t *clear = nullptr, int n_clear = 0) {
    if (M == 0 || K == 0) return MX_OK;
    const int64_t sf_tiles_k = cdiv(K / fmt_block(FMT), 4);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cdiv(K, kQTileCols), (unsigned)cdiv(M, kQTileRows), 1);
    cfg.blockDim = dim3(kQThreads, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    cfg.attrs = attr;
    cfg.numAttrs = (unsigned)pdl_attr(&attr[0]);
    // g_from_amax == 2: a tiny NVFP4 tensor whose amax every CTA takes itself
    auto kernel = quantize_kernel<FMT, RULE>;
    if constexpr (FMT == 3) {
        if (g_from_amax == 2) kernel = quantize_kernel<FMT, RULE, true>;
    }
    if (cudaLaunchKernelEx(&cfg, kernel, src, M, K, ld, static_cast<uint8_t *>(dst->codes), dst->scales, sf_tiles_k,
                           g_in, g_out, g_from_amax, band_ready, clear, n_clear) != cudaSuccess)
        return last_launch();
    return MX_OK;
}

template <int FMT>
void launch_quantize_rht(const uint16_t *src, int64_t M, int64_t K, int64_t ld, const mx_tensor *dst,
                         const float *g_in, float *g_out, cudaStream_t st, int g_from_amax = 0) {
    const int64_t sf_tiles_k = cdiv(K / fmt_block(FMT), 4);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cdiv(K, kQTileCols), (unsigned)cdiv(M, kQTileRows), 1);
    cfg.blockDim = dim3(kQThreads, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    cfg.attrs = attr;
    cfg.numAttrs = (unsigned)pdl_attr(&attr[0]);
    cudaLaunchKernelEx(&cfg, quantize_rht_kernel<FMT>, src, M, K, ld, static_cast<uint8_t *>(dst->codes), dst->scales,
                       sf_tiles_k, g_in, g_out, g_from_amax);
}

void launch_quantize_mbs(const uint16_t *src, int64_t M, int64_t K, int64_t ld, const mx_tensor *dst, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(K / kQTileCols), (unsigned)cdiv(M, kQTileRows), 1);
    cfg.blockDim = dim3(kQThreads, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    cfg.attrs = attr;
    cfg.numAttrs = (unsigned)pdl_attr(&attr[0]);
    cudaLaunchKernelEx(&cfg, quantize_mbs_kernel, src, M, K, ld, static_cast<uint8_t *>(dst->codes), dst->scales,
                       cdiv(K / 16, 4), dst->scales + tile_bytes(MX_MXFP4_MBS, M, K));
}

// SM count of the current device, read once per device.
int num_sms() {
    constexpr int kMaxDev = 64;
    static std::atomic<int> cache[kMaxDev];
    int dev = 0;
    cudaGetDevice(&dev);
    const bool cached = dev >= 0 && dev < kMaxDev;
    int n = cached ? cache[dev].load(std::memory_order_relaxed) : 0;
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        if (cached) cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

mx_status launch_fused_reset(uint32_t *words, int n, cudaStream_t st);
mx_status launch_amax_overlapped(const uint16_t *X, int64_t M, int64_t K, int64_t ldx, float *slot, cudaStream_t st);

// amax(|src|) -> slot (float bits), then g = RU(amax / 2688) in place: the
// slot's reset, the amax pass and the conversion are kernels launched with
// programmatic serialization, each launched while its predecessor runs and
// waiting for it before it touches the slot.
mx_status nvfp4_gscale_prepass(const uint16_t *src, int64_t M, int64_t K, int64_t ld, float *slot, cudaStream_t st) {
    mx_status s = launch_fused_reset(reinterpret_cast<uint32_t *>(slot), 1, st);
    if (s != MX_OK) return s;
    s = launch_amax_overlapped(src, M, K, ld, slot, st);
    if (s != MX_OK) return s;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, 1);
    cfg.blockDim = dim3(1, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    cfg.attrs = attr;
    cfg.numAttrs = (unsigned)pdl_attr(&attr[0]);
    if (cudaLaunchKernelEx(&cfg, gscale_from_amax_kernel, slot) != cudaSuccess) return last_launch();
    return last_launch();
}

mx_status check_tensor(const mx_tensor *t, bool need_codes) {
    if (!t || !valid_fmt(t->fmt) || t->rows < 0 || t->cols < 0) return MX_ERR_INVALID_ARG;
    if (t->cols % fmt_k_multiple(t->fmt) != 0) return MX_ERR_UNSUPPORTED_SHAPE;
    if (t->rows > 0 && t->cols > 0) {
        if (need_codes && (!t->codes || !t->scales)) return MX_ERR_INVALID_ARG;
        if (!aligned16(t->codes) || !aligned16(t->scales)) return MX_ERR_MISALIGNED;
        if (t->fmt == MX_NVFP4 && !t->gscale) return MX_ERR_INVALID_ARG;
    }
    return MX_OK;
}

// --- GEMM ----------------------------------------------------------------
// bf16 [rows x cols] output (row pitch ld elements), box 32 x 32, no swizzle.
bool make_tmap_c(CUtensorMap *m, void *base, int64_t rows, int64_t cols, int64_t ld) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
    cuuint32_t box[2] = {32u, 32u};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Scale tiles as a 3D tensor of 8-byte words: [bands][sf_tiles_k][64] (one
// 512-byte tile = 64 words), box = box_chunks tiles of box_bands bands.  Reads
// past either end (a ragged K or N) return zeros.
bool make_tmap_sf(CUtensorMap *m, const uint8_t *scales, int64_t bands, int64_t sf_tiles_k, int box_chunks,
                  int box_bands) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {64u, (cuuint64_t)sf_tiles_k, (cuuint64_t)bands};
    cuuint64_t strides[2] = {512u, (cuuint64_t)(sf_tiles_k * 512)};
    cuuint32_t box[3] = {64u, (cuuint32_t)box_chunks, (cuuint32_t)box_bands};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 3, const_cast<uint8_t *>(scales), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Raise the dynamic shared memory limit of kernel fn to `bytes` on the current
// device, once per (kernel, device): the attribute belongs to the device's
// context, so a process that drives several GPUs sets it on each.
cudaError_t smem_limit_once(const void *fn, int bytes) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    static std::mutex mu;
    static std::set<std::pair<const void *, int>> done;
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({fn, dev}) != 0) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.insert({fn, dev});
    return e;
}

// The activation of a fused call: bf16 x quantized inside the GEMM kernel (see
// GemmParams::fused); A's codes and scales are its destination.
// Room for the K split's partial sums (ksplit.cuh): the fused call's
// workspace provides it when it is large enough.
struct SplitRoom {
    float *partials;   // kSplitSlots slots of 8 x slot_quads 4 KB blocks
    uint32_t *flags;   // kSplitSlots counters, zero at the start of the GEMM
    int slot_quads;
};

// How many CTA pairs of this kernel the device holds at once (0 if unknown);
// a split schedule needs every worker resident, since a finishing piece waits
// for the partial sums of other workers.
int coresident_pairs(const void *kernel, size_t smem) {
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(kernel, dev);
    const auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
    }
    cache[key] = n;
    return n;
}

// The work schedule's plan and grid for a launch (fills p.ks and the slot
// pointers): a split needs the room, no GELU (the finishing piece's epilogue
// is the plain one) and every worker resident.
void plan_split(GemmParams &p, int64_t tiles, int workers, int ranks, const SplitRoom *room) {
    const bool can = room != nullptr && p.epilogue == MX_EPI_NONE && workers * ranks <= kSplitSlots;
    // the fused call walks its tiles band-major in every mode, so that the
    // same tiles are split (and summed in the same order) whichever mode runs
    if (room != nullptr) p.band_major = 1;
    p.ks = ks_plan(tiles, workers, p.num_kt, g_ksplit_mode.load(), can);
    if (p.ks.on) {
        p.ks_partials = room->partials;
        p.ks_flags = room->flags;
        p.ks_slot_quads = room->slot_quads;
    }
}

struct FusedX {
    int mode;            // GemmParams::fused: 1 in-kernel quantize, 2 quantize kernel feeding bands
    const uint16_t *x;
    int64_t ldx;
    int x_fmt;
    int ga_from_amax;
    uint32_t *band_ready;
    uint32_t *next_item;
};

void set_fused(GemmParams &p, const FusedX *fx, const void *a_codes, const uint8_t *a_scales, int64_t M, int64_t K) {
    if (fx == nullptr) return;
    p.fused = fx->mode;
    p.band_major = 1;
    p.x = fx->x;
    p.ldx = fx->ldx;
    p.x_fmt = fx->x_fmt;
    p.x_items_k = (int)cdiv(K, kQTileCols);
    p.x_bands = (int)cdiv(M, kQTileRows);
    // items per band: four 32-row items per 128 x 128 tile in the kernel's own
    // quantize, one quantize-kernel CTA per tile otherwise
    p.x_band_target = (uint32_t)p.x_items_k * (fx->mode == 1 ? (uint32_t)kFusedQuads : 1u);
    p.x_sf_tiles_k = cdiv(K / fmt_block(fx->x_fmt), 4);
    p.xq_codes = static_cast<uint8_t *>(const_cast<void *>(a_codes));
    p.xq_scales = const_cast<uint8_t *>(a_scales);
    p.band_ready = fx->band_ready;
    p.next_item = fx->next_item;
    p.ga_from_amax = fx->ga_from_amax;
}

template <int FMT, int BN, int STAGES, int A_ROWS = kBM>
mx_status launch_gemm_t(const mx_tensor *A, const mx_tensor *B, const void *a_codes, const uint8_t *a_scales,
                        const float *ga, uint16_t *C, int64_t ldc, int epilogue, float *amax_out, cudaStream_t st,
                        const FusedX *fx, const SplitRoom *room) {
    using L = GemmSmem<FMT, BN, STAGES, A_ROWS>;
    static_assert(L::kAlloc <= kSmemLimit, "shared memory budget");
    const int64_t M = A->rows, N = B->rows, K = A->cols;
    const int64_t kbytes = K / GemmFmt<FMT>::kElemPerByte;   // shared-memory bytes of a row's K
    const int64_t sf_tiles_k = cdiv(K / fmt_block(FMT), 4);
    CUtensorMap ta, tb, tc, tsa, tsb;
    if (FMT == kGemmRuntimeTypes) {
        if (!make_tmap_codes_f8f6f4(&ta, A->fmt, a_codes, M, K, A_ROWS)) return MX_ERR_CUDA;
        if (!make_tmap_codes_f8f6f4(&tb, B->fmt, B->codes, N, K, BN)) return MX_ERR_CUDA;
    } else {
        if (!make_tmap_u8(&ta, a_codes, M, kbytes, A_ROWS)) return MX_ERR_CUDA;
        if (!make_tmap_u8(&tb, B->codes, N, kbytes, BN)) return MX_ERR_CUDA;
    }
    if (!make_tmap_sf(&tsa, a_scales, cdiv(M, 128), sf_tiles_k, kSfGroup * GemmFmt<FMT>::kChunks, 1)) return MX_ERR_CUDA;
    if (!make_tmap_sf(&tsb, B->scales, cdiv(N, 128), sf_tiles_k, kSfGroup * GemmFmt<FMT>::kChunks, L::kBBands))
        return MX_ERR_CUDA;
    const bool tma_store = (ldc % 8 == 0) && aligned16(C);
    memset(&tc, 0, sizeof(tc));
    if (tma_store && !make_tmap_c(&tc, C, M, N, ldc)) return MX_ERR_CUDA;
    if (smem_limit_once(reinterpret_cast<const void *>(gemm_kernel<FMT, BN, STAGES, A_ROWS, false>), L::kAlloc) !=
            cudaSuccess ||
        smem_limit_once(reinterpret_cast<const void *>(gemm_kernel<FMT, BN, STAGES, A_ROWS, true>), L::kAlloc) !=
            cudaSuccess)
        return MX_ERR_CUDA;
    GemmParams p{};
    p.sf_tiles_k = sf_tiles_k;
    p.C = C;
    p.ldc = ldc;
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.num_kt = (int)cdiv(kbytes, kStageKBytes);
    p.m_blocks = (int)cdiv(M, kBM);
    p.n_blocks = (int)cdiv(N, BN);
    p.ga = ga;
    p.gb = B->gscale;
    p.amax_out = amax_out;
    p.epilogue = epilogue;
    p.use_tma_store = tma_store ? 1 : 0;
    p.skip_producer = g_skip_producer.load();
    p.ab_types = (f8f6f4_type(A->fmt) << 7) | (f8f6f4_type(B->fmt) << 10);
    p.stage_tx = (uint32_t)(kStageKBytes * (A_ROWS * fmt_bits(A->fmt) + BN * fmt_bits(B->fmt)) / 8);
    p.wait_limit_ns = g_wait_limit_ns.load();
    set_fused(p, fx, a_codes, a_scales, M, K);
    const int64_t tiles = (int64_t)p.m_blocks * p.n_blocks;
    if (tiles > INT32_MAX) return MX_ERR_UNSUPPORTED_SHAPE;
    const int cap = g_max_gemm_ctas.load();
    const int max_ctas = cap > 0 && cap < num_sms() ? cap : num_sms();
    plan_split(p, tiles, max_ctas, 1, room);
    const unsigned grid = (unsigned)p.ks.workers;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = L::kAlloc;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    cfg.attrs = attr;
    cfg.numAttrs = (unsigned)pdl_attr(&attr[0]);
    // the kernel compiled for the split runs only when the plan splits
    const auto kern = p.ks.on ? gemm_kernel<FMT, BN, STAGES, A_ROWS, true> : gemm_kernel<FMT, BN, STAGES, A_ROWS, false>;
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb, tc, tsa, tsb, p) != cudaSuccess) return last_launch();
    return last_launch();
}

// CTA-pair kernel: 256 x BN tiles on clusters of two CTAs (M > 128).
template <int FMT, int STAGES, int BN = 256>
mx_status launch_gemm_pair_t(const mx_tensor *A, const mx_tensor *B, const void *a_codes, const uint8_t *a_scales,
                             const float *ga, uint16_t *C, int64_t ldc, int epilogue, float *amax_out,
                             cudaStream_t st, const FusedX *fx, const SplitRoom *room) {
    using L = PairSmem<FMT, STAGES, BN>;
    static_assert(L::kAlloc <= kSmemLimit, "shared memory budget");
    const int64_t M = A->rows, N = B->rows, K = A->cols;
    const int64_t kbytes = K / GemmFmt<FMT>::kElemPerByte;   // shared-memory bytes of a row's K
    const int64_t sf_tiles_k = cdiv(K / fmt_block(FMT), 4);
    CUtensorMap ta, tb, tc, tsa, tsb;
    if (FMT == kGemmRuntimeTypes) {
        if (!make_tmap_codes_f8f6f4(&ta, A->fmt, a_codes, M, K, 128)) return MX_ERR_CUDA;
        if (!make_tmap_codes_f8f6f4(&tb, B->fmt, B->codes, N, K, BN / 2)) return MX_ERR_CUDA;
    } else {
        if (!make_tmap_u8(&ta, a_codes, M, kbytes, 128)) return MX_ERR_CUDA;
        if (!make_tmap_u8(&tb, B->codes, N, kbytes, BN / 2)) return MX_ERR_CUDA;
    }
    if (!make_tmap_sf(&tsa, a_scales, cdiv(M, 128), sf_tiles_k, kSfGroup * GemmFmt<FMT>::kChunks, 1)) return MX_ERR_CUDA;
    if (!make_tmap_sf(&tsb, B->scales, cdiv(N, 128), sf_tiles_k, kSfGroup * GemmFmt<FMT>::kChunks, BN / 128))
        return MX_ERR_CUDA;
    const bool tma_store = (ldc % 8 == 0) && aligned16(C);
    memset(&tc, 0, sizeof(tc));
    if (tma_store && !make_tmap_c(&tc, C, M, N, ldc)) return MX_ERR_CUDA;
    // only the 256-wide tiles (no GELU) have a variant compiled for the split
    constexpr bool kCanSplit = BN == 256;
    using Kern = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, GemmParams);
    const Kern kern_whole = gemm_pair_kernel<FMT, STAGES, BN, false>;
    const Kern kern_split = kCanSplit ? gemm_pair_kernel<FMT, STAGES, BN, kCanSplit> : kern_whole;
    if (smem_limit_once(reinterpret_cast<const void *>(kern_whole), L::kAlloc) != cudaSuccess ||
        smem_limit_once(reinterpret_cast<const void *>(kern_split), L::kAlloc) != cudaSuccess)
        return MX_ERR_CUDA;
    GemmParams p{};
    p.sf_tiles_k = sf_tiles_k;
    p.C = C;
    p.ldc = ldc;
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.num_kt = (int)cdiv(kbytes, kStageKBytes);
    p.m_blocks = (int)cdiv(M, 256);
    p.n_blocks = (int)cdiv(N, BN);
    p.ga = ga;
    p.gb = B->gscale;
    p.amax_out = amax_out;
    p.epilogue = epilogue;
    p.use_tma_store = tma_store ? 1 : 0;
    p.skip_producer = g_skip_producer.load();
    p.ab_types = (f8f6f4_type(A->fmt) << 7) | (f8f6f4_type(B->fmt) << 10);
    // both CTAs' copies (128 rows of A and BN/2 of B each) report to the leader's barrier
    p.stage_tx = (uint32_t)(2 * kStageKBytes * (128 * fmt_bits(A->fmt) + (BN / 2) * fmt_bits(B->fmt)) / 8);
    p.wait_limit_ns = g_wait_limit_ns.load();
    set_fused(p, fx, a_codes, a_scales, M, K);
    const int64_t tiles = (int64_t)p.m_blocks * p.n_blocks;
    if (tiles > INT32_MAX) return MX_ERR_UNSUPPORTED_SHAPE;
    const int cap = g_max_gemm_ctas.load();
    const int max_pairs = cap > 0 && cap < num_sms() ? (cap + 1) / 2 : num_sms() / 2;
    // a split plan runs only on pairs that are all resident at once
    const int resident =
        room != nullptr && kCanSplit ? coresident_pairs(reinterpret_cast<const void *>(kern_split), L::kAlloc) : 0;
    plan_split(p, tiles, resident > 0 && resident < max_pairs ? resident : max_pairs, 2, resident > 0 ? room : nullptr);
    if (!p.ks.on) p.ks = ks_plan(tiles, max_pairs, p.num_kt, 1, false);
    const unsigned pairs = (unsigned)p.ks.workers;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = L::kAlloc;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1 + (unsigned)pdl_attr(&attr[1]);
    if (cudaLaunchKernelEx(&cfg, p.ks.on ? kern_split : kern_whole, ta, tb, tc, tsa, tsb, p) != cudaSuccess)
        return last_launch();
    return last_launch();
}

template <int FMT>
mx_status launch_gemm_fmt(const mx_tensor *A, const mx_tensor *B, const void *a_codes, const uint8_t *a_scales,
                          const float *ga, uint16_t *C, int64_t ldc, int epi, float *amax_out, cudaStream_t st,
                          const FusedX *fx, const SplitRoom *room) {
    if (A->rows > 128 && B->rows > 128 && g_pair_enabled.load()) {
        // GELU: 256 x 128 tiles, whose two accumulators need no shared TMEM
        // columns, so each tile's GELU drain overlaps the next tile's MMAs
        if (epi == MX_EPI_GELU)
            return launch_gemm_pair_t<FMT, 7, 128>(A, B, a_codes, a_scales, ga, C, ldc, epi, amax_out, st, fx, room);
        return launch_gemm_pair_t<FMT, (FMT == 2 || FMT == 3) ? 5 : 6>(A, B, a_codes, a_scales, ga, C, ldc, epi,
                                                                       amax_out, st, fx, room);
    }
    if (B->rows <= 128)
        return launch_gemm_t<FMT, 128, 4>(A, B, a_codes, a_scales, ga, C, ldc, epi, amax_out, st, fx, room);
    // at most 32 rows of A (decode-like activations): the weight stream gets a
    // fifth stage from the shared memory a 128-row A tile would take
    if (A->rows <= 32)
        return launch_gemm_t<FMT, 256, 5, 32>(A, B, a_codes, a_scales, ga, C, ldc, epi, amax_out, st, fx, room);
    return launch_gemm_t<FMT, 256, 4>(A, B, a_codes, a_scales, ga, C, ldc, epi, amax_out, st, fx, room);
}

mx_status launch_gemm(const mx_tensor *A, const mx_tensor *B, const void *a_codes, const uint8_t *a_scales,
                      const float *ga, uint16_t *C, int64_t ldc, int epi, float *amax_out, cudaStream_t st,
                      const FusedX *fx = nullptr, const SplitRoom *room = nullptr) {
    if (gemm_runtime_types(A->fmt, B->fmt))
        return launch_gemm_fmt<kGemmRuntimeTypes>(A, B, a_codes, a_scales, ga, C, ldc, epi, amax_out, st, fx, room);
    switch (A->fmt) {
    case MX_MXFP8_E4M3: return launch_gemm_fmt<0>(A, B, a_codes, a_scales, ga, C, ldc, epi, amax_out, st, fx, room);
    case MX_MXFP8_E5M2: return launch_gemm_fmt<1>(A, B, a_codes, a_scales, ga, C, ldc, epi, amax_out, st, fx, room);
    case MX_MXFP4: return launch_gemm_fmt<2>(A, B, a_codes, a_scales, ga, C, ldc, epi, amax_out, st, fx, room);
    default: return launch_gemm_fmt<3>(A, B, a_codes, a_scales, ga, C, ldc, epi, amax_out, st, fx, room);
    }
}

// MXFP4-MBS x MXFP4-MBS (gemm_mbs_sm100.cuh): one CTA per 128 x 128 tile.
mx_status launch_gemm_mbs(const mx_tensor *A, const mx_tensor *B, uint16_t *C, int64_t ldc, cudaStream_t st) {
    using L = MbsLayout;
    const int64_t M = A->rows, N = B->rows, K = A->cols;
    const int64_t kbytes = K / 2;
    const int64_t sf_tiles_k = cdiv(K / 16, 4);
    CUtensorMap ta, tb, tsa, tsb;
    if (!make_tmap_u8(&ta, A->codes, M, kbytes, 128)) return MX_ERR_CUDA;
    if (!make_tmap_u8(&tb, B->codes, N, kbytes, 128)) return MX_ERR_CUDA;
    if (!make_tmap_sf(&tsa, A->scales, cdiv(M, 128), sf_tiles_k, 4, 1)) return MX_ERR_CUDA;
    if (!make_tmap_sf(&tsb, B->scales, cdiv(N, 128), sf_tiles_k, 4, 1)) return MX_ERR_CUDA;
    if (smem_limit_once(reinterpret_cast<const void *>(gemm_mbs_kernel), L::kAlloc) != cudaSuccess)
        return MX_ERR_CUDA;
    MbsParams p{};
    p.C = C;
    p.ldc = ldc;
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.num_kt = (int)cdiv(kbytes, kStageKBytes);
    p.n_macro = (int)(K / 128);
    p.m_blocks = (int)cdiv(M, 128);
    p.macro_a = A->scales + tile_bytes(MX_MXFP4_MBS, M, K);
    p.macro_b = B->scales + tile_bytes(MX_MXFP4_MBS, N, K);
    p.vec_store = (ldc % 8 == 0) && aligned16(C) ? 1 : 0;
    p.skip_producer = g_skip_producer.load();
    p.wait_limit_ns = g_wait_limit_ns.load();
    const int64_t tiles = (int64_t)p.m_blocks * cdiv(N, kMbsBN);
    if (tiles > INT32_MAX) return MX_ERR_UNSUPPORTED_SHAPE;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)tiles, 1, 1);
    cfg.blockDim = dim3(kMbsThreads, 1, 1);
    cfg.dynamicSmemBytes = L::kAlloc;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    cfg.attrs = attr;
    cfg.numAttrs = (unsigned)pdl_attr(&attr[0]);
    if (cudaLaunchKernelEx(&cfg, gemm_mbs_kernel, ta, tb, tsa, tsb, p) != cudaSuccess) return last_launch();
    return last_launch();
}

// The fused call's workspace: a header, then X's codes and scales, then
// (optional) the K split's partial-sum slots, each starting on a 256-byte
// boundary.  Header words: [0] g of X (NVFP4), [1] amax(|X|) of the pre-pass,
// [2] the fused kernel's work counter, [3] unused, [16 ..] one ready counter
// per 128-row band of X, then kSplitSlots counters of the partial-sum slots.
constexpr size_t kWsBandOffset = 64;
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
size_t fused_ws_flags(int64_t M) { return kWsBandOffset + 4 * (size_t)cdiv(M, 128); }
size_t fused_ws_header(int64_t M) { return align256(fused_ws_flags(M) + 4 * (size_t)kSplitSlots); }
size_t fused_ws_bytes(int fmt, int64_t M, int64_t K) {
    return fused_ws_header(M) + align256((size_t)(M * K * fmt_bits(fmt) / 8)) + align256(scales_bytes(fmt, M, K));
}
// 32-row quadrants of a partial-sum slot: those of a CTA's accumulator rows
// that exist (a slot holds 8 column chunks of 4 KB per quadrant)
size_t fused_split_quads(int64_t M) { return (size_t)(M < 128 ? cdiv(M, 32) : 4); }
size_t fused_ws_split_bytes(int fmt, int64_t M, int64_t K) {
    return fused_ws_bytes(fmt, M, K) + (size_t)kSplitSlots * 8 * fused_split_quads(M) * 4096;
}

// Zero the fused kernel's counters (the work counter and the band counters).
// Launched with programmatic stream serialization: it lets the GEMM that follows
// start its setup at once, and clears the counters only after the previous
// kernel in the stream (which may be a fused GEMM on the same workspace) has
// completed; the GEMM reads them only after this kernel has completed.
__global__ void fused_reset_kernel(uint32_t *__restrict__ words, int n) {
    griddep_launch_dependents();
    griddep_wait();
    for (int i = threadIdx.x; i < n; i += blockDim.x) words[i] = 0u;
}

mx_status launch_fused_reset(uint32_t *words, int n, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, 1);
    cfg.blockDim = dim3(128, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    cfg.attrs = attr;
    cfg.numAttrs = (unsigned)pdl_attr(&attr[0]);
    if (cudaLaunchKernelEx(&cfg, fused_reset_kernel, words, n) != cudaSuccess) return last_launch();
    return MX_OK;
}

// amax(|X|) into *slot by the persistent amax kernel, launched to overlap the
// previous kernel in the stream (the counter reset that zeroed the slot).
mx_status launch_amax_overlapped(const uint16_t *X, int64_t M, int64_t K, int64_t ldx, float *slot, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)amax_grid(M, K, num_sms()), 1, 1);
    cfg.blockDim = dim3(kQThreads, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    cfg.attrs = attr;
    cfg.numAttrs = (unsigned)pdl_attr(&attr[0]);
    if (cudaLaunchKernelEx(&cfg, amax_kernel, X, M, K, ldx, reinterpret_cast<unsigned int *>(slot)) != cudaSuccess)
        return last_launch();
    return MX_OK;
}

// Quantize X into the workspace as the A operand of the GEMM.  Returns the
// device pointer of X's g (NVFP4) through *ga.
mx_status fused_quantize_x(int fmt, const uint16_t *X, int64_t M, int64_t K, int64_t ldx, uint8_t *ws,
                           const float *x_gscale, const float *x_amax, mx_tensor *xa, const float **ga,
                           cudaStream_t st, uint32_t *band_ready = nullptr, uint32_t *clear = nullptr,
                           int n_clear = 0) {
    float *g_slot = reinterpret_cast<float *>(ws);
    float *amax_slot = reinterpret_cast<float *>(ws + 4);
    xa->fmt = fmt;
    xa->reserved = 0;
    xa->rows = M;
    xa->cols = K;
    xa->codes = ws + fused_ws_header(M);
    xa->scales = ws + fused_ws_header(M) + align256((size_t)(M * K * fmt_bits(fmt) / 8));
    xa->gscale = g_slot;
    *ga = nullptr;
    mx_status s = MX_OK;
    switch (fmt) {
    case MX_MXFP8_E4M3: s = launch_quantize<0>(X, M, K, ldx, xa, nullptr, nullptr, st, 0, band_ready, clear, n_clear); break;
    case MX_MXFP8_E5M2: s = launch_quantize<1>(X, M, K, ldx, xa, nullptr, nullptr, st, 0, band_ready, clear, n_clear); break;
    case MX_MXFP4: s = launch_quantize<2>(X, M, K, ldx, xa, nullptr, nullptr, st, 0, band_ready, clear, n_clear); break;
    case MX_MXFP6_E3M2: s = launch_quantize<4>(X, M, K, ldx, xa, nullptr, nullptr, st, 0, band_ready, clear, n_clear); break;
    default:
        if (x_gscale != nullptr) {
            s = launch_quantize<3>(X, M, K, ldx, xa, x_gscale, nullptr, st, 0, band_ready, clear, n_clear);
            *ga = x_gscale;
        } else {
            const float *amax = x_amax;
            if (amax == nullptr && M * K <= kTinyAmaxElements) {
                // a tiny X: each quantize CTA takes amax(|X|) itself, no pre-pass
                s = launch_quantize<3>(X, M, K, ldx, xa, nullptr, g_slot, st, /*g_from_amax=*/2, band_ready, clear,
                                       n_clear);
                *ga = g_slot;
                if (s != MX_OK) return s;
                return last_launch();
            }
            if (amax == nullptr) {
                // the amax pre-pass into the header's slot, zeroed by a one-block
                // kernel just before it (both overlap their predecessors' tails)
                s = launch_fused_reset(reinterpret_cast<uint32_t *>(amax_slot), 1, st);
                if (s != MX_OK) return s;
                s = launch_amax_overlapped(X, M, K, ldx, amax_slot, st);
                if (s != MX_OK) return s;
                amax = amax_slot;
            }
            s = launch_quantize<3>(X, M, K, ldx, xa, amax, g_slot, st, /*g_from_amax=*/1, band_ready, clear, n_clear);
            *ga = g_slot;
        }
    }
    if (s != MX_OK) return s;
    return last_launch();
}

}  // namespace

extern "C" {

size_t mx_codes_bytes(int fmt, int64_t rows, int64_t cols) {
    if (!valid_fmt(fmt) || rows < 0 || cols < 0) return 0;
    return (size_t)(rows * cols * fmt_bits(fmt) / 8);
}

size_t mx_scales_bytes(int fmt, int64_t rows, int64_t cols) {
    if (!valid_fmt(fmt) || rows < 0 || cols < 0) return 0;
    return scales_bytes(fmt, rows, cols);
}

int mx_block_size(int fmt) { return valid_fmt(fmt) ? fmt_block(fmt) : 0; }

int mx_version(void) { return 100; }

const char *mx_status_string(mx_status s) {
    switch (s) {
    case MX_OK: return "MX_OK";
    case MX_ERR_INVALID_ARG: return "MX_ERR_INVALID_ARG";
    case MX_ERR_UNSUPPORTED_SHAPE: return "MX_ERR_UNSUPPORTED_SHAPE";
    case MX_ERR_MISALIGNED: return "MX_ERR_MISALIGNED";
    case MX_ERR_CUDA: return "MX_ERR_CUDA";
    case MX_ERR_TIMEOUT: return "MX_ERR_TIMEOUT";
    case MX_ERR_DEVICE: return "MX_ERR_DEVICE";
    }
    return "MX_ERR_UNKNOWN";
}

mx_status mx_debug_set(int key, uint64_t value) {
    switch (key) {
    case MX_DEBUG_WAIT_LIMIT_NS: g_wait_limit_ns.store(value ? value : 1); return MX_OK;
    case MX_DEBUG_SKIP_PRODUCER: g_skip_producer.store(value ? 1 : 0); return MX_OK;
    case MX_DEBUG_PAIR_GEMM: g_pair_enabled.store(value ? 1 : 0); return MX_OK;
    case MX_DEBUG_OVERLAP_LAUNCH: g_pdl_enabled.store(value ? 1 : 0); return MX_OK;
    case MX_DEBUG_MAX_GEMM_CTAS: g_max_gemm_ctas.store(value > 65535 ? 0 : (int)value); return MX_OK;
    case MX_DEBUG_FUSED_MODE:
        if (value > MX_FUSED_TWO_KERNELS) return MX_ERR_INVALID_ARG;
        g_fused_mode.store((int)value);
        return MX_OK;
    case MX_DEBUG_K_SPLIT:
        if (value > MX_K_SPLIT_ALWAYS) return MX_ERR_INVALID_ARG;
        g_ksplit_mode.store((int)value);
        return MX_OK;
    default: return MX_ERR_INVALID_ARG;
    }
}

mx_status mx_quantize(int fmt, const void *src_bf16, int64_t M, int64_t K, int64_t ld_src, mx_tensor *dst,
                      const float *gscale_in, void *stream) {
    if (!valid_fmt(fmt) || !dst || M < 0 || K < 0) return MX_ERR_INVALID_ARG;
    if (dst->fmt != fmt || dst->rows != M || dst->cols != K) return MX_ERR_INVALID_ARG;
    if (K % fmt_k_multiple(fmt) != 0) return MX_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || K == 0) return MX_OK;
    if (!src_bf16 || !dst->codes || !dst->scales) return MX_ERR_INVALID_ARG;
    if (fmt == MX_NVFP4 && !dst->gscale) return MX_ERR_INVALID_ARG;
    if (ld_src < K || (ld_src & 7) != 0) return MX_ERR_MISALIGNED;
    if (!aligned16(src_bf16) || !aligned16(dst->codes) || !aligned16(dst->scales)) return MX_ERR_MISALIGNED;
    if (cdiv(M, kQTileRows) > 65535) return MX_ERR_UNSUPPORTED_SHAPE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const uint16_t *src = static_cast<const uint16_t *>(src_bf16);
    mx_status s = MX_OK;
    switch (fmt) {
    case MX_MXFP8_E4M3: s = launch_quantize<0>(src, M, K, ld_src, dst, nullptr, nullptr, st); break;
    case MX_MXFP8_E5M2: s = launch_quantize<1>(src, M, K, ld_src, dst, nullptr, nullptr, st); break;
    case MX_MXFP4: s = launch_quantize<2>(src, M, K, ld_src, dst, nullptr, nullptr, st); break;
    case MX_MXFP6_E3M2: s = launch_quantize<4>(src, M, K, ld_src, dst, nullptr, nullptr, st); break;
    case MX_MXFP4_MBS: launch_quantize_mbs(src, M, K, ld_src, dst, st); break;
    default: {
        if (gscale_in == nullptr && M * K <= kTinyAmaxElements) {
            // a tiny tensor: each CTA takes amax(|src|) itself, no pre-pass
            s = launch_quantize<3>(src, M, K, ld_src, dst, nullptr, dst->gscale, st, /*g_from_amax=*/2);
        } else if (gscale_in == nullptr) {
            s = nvfp4_gscale_prepass(src, M, K, ld_src, dst->gscale, st);
            if (s != MX_OK) return s;
            s = launch_quantize<3>(src, M, K, ld_src, dst, dst->gscale, nullptr, st);
        } else {
            s = launch_quantize<3>(src, M, K, ld_src, dst, gscale_in, gscale_in == dst->gscale ? nullptr : dst->gscale,
                                   st);
        }
    }
    }
    if (s != MX_OK) return s;
    return last_launch();
}

mx_status mx_quantize_oas(const void *src_bf16, int64_t M, int64_t K, int64_t ld_src, mx_tensor *dst, void *stream) {
    if (!dst || dst->fmt != MX_MXFP4 || M < 0 || K < 0) return MX_ERR_INVALID_ARG;
    if (dst->rows != M || dst->cols != K) return MX_ERR_INVALID_ARG;
    if (K % 32 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || K == 0) return MX_OK;
    if (!src_bf16 || !dst->codes || !dst->scales) return MX_ERR_INVALID_ARG;
    if (ld_src < K || (ld_src & 7) != 0) return MX_ERR_MISALIGNED;
    if (!aligned16(src_bf16) || !aligned16(dst->codes) || !aligned16(dst->scales)) return MX_ERR_MISALIGNED;
    if (cdiv(M, kQTileRows) > 65535) return MX_ERR_UNSUPPORTED_SHAPE;
    const mx_status s = launch_quantize<2, RULE_OAS>(static_cast<const uint16_t *>(src_bf16), M, K, ld_src, dst,
                                                     nullptr, nullptr, static_cast<cudaStream_t>(stream));
    if (s != MX_OK) return s;
    return last_launch();
}

mx_status mx_quantize_mbs_dynamic(const void *src_bf16, int64_t M, int64_t K, int64_t ld_src, mx_tensor *dst,
                                  void *stream) {
    if (!dst || dst->fmt != MX_MXFP4_MBS || M < 0 || K < 0) return MX_ERR_INVALID_ARG;
    if (dst->rows != M || dst->cols != K) return MX_ERR_INVALID_ARG;
    if (K % 128 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || K == 0) return MX_OK;
    if (!src_bf16 || !dst->codes || !dst->scales) return MX_ERR_INVALID_ARG;
    if (ld_src < K || (ld_src & 7) != 0) return MX_ERR_MISALIGNED;
    if (!aligned16(src_bf16) || !aligned16(dst->codes) || !aligned16(dst->scales)) return MX_ERR_MISALIGNED;
    if (M > 65535 || K / 128 > INT32_MAX) return MX_ERR_UNSUPPORTED_SHAPE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // padding bytes of the scale tiles and of the macro section stay zero
    if (cudaMemsetAsync(dst->scales, 0, scales_bytes(MX_MXFP4_MBS, M, K), st) != cudaSuccess) return MX_ERR_CUDA;
    quantize_mbs_dynamic_kernel<<<dim3((unsigned)(K / 128), (unsigned)M, 1), 256, 0, st>>>(
        static_cast<const uint16_t *>(src_bf16), M, K, ld_src, static_cast<uint8_t *>(dst->codes), dst->scales,
        cdiv(K / 16, 4), dst->scales + tile_bytes(MX_MXFP4_MBS, M, K));
    return last_launch();
}

mx_status mx_quantize_rht(int fmt, const void *src_bf16, int64_t M, int64_t K, int64_t ld_src, mx_tensor *dst,
                          const float *gscale_in, void *stream) {
    if (!valid_fmt(fmt) || fmt == MX_MXFP4_MBS || !dst || M < 0 || K < 0) return MX_ERR_INVALID_ARG;
    if (dst->fmt != fmt || dst->rows != M || dst->cols != K) return MX_ERR_INVALID_ARG;
    if (K % 32 != 0) return MX_ERR_UNSUPPORTED_SHAPE;   // rotation blocks of 32
    if (M == 0 || K == 0) return MX_OK;
    if (!src_bf16 || !dst->codes || !dst->scales) return MX_ERR_INVALID_ARG;
    if (fmt == MX_NVFP4 && !dst->gscale) return MX_ERR_INVALID_ARG;
    if (ld_src < K || (ld_src & 7) != 0) return MX_ERR_MISALIGNED;
    if (!aligned16(src_bf16) || !aligned16(dst->codes) || !aligned16(dst->scales)) return MX_ERR_MISALIGNED;
    if (cdiv(M, kQTileRows) > 65535) return MX_ERR_UNSUPPORTED_SHAPE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const uint16_t *src = static_cast<const uint16_t *>(src_bf16);
    switch (fmt) {
    case MX_MXFP8_E4M3: launch_quantize_rht<0>(src, M, K, ld_src, dst, nullptr, nullptr, st); break;
    case MX_MXFP8_E5M2: launch_quantize_rht<1>(src, M, K, ld_src, dst, nullptr, nullptr, st); break;
    case MX_MXFP4: launch_quantize_rht<2>(src, M, K, ld_src, dst, nullptr, nullptr, st); break;
    case MX_MXFP6_E3M2: launch_quantize_rht<4>(src, M, K, ld_src, dst, nullptr, nullptr, st); break;
    default: {
        if (gscale_in == nullptr) {
            // g from max |y| of the rotated tensor: an extra read of src
            if (cudaMemsetAsync(dst->gscale, 0, sizeof(float), st) != cudaSuccess) return MX_ERR_CUDA;
            const int64_t pairs = M * (K / 32);
            int64_t blocks = cdiv(pairs * 2, 256);
            const int64_t cap = (int64_t)num_sms() * 8;
            if (blocks > cap) blocks = cap;
            if (blocks < 1) blocks = 1;
            amax_rht_kernel<<<(unsigned)blocks, 256, 0, st>>>(src, M, K, ld_src,
                                                              reinterpret_cast<unsigned int *>(dst->gscale));
            gscale_from_amax_kernel<<<1, 1, 0, st>>>(dst->gscale);
            launch_quantize_rht<3>(src, M, K, ld_src, dst, dst->gscale, nullptr, st);
        } else {
            launch_quantize_rht<3>(src, M, K, ld_src, dst, gscale_in,
                                   gscale_in == dst->gscale ? nullptr : dst->gscale, st);
        }
    }
    }
    return last_launch();
}

mx_status mx_qsnr(const mx_tensor *q, const void *src_bf16, int64_t ld_src, double *sums, void *stream) {
    mx_status s = check_tensor(q, true);
    if (s != MX_OK) return s;
    if (!sums) return MX_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(sums) & 7u) != 0) return MX_ERR_MISALIGNED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(sums, 0, 2 * sizeof(double), st) != cudaSuccess) return MX_ERR_CUDA;
    if (q->rows == 0 || q->cols == 0) return MX_OK;
    if (!src_bf16) return MX_ERR_INVALID_ARG;
    if (ld_src < q->cols || (ld_src & 7) != 0 || !aligned16(src_bf16)) return MX_ERR_MISALIGNED;
    const int64_t n = q->rows * (q->cols / 8);
    int64_t blocks = cdiv(n, 256);
    const int64_t cap = (int64_t)num_sms() * 8;
    if (blocks > cap) blocks = cap;
    const uint16_t *x = static_cast<const uint16_t *>(src_bf16);
    const uint8_t *c = static_cast<const uint8_t *>(q->codes);
    const unsigned b = (unsigned)blocks;
    const uint8_t *mac = q->scales + tile_bytes(q->fmt, q->rows, q->cols);   // MXFP4-MBS only
    switch (q->fmt) {
    case MX_MXFP8_E4M3: qsnr_kernel<0><<<b, 256, 0, st>>>(x, ld_src, c, q->scales, nullptr, nullptr, q->rows, q->cols, sums); break;
    case MX_MXFP8_E5M2: qsnr_kernel<1><<<b, 256, 0, st>>>(x, ld_src, c, q->scales, nullptr, nullptr, q->rows, q->cols, sums); break;
    case MX_MXFP4: qsnr_kernel<2><<<b, 256, 0, st>>>(x, ld_src, c, q->scales, nullptr, nullptr, q->rows, q->cols, sums); break;
    case MX_MXFP6_E3M2: qsnr_kernel<4><<<b, 256, 0, st>>>(x, ld_src, c, q->scales, nullptr, nullptr, q->rows, q->cols, sums); break;
    case MX_MXFP4_MBS: qsnr_kernel<5><<<b, 256, 0, st>>>(x, ld_src, c, q->scales, nullptr, mac, q->rows, q->cols, sums); break;
    default: qsnr_kernel<3><<<b, 256, 0, st>>>(x, ld_src, c, q->scales, q->gscale, nullptr, q->rows, q->cols, sums);
    }
    return last_launch();
}

mx_status mx_dequantize(const mx_tensor *src, void *dst_bf16, int64_t ld_dst, void *stream) {
    mx_status s = check_tensor(src, true);
    if (s != MX_OK) return s;
    if (src->rows == 0 || src->cols == 0) return MX_OK;
    if (!dst_bf16) return MX_ERR_INVALID_ARG;
    if (ld_dst < src->cols || (ld_dst & 7) != 0 || !aligned16(dst_bf16)) return MX_ERR_MISALIGNED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t n = src->rows * (src->cols / 8);
    const unsigned blocks = (unsigned)cdiv(n, 256);
    const uint8_t *c = static_cast<const uint8_t *>(src->codes);
    uint16_t *d = static_cast<uint16_t *>(dst_bf16);
    const uint8_t *mac = src->scales + tile_bytes(src->fmt, src->rows, src->cols);   // MXFP4-MBS only
    switch (src->fmt) {
    case MX_MXFP8_E4M3: dequantize_kernel<0><<<blocks, 256, 0, st>>>(c, src->scales, nullptr, nullptr, src->rows, src->cols, d, ld_dst); break;
    case MX_MXFP8_E5M2: dequantize_kernel<1><<<blocks, 256, 0, st>>>(c, src->scales, nullptr, nullptr, src->rows, src->cols, d, ld_dst); break;
    case MX_MXFP4: dequantize_kernel<2><<<blocks, 256, 0, st>>>(c, src->scales, nullptr, nullptr, src->rows, src->cols, d, ld_dst); break;
    case MX_MXFP6_E3M2: dequantize_kernel<4><<<blocks, 256, 0, st>>>(c, src->scales, nullptr, nullptr, src->rows, src->cols, d, ld_dst); break;
    case MX_MXFP4_MBS: dequantize_kernel<5><<<blocks, 256, 0, st>>>(c, src->scales, nullptr, mac, src->rows, src->cols, d, ld_dst); break;
    default: dequantize_kernel<3><<<blocks, 256, 0, st>>>(c, src->scales, src->gscale, nullptr, src->rows, src->cols, d, ld_dst);
    }
    return last_launch();
}

mx_status mx_gemm(const mx_tensor *A, const mx_tensor *B, void *C_bf16, int64_t ldc, void *stream) {
    mx_status s = check_tensor(A, true);
    if (s != MX_OK) return s;
    s = check_tensor(B, true);
    if (s != MX_OK) return s;
    if (!gemm_pair_ok(A->fmt, B->fmt) || A->cols != B->cols) return MX_ERR_INVALID_ARG;
    const int64_t M = A->rows, N = B->rows, K = A->cols;
    if (M == 0 || N == 0) return MX_OK;
    if (!C_bf16) return MX_ERR_INVALID_ARG;
    if (ldc < N) return MX_ERR_INVALID_ARG;
    if (!aligned16(C_bf16)) return MX_ERR_MISALIGNED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (K == 0) return cuda_status(cudaMemset2DAsync(C_bf16, ldc * 2, 0, N * 2, M, st));
    if (K % 128 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
    if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX || cdiv(M, kBM) > 65535) return MX_ERR_UNSUPPORTED_SHAPE;
    if (gemm_runtime_types(A->fmt, B->fmt) && ((fmt_bits(A->fmt) < 8 && !aligned32(A->codes)) ||
                                               (fmt_bits(B->fmt) < 8 && !aligned32(B->codes))))
        return MX_ERR_MISALIGNED;
    if (A->fmt == MX_MXFP4_MBS) return launch_gemm_mbs(A, B, static_cast<uint16_t *>(C_bf16), ldc, st);
    return launch_gemm(A, B, A->codes, A->scales, A->gscale, static_cast<uint16_t *>(C_bf16), ldc, 0, nullptr, st,
                       nullptr);
}

size_t mx_fused_workspace_bytes(int fmt, int64_t M, int64_t K) {
    if (!valid_fmt(fmt) || M < 0 || K < 0 || M > INT32_MAX || K > INT32_MAX) return 0;
    return fused_ws_bytes(fmt, M, K);
}

size_t mx_fused_split_workspace_bytes(int fmt, int64_t M, int64_t K) {
    if (!valid_fmt(fmt) || M < 0 || K < 0 || M > INT32_MAX || K > INT32_MAX) return 0;
    return fused_ws_split_bytes(fmt, M, K);
}

int mx_debug_split_units(int64_t tiles, int workers, int kt, int mode, int worker, int32_t *out, int max_units,
                         int *n_workers) {
    if (tiles < 0 || tiles > INT32_MAX || workers < 1 || kt < 1 || mode < 0 || mode > MX_K_SPLIT_ALWAYS || worker < 0)
        return -1;
    const KSplitPlan plan = ks_plan(tiles, workers, kt, mode, true);
    if (n_workers) *n_workers = plan.workers;
    if (worker >= plan.workers) return 0;
    const int n = ks_units(plan, worker);
    for (int u = 0; u < n && u < max_units && out; ++u) {
        const KUnit x = ks_unit(plan, worker, u);
        out[5 * u] = x.tile;
        out[5 * u + 1] = x.kb;
        out[5 * u + 2] = x.ke;
        out[5 * u + 3] = x.kind;
        out[5 * u + 4] = x.first;
    }
    return n;
}

mx_status mx_gemm_fused_act(int fmt, const void *X_bf16, int64_t M, int64_t K, int64_t ldx, const mx_tensor *W,
                            void *C_bf16, int64_t ldc, int epilogue, float *amax_out, const float *x_gscale,
                            const float *x_amax, void *workspace, size_t workspace_bytes, void *stream) {
    if (!valid_fmt(fmt) || M < 0 || K < 0) return MX_ERR_INVALID_ARG;
    mx_status s = check_tensor(W, true);
    if (s != MX_OK) return s;
    if (!gemm_pair_ok(fmt, W->fmt) || W->cols != K) return MX_ERR_INVALID_ARG;
    if (epilogue != MX_EPI_NONE && epilogue != MX_EPI_GELU) return MX_ERR_INVALID_ARG;
    const int64_t N = W->rows;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (amax_out != nullptr) {
        if (!aligned16(amax_out) && (reinterpret_cast<uintptr_t>(amax_out) & 3u)) return MX_ERR_MISALIGNED;
        if (cudaMemsetAsync(amax_out, 0, sizeof(float), st) != cudaSuccess) return MX_ERR_CUDA;
    }
    if (M == 0 || N == 0) return MX_OK;
    if (!X_bf16 || !C_bf16) return MX_ERR_INVALID_ARG;
    if (ldc < N) return MX_ERR_INVALID_ARG;
    if (!aligned16(C_bf16) || !aligned16(X_bf16) || ldx < K || (ldx & 7) != 0) return MX_ERR_MISALIGNED;
    if (K == 0) return cuda_status(cudaMemset2DAsync(C_bf16, ldc * 2, 0, N * 2, M, st));
    if (K % 128 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
    if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX || cdiv(M, kBM) > 65535) return MX_ERR_UNSUPPORTED_SHAPE;
    if (!workspace) return MX_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MX_ERR_MISALIGNED;
    if (workspace_bytes < fused_ws_bytes(fmt, M, K)) return MX_ERR_INVALID_ARG;
    if (gemm_runtime_types(fmt, W->fmt) && fmt_bits(W->fmt) < 8 && !aligned32(W->codes)) return MX_ERR_MISALIGNED;
    mx_tensor xa;
    const float *ga = nullptr;
    const uint16_t *X = static_cast<const uint16_t *>(X_bf16);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    if (fmt == MX_MXFP4_MBS) {
        // the macro-block GEMM has the plain epilogue only
        if (epilogue != MX_EPI_NONE || amax_out != nullptr) return MX_ERR_INVALID_ARG;
        xa.fmt = fmt;
        xa.reserved = 0;
        xa.rows = M;
        xa.cols = K;
        xa.codes = ws + fused_ws_header(M);
        xa.scales = ws + fused_ws_header(M) + align256((size_t)(M * K / 2));
        xa.gscale = nullptr;
        launch_quantize_mbs(X, M, K, ldx, &xa, st);
        s = last_launch();
        if (s != MX_OK) return s;
        return launch_gemm_mbs(&xa, W, static_cast<uint16_t *>(C_bf16), ldc, st);
    }
    // room for the K split's partial sums (the GEMM decides whether to split)
    SplitRoom room;
    const SplitRoom *roomp = nullptr;
    if (workspace_bytes >= fused_ws_split_bytes(fmt, M, K) && epilogue == MX_EPI_NONE) {
        room.partials = reinterpret_cast<float *>(ws + fused_ws_bytes(fmt, M, K));
        room.flags = reinterpret_cast<uint32_t *>(ws + fused_ws_flags(M));
        room.slot_quads = (int)fused_split_quads(M);
        roomp = &room;
    }
    int mode = g_fused_mode.load();
    // a single 128-row band is written only when the whole quantize is: no band
    // of it to start early on, so the pipelined mode would only add its counter
    // reset
    if (mode == MX_FUSED_PIPELINED && M <= kQTileRows) mode = MX_FUSED_TWO_KERNELS;
    if (mode == MX_FUSED_TWO_KERNELS) {
        // quantize_kernel into the workspace (clearing the slot counters, with
        // split room), then the plain GEMM in stream order
        s = fused_quantize_x(fmt, X, M, K, ldx, ws, x_gscale, x_amax, &xa, &ga, st, nullptr,
                             roomp != nullptr ? room.flags : nullptr, kSplitSlots);
        if (s != MX_OK) return s;
        return launch_gemm(&xa, W, xa.codes, xa.scales, ga, static_cast<uint16_t *>(C_bf16), ldc, epilogue, amax_out,
                           st, nullptr, roomp);
    }
    // X quantized by the GEMM kernel itself (MX_FUSED_IN_KERNEL) or by the
    // quantize kernel, band by band, with the GEMM starting on the bands already
    // written (MX_FUSED_PIPELINED); either way the workspace's counters are
    // cleared first, and NVFP4 without a given g or amax first runs the amax
    // pre-pass into the header.
    xa.fmt = fmt;
    xa.reserved = 0;
    xa.rows = M;
    xa.cols = K;
    xa.codes = ws + fused_ws_header(M);
    xa.scales = ws + fused_ws_header(M) + align256((size_t)(M * K * fmt_bits(fmt) / 8));
    xa.gscale = reinterpret_cast<float *>(ws);
    FusedX fx;
    fx.mode = mode == MX_FUSED_IN_KERNEL ? 1 : 2;
    fx.x = X;
    fx.ldx = ldx;
    fx.x_fmt = fmt;
    fx.ga_from_amax = 0;
    fx.band_ready = reinterpret_cast<uint32_t *>(ws + kWsBandOffset);
    fx.next_item = reinterpret_cast<uint32_t *>(ws + 8);
    // gA for the GEMM's epilogue: never the g the quantize kernel writes (the
    // pipelined GEMM may run before that store is visible), always its source
    float *amax_slot = reinterpret_cast<float *>(ws + 4);
    const float *x_amax_src = x_amax;
    bool prepass = false;
    if (fmt == MX_NVFP4) {
        if (x_gscale != nullptr) {
            ga = x_gscale;
        } else {
            fx.ga_from_amax = 1;
            if (x_amax == nullptr) {
                prepass = true;
                x_amax_src = amax_slot;
            }
            ga = x_amax_src;
        }
    }
    // words 2 .. 15, the band counters and the slot counters (and word 1, the
    // amax slot, before the pre-pass), then the pre-pass: each kernel of the
    // chain overlaps the tail of the one before it
    const int w0 = prepass ? 1 : 2;
    s = launch_fused_reset(reinterpret_cast<uint32_t *>(ws + 4 * w0), (int)(fused_ws_header(M) / 4 - w0), st);
    if (s != MX_OK) return s;
    if (prepass) {
        s = launch_amax_overlapped(X, M, K, ldx, amax_slot, st);
        if (s != MX_OK) return s;
    }
    if (fx.mode == 2) {
        mx_tensor xq;
        const float *unused = nullptr;
        s = fused_quantize_x(fmt, X, M, K, ldx, ws, x_gscale, x_amax_src, &xq, &unused, st, fx.band_ready);
        if (s != MX_OK) return s;
    }
    return launch_gemm(&xa, W, xa.codes, xa.scales, ga, static_cast<uint16_t *>(C_bf16), ldc, epilogue, amax_out, st,
                       &fx, roomp);
}

}  // extern "C"

// --- mx_gemm_fused_act_noalloc: scratch without allocation -------------------
// The scratch lives in this file-scope device array.  Host code must not pass
// the symbol itself to a kernel (on the host it is only a stand-in, not a
// device address): its device address is looked up once per device below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[MX_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 128;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (set up on first use).
mx_status noalloc_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MX_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MX_ERR_UNSUPPORTED_SHAPE;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MX_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return MX_OK;
}
}  // namespace

extern "C" {

mx_status mx_gemm_fused_act_noalloc(int fmt, const void *X_bf16, int64_t M, int64_t K, int64_t ldx,
                                    const mx_tensor *W, void *C_bf16, int64_t ldc, int epilogue, float *amax_out,
                                    const float *x_gscale, const float *x_amax, void *stream) {
    if (!valid_fmt(fmt) || M < 0 || K < 0) return MX_ERR_INVALID_ARG;
    // sizes the fused call rejects anyway, checked first so that the byte
    // count below cannot overflow
    if (M > INT32_MAX || K > INT32_MAX || cdiv(M, kBM) > 65535) return MX_ERR_UNSUPPORTED_SHAPE;
    if (fused_ws_bytes(fmt, M, K) > MX_NOALLOC_SCRATCH_BYTES) return MX_ERR_UNSUPPORTED_SHAPE;
    void *scratch = nullptr;
    const mx_status s = noalloc_scratch(&scratch);
    if (s != MX_OK) return s;
    return mx_gemm_fused_act(fmt, X_bf16, M, K, ldx, W, C_bf16, ldc, epilogue, amax_out, x_gscale, x_amax, scratch,
                             MX_NOALLOC_SCRATCH_BYTES, stream);
}

mx_status mx_check_device_error(void *stream, uint32_t info[4]) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) {
        fprintf(stderr, "libmx: stream error: %s\n", cudaGetErrorString(e));
        return MX_ERR_CUDA;
    }
    uint32_t w[4] = {0, 0, 0, 0};
    if (cudaMemcpyFromSymbol(w, g_error_word, sizeof(w)) != cudaSuccess) return MX_ERR_CUDA;
    const uint32_t zero[4] = {0, 0, 0, 0};
    if (cudaMemcpyToSymbol(g_error_word, zero, sizeof(zero)) != cudaSuccess) return MX_ERR_CUDA;
    if (info) memcpy(info, w, sizeof(w));
    if (w[0] & DEVERR_TIMEOUT) return MX_ERR_TIMEOUT;
    if (w[0] & DEVERR_BOUNDS) return MX_ERR_DEVICE;
    return MX_OK;
}

}  // extern "C"
