// libmxmoe: C ABI of the MXFP8 routed-experts MLP (declared in include/mxmoe.h).
//
// One translation unit: the cast kernels (quant.cuh), the tcgen05 grouped
// GEMM (gemm.cuh), the token dispatcher (route.cuh) and the host code below,
// which validates every argument, encodes the TMA tensor maps, launches on
// the caller's stream and chains the composites.  Nothing here calls a
// device allocator.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/mxmoe.h"
#include "gemm.cuh"
#include "quant.cuh"
#include "route.cuh"

using namespace mxmoe;

// Build-time choices, for measuring one tiling against another:
// tile width of the single-CTA weight-gradient (ragged-K) GEMM when Kx allows
// both, 256 (one TMEM accumulator) or 128 (two, the epilogue overlapped with
// the next tile's MMAs) ...
#ifndef MXMOE_WGRAD_BN
#define MXMOE_WGRAD_BN 256
#endif
// ... and 256 x 256 tiles on CTA pairs (cta_group::2) wherever the shapes
// allow, for the ragged-M GEMMs and for the weight gradients.
#ifndef MXMOE_USE_PAIRS
#define MXMOE_USE_PAIRS 1
#endif
#ifndef MXMOE_WGRAD_PAIRS
#define MXMOE_WGRAD_PAIRS 1
#endif

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(MXMOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define MX_CHECK_CUDA(call, what)              \
  do {                                         \
    cudaError_t e_ = (call);                   \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

#define MX_TRY(expr)          \
  do {                        \
    int s_ = (expr);          \
    if (s_ != MXMOE_OK) return s_; \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

constexpr int kMaxDevices = 64;
struct DevInfo {
  int checked = 0;   // 1 ok, -1 wrong arch
  int sms = 0;
  unsigned attr_set = 0;  // bitmask of kernel instantiations with smem attribute set
};
DevInfo g_dev[kMaxDevices];
std::mutex g_mu;

int device_info(DevInfo** out) {
  int dev = 0;
  MX_CHECK_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MXMOE_ERR_CUDA, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  DevInfo& d = g_dev[dev];
  if (d.checked == 0) {
    int major = 0, minor = 0, sms = 0;
    MX_CHECK_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev), "attr");
    MX_CHECK_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev), "attr");
    MX_CHECK_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "attr");
    d.sms = sms;
    d.checked = (major == 10 && minor == 0) ? 1 : -1;
  }
  if (d.checked < 0) return fail(MXMOE_ERR_ARCH, "device %d is not sm_100 (this library is built for sm_100a)", dev);
  *out = &d;
  return MXMOE_OK;
}

// ---------------------------------------------------------------- TMA tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int get_encode(EncodeTiledFn* fn) {
  static EncodeTiledFn cached = nullptr;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) cached = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (!cached) return fail(MXMOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(err));
  *fn = cached;
  return MXMOE_OK;
}

// 2-D uint8 K-major operand [rows, kext], box 128 bytes x box_rows, 128-byte swizzle.
int make_operand_map(CUtensorMap* map, const uint8_t* base, int64_t rows, int64_t kext, uint32_t box_rows = 128) {
  EncodeTiledFn enc;
  MX_TRY(get_encode(&enc));
  cuuint64_t dims[2] = {cuuint64_t(kext), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(kext)};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MXMOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return MXMOE_OK;
}

struct GatherArgs {
  const int32_t* row_slot;
  const float* slot_weight;
  int64_t n_slots;
  int top_k;
};

// 3-D bf16 cast input [batch, rows, ld], box 64 x box_rows x 1 (128-byte rows)
// in the 128-byte swizzle, zero fill past the edges.
int make_cast_map(CUtensorMap* map, const void* base, int64_t batch, int64_t rows, int64_t ld, uint32_t box_rows) {
  EncodeTiledFn enc;
  MX_TRY(get_encode(&enc));
  cuuint64_t dims[3] = {cuuint64_t(ld), cuuint64_t(rows), cuuint64_t(batch)};
  cuuint64_t strides[2] = {cuuint64_t(ld * 2), cuuint64_t(rows * ld * 2)};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MXMOE_ERR_CUDA, "cuTensorMapEncodeTiled (cast) failed (%d)", int(r));
  return MXMOE_OK;
}

// 2-D bf16 token matrix [tokens, ld] for four-row gathers: box 128 x 1, no
// swizzle, zero fill past the column edge.
int make_gather_map(CUtensorMap* map, const void* base, int64_t tokens, int64_t ld) {
  EncodeTiledFn enc;
  MX_TRY(get_encode(&enc));
  cuuint64_t dims[2] = {cuuint64_t(ld), cuuint64_t(tokens > 0 ? tokens : 1)};
  cuuint64_t strides[1] = {cuuint64_t(ld * 2)};
  cuuint32_t box[2] = {128, 1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MXMOE_ERR_CUDA, "cuTensorMapEncodeTiled (gather) failed (%d)", int(r));
  return MXMOE_OK;
}

template <int kMode, int kElem = 0>
int launch_cast(const void* in, int64_t batch, int64_t rows, int64_t cols, int modes, int layout, uint8_t* rc,
                uint8_t* rs, uint8_t* cc, uint8_t* cs, const int32_t* dev_rows, cudaStream_t stream,
                const GatherArgs* g = nullptr) {
  using C = CastCfg<kMode>;
  constexpr bool kSwiglu = kMode == kCastSwiglu;
  DevInfo* d;
  MX_TRY(device_info(&d));
  // attribute bits 17.. (the GEMMs use 0-16): one per (mode, element)
  const int bit = 17 + kMode * 2 + kElem;
  auto kern = mx_cast_kernel<kMode, kElem>;
  if (!(d->attr_set & (1u << bit))) {
    MX_CHECK_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem),
                  "cudaFuncSetAttribute");
    std::lock_guard<std::mutex> lk(g_mu);
    d->attr_set |= (1u << bit);
  }
  CUtensorMap map;
  if constexpr (kMode == kCastGather) {
    if (!g) return fail(MXMOE_ERR_ARG, "gather cast without a slot table");
    MX_TRY(make_gather_map(&map, in, g->n_slots / g->top_k, cols));
  } else
    MX_TRY(make_cast_map(&map, in, batch, rows, kSwiglu ? 2 * cols : cols, C::kTileRows));
  CastArgs a;
  memset(&a, 0, sizeof(a));
  if (g) {
    a.src = static_cast<const uint16_t*>(in);
    a.row_slot = g->row_slot;
    a.slot_weight = g->slot_weight;
    a.n_slots = g->n_slots;
    a.top_k = g->top_k;
  }
  a.rows = rows;
  a.cols = cols;
  a.batch = batch;
  a.up_off = kSwiglu ? cols : 0;
  a.tiles_c = (cols + 127) / 128;
  a.tiles_r = (rows + C::kTileRows - 1) / C::kTileRows;
  a.modes = modes;
  a.mma_layout = layout;
  a.row_codes = rc;
  a.row_scales = rs;
  a.col_codes = cc;
  a.col_scales = cs;
  a.dev_rows = dev_rows;
  const int64_t ntiles = batch * a.tiles_r * a.tiles_c;
  if (ntiles >= (int64_t(1) << 31)) return fail(MXMOE_ERR_SHAPE, "cast of %lld tiles: too large", (long long)ntiles);
  const int64_t per_sm = C::kCtasPerSm;
  const int grid = int(ntiles < per_sm * d->sms ? ntiles : per_sm * d->sms);
  kern<<<grid, C::kThreads, C::kSmem, stream>>>(map, a);
  MX_CHECK_CUDA(cudaGetLastError(), "cast launch");
  return MXMOE_OK;
}

// bf16 output [rows, cols] stored in 32 x 32 boxes with the 64-byte swizzle.
int make_out_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols) {
  EncodeTiledFn enc;
  MX_TRY(get_encode(&enc));
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(cols * 2)};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MXMOE_ERR_CUDA, "cuTensorMapEncodeTiled (output) failed (%d)", int(r));
  return MXMOE_OK;
}

// Scale atoms of an MMA-layout scale buffer of `bytes` bytes as a 2-D uint8
// map [bytes/256, 256] with 256 x 2 boxes (one 512-byte atom per box).
int make_scale_map(CUtensorMap* map, const uint8_t* base, int64_t bytes) {
  EncodeTiledFn enc;
  MX_TRY(get_encode(&enc));
  cuuint64_t dims[2] = {256, cuuint64_t(bytes / 256)};
  cuuint64_t strides[1] = {256};
  cuuint32_t box[2] = {256, 2};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MXMOE_ERR_CUDA, "cuTensorMapEncodeTiled (scales) failed (%d)", int(r));
  return MXMOE_OK;
}

// ---------------------------------------------------------------- GEMM launch
template <int kMode, int kEpi, int BN, bool kPair>
int launch_gemm(const uint8_t* a, int64_t a_rows, const uint8_t* b, int64_t b_rows, gemm::Params p,
                int64_t max_tiles, cudaStream_t stream, int attr_bit) {
  using C = gemm::Cfg<kMode, kEpi, BN, kPair>;
  DevInfo* d;
  MX_TRY(device_info(&d));
  auto kern = gemm::grouped_gemm_kernel<kMode, kEpi, BN, kPair>;
  if (!(d->attr_set & (1u << attr_bit))) {
    MX_CHECK_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES),
                  "cudaFuncSetAttribute");
    std::lock_guard<std::mutex> lk(g_mu);
    d->attr_set |= (1u << attr_bit);
  }
  if (p.E > C::MAX_E) return fail(MXMOE_ERR_SHAPE, "E=%d exceeds the supported maximum %d", p.E, C::MAX_E);
  CUtensorMap ma, mb, msa, msb;
  MX_TRY(make_operand_map(&ma, a, a_rows, p.kext));
  MX_TRY(make_operand_map(&mb, b, b_rows, p.kext, kPair ? BN / 2 : 128));
  if constexpr (kPair) {
    MX_TRY(make_scale_map(&msa, p.a_scales, a_rows * p.kext / 32));
    MX_TRY(make_scale_map(&msb, p.b_scales, b_rows * p.kext / 32));
  } else {
    msa = ma;   // unused by the single-CTA kernel
    msb = mb;
  }
  // bf16 output written by TMA stores: [M, N] (ragged M), [E*N, Kx] (ragged K), h13 [M, 2F] (SwiGLU)
  CUtensorMap mo = ma;
  if (p.out != nullptr) {
    if constexpr (kEpi == gemm::kEpiBF16) {
      if constexpr (kMode == gemm::kRaggedK)
        MX_TRY(make_out_map(&mo, p.out, int64_t(p.E) * p.rows_a, p.n_out));
      else
        MX_TRY(make_out_map(&mo, p.out, p.M, p.n_out));
    } else if constexpr (kEpi == gemm::kEpiSwiGLU) {
      MX_TRY(make_out_map(&mo, p.out, p.M, 2 * p.F));
    }
  }
  if (max_tiles <= 0) return MXMOE_OK;
  if constexpr (!kPair) {
    const int grid = int(max_tiles < d->sms ? max_tiles : d->sms);
    kern<<<grid, 384, C::SMEM_BYTES, stream>>>(ma, mb, msa, msb, mo, p);
  } else {
    // clusters of two CTAs, one pair per two SMs (as many as can be resident)
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(384, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int pairs = d->sms / 2;
    cfg.gridDim = dim3(unsigned(2 * pairs), 1, 1);
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, kern, &cfg) == cudaSuccess && active > 0 && active < pairs)
      pairs = active;
    cudaGetLastError();
    if (max_tiles < pairs) pairs = int(max_tiles);
    cfg.gridDim = dim3(unsigned(2 * pairs), 1, 1);
    MX_CHECK_CUDA(cudaLaunchKernelEx(&cfg, kern, ma, mb, msa, msb, mo, p), "grouped GEMM (CTA pair) launch");
  }
  MX_CHECK_CUDA(cudaGetLastError(), "grouped GEMM launch");
  return MXMOE_OK;
}

int check_offsets_args(const int32_t* offsets, int E, int pad) {
  if (!offsets) return fail(MXMOE_ERR_NULL, "expert_offsets is NULL");
  if (E <= 0) return fail(MXMOE_ERR_SHAPE, "E=%d must be positive", E);
  if (pad < 128 || pad % 128 != 0)
    return fail(MXMOE_ERR_SHAPE, "pad_multiple=%d must be a positive multiple of 128", pad);
  return MXMOE_OK;
}

int check_mult(const char* name, int64_t v, int64_t m) {
  if (v <= 0 || v % m != 0) return fail(MXMOE_ERR_SHAPE, "%s=%lld must be a positive multiple of %lld", name,
                                        (long long)v, (long long)m);
  return MXMOE_OK;
}

int check_ptrs(std::initializer_list<std::pair<const char*, const void*>> ps) {
  for (auto& kv : ps) {
    if (!kv.second) return fail(MXMOE_ERR_NULL, "%s is NULL", kv.first);
    if (!aligned16(kv.second)) return fail(MXMOE_ERR_ALIGN, "%s is not 16-byte aligned", kv.first);
  }
  return MXMOE_OK;
}

// ---------------------------------------------------------------- casts
int quantize_impl(const void* x, int64_t batch, int64_t rows, int64_t cols, int modes, int layout,
                  uint8_t* rc, uint8_t* rs, uint8_t* cc, uint8_t* cs, cudaStream_t stream,
                  bool swiglu = false, int elem = 0) {
  if (modes < 1 || modes > 3) return fail(MXMOE_ERR_ARG, "modes=%d must be MXFP8_ROW, MXFP8_COL or both", modes);
  if (layout != MXFP8_SCALE_PLAIN && layout != MXFP8_SCALE_MMA)
    return fail(MXMOE_ERR_ARG, "scale_layout=%d invalid", layout);
  if (batch <= 0 || rows <= 0 || cols <= 0)
    return fail(MXMOE_ERR_SHAPE, "batch=%lld rows=%lld cols=%lld must be positive", (long long)batch,
                (long long)rows, (long long)cols);
  if (!x) return fail(MXMOE_ERR_NULL, "input is NULL");
  const bool row = modes & MXFP8_ROW, col = modes & MXFP8_COL;
  if (row && (!rc || !rs)) return fail(MXMOE_ERR_NULL, "row_codes/row_scales NULL with MXFP8_ROW");
  if (col && (!cc || !cs)) return fail(MXMOE_ERR_NULL, "col_codes/col_scales NULL with MXFP8_COL");
  if (col && rows % 32 != 0) return fail(MXMOE_ERR_SHAPE, "MXFP8_COL needs rows %% 32 == 0 (rows=%lld)", (long long)rows);
  if (layout == MXFP8_SCALE_MMA && (rows % 128 != 0 || cols % 128 != 0))
    return fail(MXMOE_ERR_SHAPE, "MMA scale layout needs rows and cols multiples of 128 (%lld x %lld)",
                (long long)rows, (long long)cols);
  if (layout == MXFP8_SCALE_MMA && ((row && !aligned16(rs)) || (col && !aligned16(cs))))
    return fail(MXMOE_ERR_ALIGN, "MMA-layout scale buffers must be 16-byte aligned");
  const bool vec_ok = cols % 32 == 0 && aligned16(x) && (!row || aligned16(rc)) && (!col || aligned16(cc)) &&
                      (!col || rows % 16 == 0);
  if (swiglu && !vec_ok) return fail(MXMOE_ERR_SHAPE, "SwiGLU quant needs F %% 32 == 0 and 16-byte aligned buffers");
  const uint16_t* in = static_cast<const uint16_t*>(x);
  DevInfo* d;
  MX_TRY(device_info(&d));
  if (!vec_ok) {
    if (col) return fail(MXMOE_ERR_SHAPE, "MXFP8_COL needs cols %% 32 == 0 and 16-byte aligned buffers");
    if (layout == MXFP8_SCALE_MMA) return fail(MXMOE_ERR_SHAPE, "MMA layout needs aligned buffers");
    const int64_t R = batch * rows;
    const int64_t warps = R * ((cols + 31) / 32);
    const int64_t blocks = (warps * 32 + 255) / 256;
    if (blocks > 0x7FFFFFFF) return fail(MXMOE_ERR_SHAPE, "tensor too large");
    if (elem == 1)
      mx_row_generic_kernel<1><<<unsigned(blocks), 256, 0, stream>>>(in, R, cols, rc, rs);
    else
      mx_row_generic_kernel<0><<<unsigned(blocks), 256, 0, stream>>>(in, R, cols, rc, rs);
    MX_CHECK_CUDA(cudaGetLastError(), "cast launch");
    return MXMOE_OK;
  }
  if (swiglu)
    return launch_cast<kCastSwiglu>(x, 1, rows, cols, modes, layout, rc, rs, cc, cs, nullptr, stream);
  if (elem == 1) return launch_cast<kCastPlain, 1>(x, batch, rows, cols, modes, layout, rc, rs, cc, cs, nullptr, stream);
  return launch_cast<kCastPlain>(x, batch, rows, cols, modes, layout, rc, rs, cc, cs, nullptr, stream);
}

// Cast of the token buffer used inside the composites: rows at or past
// offsets[E] (read on the device) are neither read nor written.
int quantize_tokens(const void* x, int64_t rows, int64_t cols, const int32_t* rows_dev, uint8_t* rc, uint8_t* rs,
                    uint8_t* cc, uint8_t* cs, cudaStream_t stream) {
  return launch_cast<kCastPlain>(x, 1, rows, cols, MXFP8_ROW | MXFP8_COL, MXFP8_SCALE_MMA, rc, rs, cc, cs, rows_dev,
                            stream);
}

int gemm_ragged_m(const uint8_t* a, const uint8_t* as, int64_t M, int64_t K, const uint8_t* w,
                  const uint8_t* ws, int E, int64_t N, const int32_t* offsets, int pad, void* out,
                  cudaStream_t stream) {
  gemm::Params p{};
  p.E = E;
  p.rows_a = M;
  p.kext = K;
  p.n_out = N;
  p.M = M;
  p.offsets = offsets;
  p.pad = pad;
  p.a_scales = as;
  p.b_scales = ws;
  p.out = static_cast<uint16_t*>(out);
  if (MXMOE_USE_PAIRS && N % 256 == 0 && pad % 256 == 0)
    return launch_gemm<gemm::kRaggedM, gemm::kEpiBF16, 256, true>(a, M, w, int64_t(E) * N, p,
                                                                  (M / 256) * (N / 256), stream, 9);
  if (N % 256 == 0)
    return launch_gemm<gemm::kRaggedM, gemm::kEpiBF16, 256, false>(a, M, w, int64_t(E) * N, p,
                                                                   (M / 128) * (N / 256), stream, 0);
  return launch_gemm<gemm::kRaggedM, gemm::kEpiBF16, 128, false>(a, M, w, int64_t(E) * N, p, (M / 128) * (N / 128),
                                                                 stream, 1);
}

int gemm_ragged_k(const uint8_t* gt, const uint8_t* gs, int64_t N, const uint8_t* xt, const uint8_t* xs,
                  int64_t Kx, int64_t M, const int32_t* offsets, const int32_t* rows, int E, int pad, void* dw,
                  cudaStream_t stream) {
  gemm::Params p{};
  p.rows = rows;
  p.E = E;
  p.rows_a = N;
  p.kext = M;
  p.n_out = Kx;
  p.M = M;
  p.offsets = offsets;
  p.pad = pad;
  p.a_scales = gs;
  p.b_scales = xs;
  p.out = static_cast<uint16_t*>(dw);
  // CTA pairs (256 x 256 tiles, 128 x 256 per CTA) when N and Kx allow: they
  // halve each SM's B-operand loads; the accumulator hand-off, paid once
  // per tile over each expert's short K, uses a CTA-scope arrive
  if (MXMOE_WGRAD_PAIRS && Kx % 256 == 0 && N % 256 == 0)
    return launch_gemm<gemm::kRaggedK, gemm::kEpiBF16, 256, true>(gt, N, xt, Kx, p,
                                                                  int64_t(E) * (N / 256) * (Kx / 256), stream, 10);
  if (Kx % 256 == 0 && MXMOE_WGRAD_BN == 256)
    return launch_gemm<gemm::kRaggedK, gemm::kEpiBF16, 256, false>(gt, N, xt, Kx, p,
                                                                   int64_t(E) * (N / 128) * (Kx / 256), stream, 2);
  return launch_gemm<gemm::kRaggedK, gemm::kEpiBF16, 128, false>(gt, N, xt, Kx, p,
                                                                 int64_t(E) * (N / 128) * (Kx / 128), stream, 3);
}

int gemm_swiglu(const uint8_t* a, const uint8_t* as, int64_t M, int64_t K, const uint8_t* w13, const uint8_t* ws,
                int E, int64_t F, const int32_t* offsets, int pad, void* h13, uint8_t* hrc, uint8_t* hrs,
                uint8_t* hcc, uint8_t* hcs, cudaStream_t stream) {
  gemm::Params p{};
  p.E = E;
  p.rows_a = M;
  p.kext = K;
  p.n_out = 2 * F;
  p.M = M;
  p.offsets = offsets;
  p.pad = pad;
  p.a_scales = as;
  p.b_scales = ws;
  p.out = static_cast<uint16_t*>(h13);
  p.F = F;
  p.row_codes = hrc;
  p.row_scales = hrs;
  p.col_codes = hcc;
  p.col_scales = hcs;
  if (MXMOE_USE_PAIRS && pad % 256 == 0)
    return launch_gemm<gemm::kRaggedM, gemm::kEpiSwiGLU, 256, true>(a, M, w13, int64_t(E) * 2 * F, p,
                                                                    (M / 256) * (F / 128), stream, 11);
  return launch_gemm<gemm::kRaggedM, gemm::kEpiSwiGLU, 256, false>(a, M, w13, int64_t(E) * 2 * F, p,
                                                                   (M / 128) * (F / 128), stream, 4);
}

int gemm_dswiglu(const uint8_t* dy, const uint8_t* ds, int64_t M, int64_t D, const uint8_t* w2t,
                 const uint8_t* w2ts, int E, int64_t F, const int32_t* offsets, int pad, const void* h13,
                 uint8_t* grc, uint8_t* grs, uint8_t* gcc, uint8_t* gcs, cudaStream_t stream) {
  gemm::Params p{};
  p.E = E;
  p.rows_a = M;
  p.kext = D;
  p.n_out = F;
  p.M = M;
  p.offsets = offsets;
  p.pad = pad;
  p.a_scales = ds;
  p.b_scales = w2ts;
  p.h13 = static_cast<const uint16_t*>(h13);
  p.F = F;
  p.row_codes = grc;
  p.row_scales = grs;
  p.col_codes = gcc;
  p.col_scales = gcs;
  if (MXMOE_USE_PAIRS && F % 256 == 0 && pad % 256 == 0)
    return launch_gemm<gemm::kRaggedM, gemm::kEpiDSwiGLU, 256, true>(dy, M, w2t, int64_t(E) * F, p,
                                                                     (M / 256) * (F / 256), stream, 12);
  if (F % 256 == 0)
    return launch_gemm<gemm::kRaggedM, gemm::kEpiDSwiGLU, 256, false>(dy, M, w2t, int64_t(E) * F, p,
                                                                      (M / 128) * (F / 256), stream, 5);
  return launch_gemm<gemm::kRaggedM, gemm::kEpiDSwiGLU, 128, false>(dy, M, w2t, int64_t(E) * F, p,
                                                                    (M / 128) * (F / 128), stream, 6);
}

// ---------------------------------------------------------------- workspace
struct Carver {
  uint8_t* base;
  size_t off = 0;
  template <class T>
  T* take(size_t bytes) {
    off = (off + 255) & ~size_t(255);
    T* r = reinterpret_cast<T*>(base ? base + off : nullptr);
    off += bytes;
    return r;
  }
};

struct FwdWs {
  uint8_t *x_rc, *x_rs, *h_rc, *h_rs;
  mxmoe_qweights qw;   // ROW weight codes when the caller gives bf16 weights
};
struct BwdWs {
  uint8_t *dy_rc, *dy_rs, *dy_cc, *dy_cs, *g_rc, *g_rs, *g_cc, *g_cs;
  mxmoe_qweights qw;   // COL weight codes when the caller gives bf16 weights
};

// with_weights: also carve room for the weight codes (bf16-weight composites)
size_t carve_fwd(uint8_t* base, int64_t M, int64_t D, int E, int64_t F, FwdWs* w, bool with_weights) {
  Carver c{base};
  w->x_rc = c.take<uint8_t>(M * D);
  w->x_rs = c.take<uint8_t>(M * D / 32);
  w->h_rc = c.take<uint8_t>(M * F);
  w->h_rs = c.take<uint8_t>(M * F / 32);
  w->qw = mxmoe_qweights{};
  if (with_weights) {
    w->qw.w13_codes = c.take<uint8_t>(int64_t(E) * 2 * F * D);
    w->qw.w13_scales = c.take<uint8_t>(int64_t(E) * 2 * F * D / 32);
    w->qw.w2_codes = c.take<uint8_t>(int64_t(E) * D * F);
    w->qw.w2_scales = c.take<uint8_t>(int64_t(E) * D * F / 32);
  }
  return c.off + 256;
}

size_t carve_bwd(uint8_t* base, int64_t M, int64_t D, int E, int64_t F, BwdWs* w, bool with_weights) {
  Carver c{base};
  w->dy_rc = c.take<uint8_t>(M * D);
  w->dy_rs = c.take<uint8_t>(M * D / 32);
  w->dy_cc = c.take<uint8_t>(M * D);
  w->dy_cs = c.take<uint8_t>(M * D / 32);
  w->g_rc = c.take<uint8_t>(M * 2 * F);
  w->g_rs = c.take<uint8_t>(M * 2 * F / 32);
  w->g_cc = c.take<uint8_t>(M * 2 * F);
  w->g_cs = c.take<uint8_t>(M * 2 * F / 32);
  w->qw = mxmoe_qweights{};
  if (with_weights) {
    w->qw.w2t_codes = c.take<uint8_t>(int64_t(E) * D * F);
    w->qw.w2t_scales = c.take<uint8_t>(int64_t(E) * D * F / 32);
    w->qw.w13t_codes = c.take<uint8_t>(int64_t(E) * 2 * F * D);
    w->qw.w13t_scales = c.take<uint8_t>(int64_t(E) * 2 * F * D / 32);
  }
  return c.off + 256;
}

// forward with ROW-quantized weights in qw (a1, a3, a4)
int fwd_core(const void* x, int64_t M, int64_t D, const mxmoe_qweights& qw, int E, int64_t F,
             const int32_t* offsets, int pad, void* y, const mxmoe_saved* saved, const FwdWs& w,
             cudaStream_t stream) {
  // a1: x -> ROW (FC1 operand) + COL (dW13 operand, saved)
  MX_TRY(quantize_tokens(x, M, D, offsets + E, w.x_rc, w.x_rs, saved->x_col_codes, saved->x_col_scales, stream));
  // a3: FC1 + SwiGLU + dual quantization
  MX_TRY(gemm_swiglu(w.x_rc, w.x_rs, M, D, qw.w13_codes, qw.w13_scales, E, F, offsets, pad, saved->h13, w.h_rc,
                     w.h_rs, saved->h_col_codes, saved->h_col_scales, stream));
  // a4: FC2
  return gemm_ragged_m(w.h_rc, w.h_rs, M, F, qw.w2_codes, qw.w2_scales, E, D, offsets, pad, y, stream);
}

// backward with COL-quantized weights in qw (a5 - a9)
int bwd_core(const void* dy, int64_t M, int64_t D, const mxmoe_qweights& qw, int E, int64_t F,
             const int32_t* offsets, int pad, const mxmoe_saved* saved, void* dx, void* dw13, void* dw2,
             const BwdWs& w, cudaStream_t stream) {
  // a5: dY -> ROW (dh operand) + COL (dW2 operand)
  MX_TRY(quantize_tokens(dy, M, D, offsets + E, w.dy_rc, w.dy_rs, w.dy_cc, w.dy_cs, stream));
  // a6: dh = dY . W2[e] with the fused dSwiGLU + dual quantization
  MX_TRY(gemm_dswiglu(w.dy_rc, w.dy_rs, M, D, qw.w2t_codes, qw.w2t_scales, E, F, offsets, pad, saved->h13, w.g_rc,
                      w.g_rs, w.g_cc, w.g_cs, stream));
  // a7: dW2[e] = dY_e^T . h_e
  MX_TRY(gemm_ragged_k(w.dy_cc, w.dy_cs, D, saved->h_col_codes, saved->h_col_scales, F, M, offsets, nullptr, E, pad, dw2,
                       stream));
  // a8: dx = dh13 . W13[e]
  MX_TRY(gemm_ragged_m(w.g_rc, w.g_rs, M, 2 * F, qw.w13t_codes, qw.w13t_scales, E, D, offsets, pad, dx, stream));
  // a9: dW13[e] = dh13_e^T . x_e
  return gemm_ragged_k(w.g_cc, w.g_cs, 2 * F, saved->x_col_codes, saved->x_col_scales, D, M, offsets, nullptr, E, pad, dw13,
                       stream);
}

int check_qweights(const mxmoe_qweights* qw, bool fwd, bool bwd) {
  if (!qw) return fail(MXMOE_ERR_NULL, "qweights is NULL");
  if (fwd) MX_TRY(check_ptrs({{"qw.w13_codes", qw->w13_codes}, {"qw.w13_scales", qw->w13_scales},
                              {"qw.w2_codes", qw->w2_codes}, {"qw.w2_scales", qw->w2_scales}}));
  if (bwd) MX_TRY(check_ptrs({{"qw.w13t_codes", qw->w13t_codes}, {"qw.w13t_scales", qw->w13t_scales},
                              {"qw.w2t_codes", qw->w2t_codes}, {"qw.w2t_scales", qw->w2t_scales}}));
  return MXMOE_OK;
}

int check_saved(const mxmoe_saved* saved) {
  if (!saved) return fail(MXMOE_ERR_NULL, "saved is NULL");
  return check_ptrs({{"saved.h13", saved->h13}, {"saved.h_col_codes", saved->h_col_codes},
                     {"saved.h_col_scales", saved->h_col_scales}, {"saved.x_col_codes", saved->x_col_codes},
                     {"saved.x_col_scales", saved->x_col_scales}});
}

int check_mlp_shapes(int64_t M, int64_t D, int E, int64_t F, const int32_t* offsets, int pad) {
  MX_TRY(check_offsets_args(offsets, E, pad));
  MX_TRY(check_mult("M", M, 128));
  MX_TRY(check_mult("D", D, 128));
  MX_TRY(check_mult("F", F, 128));
  return MXMOE_OK;
}

uint8_t* align_ws(void* ws) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
}

// ---------------------------------------------------------------- layer composites
// Token-major layer: routing + gather/cast in front of the MLP, combine behind.
struct LayerFwdWs {
  FwdWs mlp;
  int32_t* route_ws;
};
struct LayerBwdWs {
  BwdWs mlp;
  uint16_t* dx_rows;   // dx of the padded rows, before the unpermute
  int32_t* rows;       // real rows of each expert (the weight gradients skip the all-pad K blocks)
};

int64_t route_chunks(int64_t T, int k) { return (T * k + kRouteChunk - 1) / kRouteChunk; }

size_t carve_layer_fwd(uint8_t* base, int64_t T, int k, int64_t m_cap, int64_t D, int E, int64_t F, LayerFwdWs* w) {
  Carver c{base};
  w->mlp.x_rc = c.take<uint8_t>(m_cap * D);
  w->mlp.x_rs = c.take<uint8_t>(m_cap * D / 32);
  w->mlp.h_rc = c.take<uint8_t>(m_cap * F);
  w->mlp.h_rs = c.take<uint8_t>(m_cap * F / 32);
  w->mlp.qw = mxmoe_qweights{};
  w->route_ws = c.take<int32_t>(size_t(route_chunks(T, k)) * E * 4 + 16);
  return c.off + 256;
}

size_t carve_layer_bwd(uint8_t* base, int64_t m_cap, int64_t D, int E, int64_t F, LayerBwdWs* w) {
  Carver c{base};
  BwdWs& b = w->mlp;
  b.dy_rc = c.take<uint8_t>(m_cap * D);
  b.dy_rs = c.take<uint8_t>(m_cap * D / 32);
  b.dy_cc = c.take<uint8_t>(m_cap * D);
  b.dy_cs = c.take<uint8_t>(m_cap * D / 32);
  b.g_rc = c.take<uint8_t>(m_cap * 2 * F);
  b.g_rs = c.take<uint8_t>(m_cap * 2 * F / 32);
  b.g_cc = c.take<uint8_t>(m_cap * 2 * F);
  b.g_cs = c.take<uint8_t>(m_cap * 2 * F / 32);
  b.qw = mxmoe_qweights{};
  w->dx_rows = c.take<uint16_t>(m_cap * D * 2);
  w->rows = c.take<int32_t>(size_t(E) * 4);
  return c.off + 256;
}

int check_layer_args(int64_t T, int64_t D, int top_k, int E, int64_t F, int pad, int64_t* m_cap) {
  if (T <= 0 || top_k <= 0 || top_k > 64 || top_k > E)
    return fail(MXMOE_ERR_SHAPE, "T=%lld top_k=%d (1..min(64, E)) E=%d", (long long)T, top_k, E);
  if (E > kRouteMaxE) return fail(MXMOE_ERR_SHAPE, "E=%d exceeds %d", E, kRouteMaxE);
  if (pad <= 0 || pad % 128 != 0) return fail(MXMOE_ERR_SHAPE, "pad_multiple=%d must be a positive multiple of 128", pad);
  MX_TRY(check_mult("D", D, 128));
  MX_TRY(check_mult("F", F, 128));
  if (T > 0x7FFFFFFF / top_k) return fail(MXMOE_ERR_SHAPE, "T*top_k must be below 2^31");
  *m_cap = mxmoe_route_capacity(T, top_k, E, pad);
  if (*m_cap <= 0 || *m_cap >= (int64_t(1) << 31)) return fail(MXMOE_ERR_SHAPE, "layer too large");
  return MXMOE_OK;
}

int check_layer_saved(const mxmoe_layer_saved* s) {
  if (!s) return fail(MXMOE_ERR_NULL, "layer saved is NULL");
  MX_TRY(check_ptrs({{"saved.offsets", s->offsets}, {"saved.row_slot", s->row_slot},
                     {"saved.slot_row", s->slot_row}, {"saved.y", s->y}}));
  return check_saved(&s->mlp);
}

}  // namespace

// One thread waits on a barrier nothing arrives on: the bounded wait gives up
// and the kernel records the timeout (exercises the failure path).
__global__ void selftest_wait_kernel() {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mxmoe::sm100::mbar_init(mxmoe::sm100::smem_u32(&bar), 1);
    mxmoe::sm100::fence_mbar_init();
    if (!mxmoe::sm100::mbar_wait(mxmoe::sm100::smem_u32(&bar), 0)) raise_device_error(MXMOE_ERR_DEVICE_TIMEOUT);
  }
}

// =====================================================================================
template <int kElem>
int dequantize_impl(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols, void* out,
                    cudaStream_t stream) {
  if (!codes || !scales || !out) return fail(MXMOE_ERR_NULL, "codes/scales/out is NULL");
  if (rows <= 0 || cols <= 0) return fail(MXMOE_ERR_SHAPE, "rows and cols must be positive");
  DevInfo* d;
  MX_TRY(device_info(&d));
  const int64_t n = rows * cols;
  const bool vec = cols % 16 == 0 && reinterpret_cast<uintptr_t>(codes) % 16 == 0 &&
                   reinterpret_cast<uintptr_t>(out) % 16 == 0;
  if (vec) {
    const int64_t n16 = n / 16, cpr = cols / 16, ncb = (cols + 31) / 32;
    const int64_t blocks = std::min<int64_t>((n16 + 255) / 256, int64_t(d->sms) * 8);
    const auto* c4 = reinterpret_cast<const uint4*>(codes);
    auto* o4 = static_cast<uint4*>(out);
    if (n16 < (int64_t(1) << 31))
      mx_dequant16_kernel<uint32_t, kElem><<<unsigned(blocks), 256, 0, stream>>>(c4, scales, uint32_t(n16),
                                                                                 uint32_t(cpr), uint32_t(ncb), o4);
    else
      mx_dequant16_kernel<uint64_t, kElem><<<unsigned(blocks), 256, 0, stream>>>(c4, scales, uint64_t(n16),
                                                                                 uint64_t(cpr), uint64_t(ncb), o4);
    MX_CHECK_CUDA(cudaGetLastError(), "dequant launch");
    return MXMOE_OK;
  }
  const int64_t blocks = (n + 255) / 256;
  if (blocks > 0x7FFFFFFF) return fail(MXMOE_ERR_SHAPE, "tensor too large");
  mx_dequant_kernel<kElem><<<unsigned(blocks), 256, 0, stream>>>(codes, scales, rows, cols,
                                                                 static_cast<uint16_t*>(out));
  MX_CHECK_CUDA(cudaGetLastError(), "dequant launch");
  return MXMOE_OK;
}

extern "C" {

int mxmoe_selftest_wait_timeout(cudaStream_t stream) {
  DevInfo* d;
  MX_TRY(device_info(&d));
  selftest_wait_kernel<<<1, 32, 0, stream>>>();
  MX_CHECK_CUDA(cudaGetLastError(), "self-test launch");
  return MXMOE_OK;
}

const char* mxmoe_last_error_message(void) { return g_err; }

const char* mxmoe_version(void) { return "mxmoe 0.1 (sm_100a, tcgen05 block-scaled MXFP8)"; }

int mxmoe_check_device_error(cudaStream_t stream, int reset, int* code) {
  if (!code) return fail(MXMOE_ERR_NULL, "code is NULL");
  MX_CHECK_CUDA(cudaStreamSynchronize(stream), "cudaStreamSynchronize");
  int v = 0;
  MX_CHECK_CUDA(cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)), "read device error");
  if (reset) {
    const int z = 0;
    MX_CHECK_CUDA(cudaMemcpyToSymbol(g_device_error, &z, sizeof(int)), "reset device error");
  }
  *code = v;
  return MXMOE_OK;
}

int mxfp8_quantize(const void* x, int64_t batch, int64_t rows, int64_t cols, int modes, int scale_layout,
                   uint8_t* row_codes, uint8_t* row_scales, uint8_t* col_codes, uint8_t* col_scales,
                   cudaStream_t stream) {
  return quantize_impl(x, batch, rows, cols, modes, scale_layout, row_codes, row_scales, col_codes, col_scales,
                       stream);
}

int mxfp8_quantize_e5m2(const void* x, int64_t batch, int64_t rows, int64_t cols, int modes, int scale_layout,
                        uint8_t* row_codes, uint8_t* row_scales, uint8_t* col_codes, uint8_t* col_scales,
                        cudaStream_t stream) {
  return quantize_impl(x, batch, rows, cols, modes, scale_layout, row_codes, row_scales, col_codes, col_scales,
                       stream, false, 1);
}

int mxfp8_swiglu_quant(const void* h13, int64_t rows, int64_t F, int modes, int scale_layout, uint8_t* row_codes,
                       uint8_t* row_scales, uint8_t* col_codes, uint8_t* col_scales, cudaStream_t stream) {
  if (F % 32 != 0) return fail(MXMOE_ERR_SHAPE, "F=%lld must be a multiple of 32", (long long)F);
  return quantize_impl(h13, 1, rows, F, modes, scale_layout, row_codes, row_scales, col_codes, col_scales, stream,
                       true);
}

int mxfp8_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols, void* out,
                     cudaStream_t stream) {
  return dequantize_impl<0>(codes, scales, rows, cols, out, stream);
}

int mxfp8_dequantize_e5m2(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols, void* out,
                          cudaStream_t stream) {
  return dequantize_impl<1>(codes, scales, rows, cols, out, stream);
}

int mxfp8_grouped_gemm(const uint8_t* a, const uint8_t* a_scales, int64_t M, int64_t K, const uint8_t* w,
                       const uint8_t* w_scales, int E, int64_t N, const int32_t* expert_offsets, int pad_multiple,
                       void* out, cudaStream_t stream) {
  MX_TRY(check_offsets_args(expert_offsets, E, pad_multiple));
  MX_TRY(check_mult("M", M, 128));
  MX_TRY(check_mult("K", K, 128));
  MX_TRY(check_mult("N", N, 128));
  MX_TRY(check_ptrs({{"a", a}, {"a_scales", a_scales}, {"w", w}, {"w_scales", w_scales}, {"out", out}}));
  return gemm_ragged_m(a, a_scales, M, K, w, w_scales, E, N, expert_offsets, pad_multiple, out, stream);
}

int mxfp8_grouped_gemm_wgrad(const uint8_t* gt, const uint8_t* gt_scales, int64_t N, const uint8_t* xt,
                             const uint8_t* xt_scales, int64_t Kx, int64_t M, const int32_t* expert_offsets,
                             const int32_t* expert_rows, int E, int pad_multiple, void* dw, cudaStream_t stream) {
  MX_TRY(check_offsets_args(expert_offsets, E, pad_multiple));
  MX_TRY(check_mult("M", M, 128));
  MX_TRY(check_mult("N", N, 128));
  MX_TRY(check_mult("Kx", Kx, 128));
  MX_TRY(check_ptrs({{"gt", gt}, {"gt_scales", gt_scales}, {"xt", xt}, {"xt_scales", xt_scales}, {"dw", dw}}));
  return gemm_ragged_k(gt, gt_scales, N, xt, xt_scales, Kx, M, expert_offsets, expert_rows, E, pad_multiple, dw,
                       stream);
}

int mxfp8_grouped_gemm_swiglu_quant(const uint8_t* a, const uint8_t* a_scales, int64_t M, int64_t K,
                                    const uint8_t* w13, const uint8_t* w13_scales, int E, int64_t F,
                                    const int32_t* expert_offsets, int pad_multiple, void* h13_out,
                                    uint8_t* h_row_codes, uint8_t* h_row_scales, uint8_t* h_col_codes,
                                    uint8_t* h_col_scales, cudaStream_t stream) {
  MX_TRY(check_offsets_args(expert_offsets, E, pad_multiple));
  MX_TRY(check_mult("M", M, 128));
  MX_TRY(check_mult("K", K, 128));
  MX_TRY(check_mult("F", F, 128));
  MX_TRY(check_ptrs({{"a", a}, {"a_scales", a_scales}, {"w13", w13}, {"w13_scales", w13_scales},
                     {"h_row_codes", h_row_codes}, {"h_row_scales", h_row_scales}, {"h_col_codes", h_col_codes},
                     {"h_col_scales", h_col_scales}}));
  if (h13_out && !aligned16(h13_out)) return fail(MXMOE_ERR_ALIGN, "h13_out is not 16-byte aligned");
  return gemm_swiglu(a, a_scales, M, K, w13, w13_scales, E, F, expert_offsets, pad_multiple, h13_out, h_row_codes,
                     h_row_scales, h_col_codes, h_col_scales, stream);
}

int mxfp8_grouped_gemm_dswiglu_quant(const uint8_t* dy, const uint8_t* dy_scales, int64_t M, int64_t D,
                                     const uint8_t* w2t, const uint8_t* w2t_scales, int E, int64_t F,
                                     const int32_t* expert_offsets, int pad_multiple, const void* h13,
                                     uint8_t* g_row_codes, uint8_t* g_row_scales, uint8_t* g_col_codes,
                                     uint8_t* g_col_scales, cudaStream_t stream) {
  MX_TRY(check_offsets_args(expert_offsets, E, pad_multiple));
  MX_TRY(check_mult("M", M, 128));
  MX_TRY(check_mult("D", D, 128));
  MX_TRY(check_mult("F", F, 128));
  MX_TRY(check_ptrs({{"dy", dy}, {"dy_scales", dy_scales}, {"w2t", w2t}, {"w2t_scales", w2t_scales},
                     {"h13", h13}, {"g_row_codes", g_row_codes}, {"g_row_scales", g_row_scales},
                     {"g_col_codes", g_col_codes}, {"g_col_scales", g_col_scales}}));
  return gemm_dswiglu(dy, dy_scales, M, D, w2t, w2t_scales, E, F, expert_offsets, pad_multiple, h13, g_row_codes,
                      g_row_scales, g_col_codes, g_col_scales, stream);
}

size_t mxmoe_workspace_size(int64_t M, int64_t D, int E, int64_t F, int which) {
  if (M <= 0 || D <= 0 || E <= 0 || F <= 0) return 0;
  FwdWs f;
  BwdWs b;
  switch (which) {
    case 1: return carve_fwd(nullptr, M, D, E, F, &f, true);
    case 2: return carve_bwd(nullptr, M, D, E, F, &b, true);
    case 3: return carve_fwd(nullptr, M, D, E, F, &f, false);
    case 4: return carve_bwd(nullptr, M, D, E, F, &b, false);
    default: return 0;
  }
}

int mxmoe_quantize_weights(const void* w13, const void* w2, int E, int64_t D, int64_t F, const mxmoe_qweights* qw,
                           cudaStream_t stream) {
  if (E <= 0) return fail(MXMOE_ERR_SHAPE, "E=%d must be positive", E);
  MX_TRY(check_mult("D", D, 128));
  MX_TRY(check_mult("F", F, 128));
  MX_TRY(check_ptrs({{"w13", w13}, {"w2", w2}}));
  MX_TRY(check_qweights(qw, true, true));
  // W13[e] [2F, D]: ROW along D (FC1) and COL along 2F (dx), one read of W13
  MX_TRY(quantize_impl(w13, E, 2 * F, D, MXFP8_ROW | MXFP8_COL, MXFP8_SCALE_MMA, qw->w13_codes, qw->w13_scales,
                       qw->w13t_codes, qw->w13t_scales, stream));
  // W2[e] [D, F]: ROW along F (FC2) and COL along D (dh), one read of W2
  return quantize_impl(w2, E, D, F, MXFP8_ROW | MXFP8_COL, MXFP8_SCALE_MMA, qw->w2_codes, qw->w2_scales,
                       qw->w2t_codes, qw->w2t_scales, stream);
}

int moe_mlp_fwd(const void* x, int64_t M, int64_t D, const void* w13, const void* w2, int E, int64_t F,
                const int32_t* expert_offsets, int pad_multiple, void* y, const mxmoe_saved* saved, void* workspace,
                size_t workspace_bytes, cudaStream_t stream) {
  MX_TRY(check_mlp_shapes(M, D, E, F, expert_offsets, pad_multiple));
  MX_TRY(check_ptrs({{"x", x}, {"w13", w13}, {"w2", w2}, {"y", y}}));
  MX_TRY(check_saved(saved));
  FwdWs w;
  const size_t need = carve_fwd(nullptr, M, D, E, F, &w, true);
  if (!workspace || workspace_bytes < need)
    return fail(MXMOE_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes, need);
  carve_fwd(align_ws(workspace), M, D, E, F, &w, true);
  // a2: weights, ROW along the contraction dimension of each forward GEMM
  MX_TRY(quantize_impl(w13, 1, int64_t(E) * 2 * F, D, MXFP8_ROW, MXFP8_SCALE_MMA, w.qw.w13_codes, w.qw.w13_scales,
                       nullptr, nullptr, stream));
  MX_TRY(quantize_impl(w2, 1, int64_t(E) * D, F, MXFP8_ROW, MXFP8_SCALE_MMA, w.qw.w2_codes, w.qw.w2_scales, nullptr,
                       nullptr, stream));
  return fwd_core(x, M, D, w.qw, E, F, expert_offsets, pad_multiple, y, saved, w, stream);
}

int moe_mlp_bwd(const void* dy, int64_t M, int64_t D, const void* w13, const void* w2, int E, int64_t F,
                const int32_t* expert_offsets, int pad_multiple, const mxmoe_saved* saved, void* dx, void* dw13,
                void* dw2, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  MX_TRY(check_mlp_shapes(M, D, E, F, expert_offsets, pad_multiple));
  MX_TRY(check_ptrs({{"dy", dy}, {"w13", w13}, {"w2", w2}, {"dx", dx}, {"dw13", dw13}, {"dw2", dw2}}));
  MX_TRY(check_saved(saved));
  BwdWs w;
  const size_t need = carve_bwd(nullptr, M, D, E, F, &w, true);
  if (!workspace || workspace_bytes < need)
    return fail(MXMOE_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes, need);
  carve_bwd(align_ws(workspace), M, D, E, F, &w, true);
  // a2 (backward): W2 COL along D, W13 COL along 2F, per expert
  MX_TRY(quantize_impl(w2, E, D, F, MXFP8_COL, MXFP8_SCALE_MMA, nullptr, nullptr, w.qw.w2t_codes, w.qw.w2t_scales,
                       stream));
  MX_TRY(quantize_impl(w13, E, 2 * F, D, MXFP8_COL, MXFP8_SCALE_MMA, nullptr, nullptr, w.qw.w13t_codes,
                       w.qw.w13t_scales, stream));
  return bwd_core(dy, M, D, w.qw, E, F, expert_offsets, pad_multiple, saved, dx, dw13, dw2, w, stream);
}

int moe_mlp_fwd_q(const void* x, int64_t M, int64_t D, const mxmoe_qweights* qw, int E, int64_t F,
                  const int32_t* expert_offsets, int pad_multiple, void* y, const mxmoe_saved* saved,
                  void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  MX_TRY(check_mlp_shapes(M, D, E, F, expert_offsets, pad_multiple));
  MX_TRY(check_ptrs({{"x", x}, {"y", y}}));
  MX_TRY(check_qweights(qw, true, false));
  MX_TRY(check_saved(saved));
  FwdWs w;
  const size_t need = carve_fwd(nullptr, M, D, E, F, &w, false);
  if (!workspace || workspace_bytes < need)
    return fail(MXMOE_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes, need);
  carve_fwd(align_ws(workspace), M, D, E, F, &w, false);
  return fwd_core(x, M, D, *qw, E, F, expert_offsets, pad_multiple, y, saved, w, stream);
}

int moe_mlp_fwd_unfused_q(const void* x, int64_t M, int64_t D, const mxmoe_qweights* qw, int E, int64_t F,
                          const int32_t* expert_offsets, int pad_multiple, void* y, const mxmoe_saved* saved,
                          void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  MX_TRY(check_mlp_shapes(M, D, E, F, expert_offsets, pad_multiple));
  MX_TRY(check_ptrs({{"x", x}, {"y", y}}));
  MX_TRY(check_qweights(qw, true, false));
  MX_TRY(check_saved(saved));
  FwdWs w;
  const size_t need = carve_fwd(nullptr, M, D, E, F, &w, false);
  if (!workspace || workspace_bytes < need)
    return fail(MXMOE_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes, need);
  carve_fwd(align_ws(workspace), M, D, E, F, &w, false);
  MX_TRY(quantize_tokens(x, M, D, expert_offsets + E, w.x_rc, w.x_rs, saved->x_col_codes, saved->x_col_scales,
                         stream));
  // FC1 to a bf16 h13 in HBM ([gate | up] columns of the plain W13 rows)
  MX_TRY(gemm_ragged_m(w.x_rc, w.x_rs, M, D, qw->w13_codes, qw->w13_scales, E, 2 * F, expert_offsets, pad_multiple,
                       saved->h13, stream));
  // standalone SwiGLU + dual quantization of the rows below offsets[E]
  MX_TRY(launch_cast<kCastSwiglu>(saved->h13, 1, M, F, MXFP8_ROW | MXFP8_COL, MXFP8_SCALE_MMA, w.h_rc, w.h_rs,
                           saved->h_col_codes, saved->h_col_scales, expert_offsets + E, stream));
  return gemm_ragged_m(w.h_rc, w.h_rs, M, F, qw->w2_codes, qw->w2_scales, E, D, expert_offsets, pad_multiple, y,
                       stream);
}

int moe_mlp_bwd_q(const void* dy, int64_t M, int64_t D, const mxmoe_qweights* qw, int E, int64_t F,
                  const int32_t* expert_offsets, int pad_multiple, const mxmoe_saved* saved, void* dx, void* dw13,
                  void* dw2, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  MX_TRY(check_mlp_shapes(M, D, E, F, expert_offsets, pad_multiple));
  MX_TRY(check_ptrs({{"dy", dy}, {"dx", dx}, {"dw13", dw13}, {"dw2", dw2}}));
  MX_TRY(check_qweights(qw, false, true));
  MX_TRY(check_saved(saved));
  BwdWs w;
  const size_t need = carve_bwd(nullptr, M, D, E, F, &w, false);
  if (!workspace || workspace_bytes < need)
    return fail(MXMOE_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes, need);
  carve_bwd(align_ws(workspace), M, D, E, F, &w, false);
  return bwd_core(dy, M, D, *qw, E, F, expert_offsets, pad_multiple, saved, dx, dw13, dw2, w, stream);
}

}  // extern "C"

// Forward composite for callers that cannot allocate (see the header): the
// workspace is a static device array of this translation unit.  Host code
// cannot use the array's name as a device address, so its address is looked
// up with cudaGetSymbolAddress, once per device and CUDA context (a reset
// device or a new context gets a fresh lookup), and passed to the kernels.
static __device__ __align__(256) uint8_t g_noalloc_scratch[MXMOE_NOALLOC_SCRATCH_BYTES];

namespace {
using CtxGetCurrentFn = CUresult (*)(CUcontext*);

int current_context(CUcontext* ctx) {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  if (!fn) return fail(MXMOE_ERR_CUDA, "cuCtxGetCurrent unavailable");
  if (fn(ctx) != CUDA_SUCCESS) return fail(MXMOE_ERR_CUDA, "cuCtxGetCurrent failed");
  return MXMOE_OK;
}

struct ScratchAddr {
  CUcontext ctx = nullptr;
  void* ptr = nullptr;
};
ScratchAddr g_scratch[kMaxDevices];

int noalloc_scratch(void** out) {
  int dev = 0;
  MX_CHECK_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MXMOE_ERR_CUDA, "device index %d out of range", dev);
  CUcontext ctx = nullptr;
  MX_TRY(current_context(&ctx));
  std::lock_guard<std::mutex> lk(g_mu);
  ScratchAddr& a = g_scratch[dev];
  if (ctx == nullptr || a.ptr == nullptr || a.ctx != ctx) {
    void* p = nullptr;
    MX_CHECK_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress(scratch)");
    MX_TRY(current_context(&ctx));     // the lookup made the device's context current if it was not
    a.ctx = ctx;
    a.ptr = p;
  }
  *out = a.ptr;
  return MXMOE_OK;
}
}  // namespace

extern "C" int moe_mlp_fwd_noalloc(const void* x, int64_t M, int64_t D, const void* w13, const void* w2, int E,
                                   int64_t F, const int32_t* expert_offsets, int pad_multiple, void* y,
                                   const mxmoe_saved* saved, cudaStream_t stream) {
  MX_TRY(check_mlp_shapes(M, D, E, F, expert_offsets, pad_multiple));
  FwdWs w;
  const size_t need = carve_fwd(nullptr, M, D, E, F, &w, true);
  if (need > MXMOE_NOALLOC_SCRATCH_BYTES)
    return fail(MXMOE_ERR_WORKSPACE,
                "moe_mlp_fwd_noalloc: this layer needs %zu bytes of scratch, the static scratch holds %zu; "
                "use moe_mlp_fwd with a caller workspace",
                need, (size_t)MXMOE_NOALLOC_SCRATCH_BYTES);
  void* ws = nullptr;
  MX_TRY(noalloc_scratch(&ws));
  return moe_mlp_fwd(x, M, D, w13, w2, E, F, expert_offsets, pad_multiple, y, saved, ws,
                     MXMOE_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" {
// ---------------------------------------------------------------- dispatcher
int64_t mxmoe_route_capacity(int64_t T, int top_k, int E, int pad_multiple) {
  if (T < 0 || top_k <= 0 || E <= 0 || pad_multiple <= 0) return -1;
  if (T > (int64_t(1) << 40) / top_k) return -1;
  const int64_t n = T * top_k;
  const int64_t busy = n < E ? n : E;
  const int64_t cap = n + busy * (pad_multiple - 1);
  return (cap + 127) / 128 * 128;
}

size_t mxmoe_route_workspace_size(int64_t T, int top_k, int E) {
  if (T <= 0 || top_k <= 0 || E <= 0) return 0;
  const int64_t chunks = (T * top_k + kRouteChunk - 1) / kRouteChunk;
  return size_t(chunks) * size_t(E) * 4;
}

int mxmoe_route(const int32_t* topk_ids, int64_t T, int top_k, int E, int pad_multiple, int64_t m_cap,
                int32_t* offsets, int32_t* row_slot, int32_t* slot_row, void* workspace, size_t workspace_bytes,
                cudaStream_t stream) {
  if (!offsets) return fail(MXMOE_ERR_NULL, "offsets is NULL");
  if (T < 0 || top_k <= 0) return fail(MXMOE_ERR_SHAPE, "T=%lld top_k=%d", (long long)T, top_k);
  if (E <= 0 || E > kRouteMaxE) return fail(MXMOE_ERR_SHAPE, "E=%d must be in [1, %d]", E, kRouteMaxE);
  if (pad_multiple <= 0) return fail(MXMOE_ERR_ARG, "pad_multiple=%d must be positive", pad_multiple);
  if (m_cap < 0 || m_cap >= (int64_t(1) << 31)) return fail(MXMOE_ERR_SHAPE, "m_cap=%lld", (long long)m_cap);
  if (T > ((int64_t(1) << 31) - 1) / top_k) return fail(MXMOE_ERR_SHAPE, "T*top_k must be below 2^31");
  const int64_t n = T * top_k;
  if (n + int64_t(E) * (pad_multiple - 1) >= (int64_t(1) << 31))
    return fail(MXMOE_ERR_SHAPE, "T*top_k + E*(pad_multiple-1) must be below 2^31");
  if (n > 0 && (!topk_ids || !slot_row)) return fail(MXMOE_ERR_NULL, "topk_ids/slot_row is NULL");
  if (m_cap > 0 && !row_slot) return fail(MXMOE_ERR_NULL, "row_slot is NULL");
  const size_t need = mxmoe_route_workspace_size(T, top_k, E);
  if (need > 0 && (!workspace || workspace_bytes < need))
    return fail(MXMOE_ERR_WORKSPACE, "mxmoe_route needs %zu workspace bytes, got %zu", need, workspace_bytes);
  if (need > 0 && reinterpret_cast<uintptr_t>(workspace) % 4 != 0)
    return fail(MXMOE_ERR_ALIGN, "workspace is not 4-byte aligned");
  DevInfo* d;
  MX_TRY(device_info(&d));
  const int chunks = int((n + kRouteChunk - 1) / kRouteChunk);
  auto* counts = static_cast<int32_t*>(workspace);
  if (chunks > 0) {
    route_count_kernel<<<chunks, kRouteThreads, 0, stream>>>(topk_ids, n, E, counts);
    MX_CHECK_CUDA(cudaGetLastError(), "route count launch");
  }
  route_scan_kernel<<<1, kRouteThreads, 0, stream>>>(counts, chunks, E, pad_multiple, m_cap, offsets, row_slot);
  MX_CHECK_CUDA(cudaGetLastError(), "route scan launch");
  if (chunks > 0) {
    const int smem = E * 4 + 32 * E * 2;
    if (smem > 48 * 1024 && !(d->attr_set & (1u << 14))) {
      MX_CHECK_CUDA(cudaFuncSetAttribute(route_assign_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
                    "cudaFuncSetAttribute(route)");
      std::lock_guard<std::mutex> lk(g_mu);
      d->attr_set |= (1u << 14);
    }
    route_assign_kernel<<<chunks, kRouteThreads, smem, stream>>>(topk_ids, n, E, counts, m_cap, row_slot, slot_row);
    MX_CHECK_CUDA(cudaGetLastError(), "route assign launch");
  }
  return MXMOE_OK;
}

int mxmoe_permute_quant(const void* x_tokens, int64_t T, int64_t D, const int32_t* row_slot, int top_k,
                        const float* slot_weights, int64_t m_cap, const int32_t* rows_dev, int modes,
                        int scale_layout, uint8_t* row_codes, uint8_t* row_scales, uint8_t* col_codes,
                        uint8_t* col_scales, cudaStream_t stream) {
  if (!x_tokens || !row_slot) return fail(MXMOE_ERR_NULL, "x_tokens/row_slot is NULL");
  if (T < 0 || top_k <= 0 || D <= 0 || m_cap <= 0)
    return fail(MXMOE_ERR_SHAPE, "T=%lld top_k=%d D=%lld m_cap=%lld", (long long)T, top_k, (long long)D,
                (long long)m_cap);
  if (modes < 1 || modes > 3) return fail(MXMOE_ERR_ARG, "modes=%d must be MXFP8_ROW, MXFP8_COL or both", modes);
  if (scale_layout != MXFP8_SCALE_PLAIN && scale_layout != MXFP8_SCALE_MMA)
    return fail(MXMOE_ERR_ARG, "scale_layout=%d invalid", scale_layout);
  const bool row = modes & MXFP8_ROW, col = modes & MXFP8_COL;
  if (row && (!row_codes || !row_scales)) return fail(MXMOE_ERR_NULL, "row_codes/row_scales NULL with MXFP8_ROW");
  if (col && (!col_codes || !col_scales)) return fail(MXMOE_ERR_NULL, "col_codes/col_scales NULL with MXFP8_COL");
  if (D % 32 != 0 || m_cap % 32 != 0)
    return fail(MXMOE_ERR_SHAPE, "D=%lld and m_cap=%lld must be multiples of 32", (long long)D, (long long)m_cap);
  if (scale_layout == MXFP8_SCALE_MMA && (D % 128 != 0 || m_cap % 128 != 0))
    return fail(MXMOE_ERR_SHAPE, "MMA scale layout needs D and m_cap multiples of 128");
  if (!aligned16(x_tokens) || (row && !aligned16(row_codes)) || (col && !aligned16(col_codes)))
    return fail(MXMOE_ERR_ALIGN, "x_tokens and code buffers must be 16-byte aligned");
  if (scale_layout == MXFP8_SCALE_MMA && ((row && !aligned16(row_scales)) || (col && !aligned16(col_scales))))
    return fail(MXMOE_ERR_ALIGN, "MMA-layout scale buffers must be 16-byte aligned");
  if (T > 0x7FFFFFFF / top_k || m_cap >= (int64_t(1) << 31))
    return fail(MXMOE_ERR_SHAPE, "T*top_k and m_cap must be below 2^31");
  GatherArgs g{row_slot, slot_weights, T * top_k, top_k};
  return launch_cast<kCastGather>(x_tokens, 1, m_cap, D, modes, scale_layout, row_codes, row_scales, col_codes,
                                  col_scales, rows_dev, stream, &g);
}

static int check_combine_args(const void* a, const void* y, const int32_t* slot_row, const void* out, int64_t m_rows,
                              int64_t D, int64_t T, int top_k) {
  if (!a || !y || !slot_row || !out) return fail(MXMOE_ERR_NULL, "a required pointer is NULL");
  if (m_rows < 0 || D <= 0 || D % 8 != 0 || T < 0 || top_k <= 0 || top_k > 64)
    return fail(MXMOE_ERR_SHAPE, "m_rows=%lld D=%lld (multiple of 8) T=%lld top_k=%d (1..64)", (long long)m_rows,
                (long long)D, (long long)T, top_k);
  if (T > 0x7FFFFFFF) return fail(MXMOE_ERR_SHAPE, "T=%lld too large", (long long)T);
  if (!aligned16(a) || !aligned16(y)) return fail(MXMOE_ERR_ALIGN, "bf16 tensors must be 16-byte aligned");
  return MXMOE_OK;
}

int mxmoe_unpermute_combine(const void* y, int64_t m_rows, int64_t D, const int32_t* slot_row,
                            const float* slot_weights, int64_t T, int top_k, void* out, cudaStream_t stream) {
  MX_TRY(check_combine_args(out, y, slot_row, out, m_rows, D, T, top_k));
  DevInfo* d;
  MX_TRY(device_info(&d));
  if (T == 0) return MXMOE_OK;
  combine_kernel<<<unsigned(T), 256, 0, stream>>>(static_cast<const uint16_t*>(y), m_rows, slot_row, slot_weights,
                                                 top_k, D, static_cast<uint16_t*>(out));
  MX_CHECK_CUDA(cudaGetLastError(), "combine launch");
  return MXMOE_OK;
}

int mxmoe_combine_weight_grad(const void* dout, const void* y, int64_t m_rows, int64_t D, const int32_t* slot_row,
                              int64_t T, int top_k, float* dweights, cudaStream_t stream) {
  MX_TRY(check_combine_args(dout, y, slot_row, dweights, m_rows, D, T, top_k));
  DevInfo* d;
  MX_TRY(device_info(&d));
  if (T == 0) return MXMOE_OK;
  combine_weight_grad_kernel<<<unsigned(T), 256, 0, stream>>>(static_cast<const uint16_t*>(dout),
                                                             static_cast<const uint16_t*>(y), m_rows, slot_row,
                                                             top_k, D, dweights);
  MX_CHECK_CUDA(cudaGetLastError(), "combine weight-grad launch");
  return MXMOE_OK;
}

// ---------------------------------------------------------------- layer composites
size_t moe_layer_workspace_size(int64_t T, int top_k, int64_t D, int E, int64_t F, int pad_multiple, int which) {
  if (T <= 0 || top_k <= 0 || D <= 0 || E <= 0 || F <= 0 || pad_multiple <= 0) return 0;
  const int64_t m_cap = mxmoe_route_capacity(T, top_k, E, pad_multiple);
  if (m_cap <= 0) return 0;
  LayerFwdWs f;
  LayerBwdWs b;
  if (which == 1) return carve_layer_fwd(nullptr, T, top_k, m_cap, D, E, F, &f);
  if (which == 2) return carve_layer_bwd(nullptr, m_cap, D, E, F, &b);
  return 0;
}

int moe_layer_fwd_q(const void* x_tokens, int64_t T, int64_t D, const int32_t* topk_ids, const float* topk_weights,
                    int top_k, const mxmoe_qweights* qw, int E, int64_t F, int pad_multiple, void* out_tokens,
                    const mxmoe_layer_saved* saved, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  int64_t m_cap = 0;
  MX_TRY(check_layer_args(T, D, top_k, E, F, pad_multiple, &m_cap));
  MX_TRY(check_ptrs({{"x_tokens", x_tokens}, {"out_tokens", out_tokens}}));
  if (!topk_ids || !topk_weights) return fail(MXMOE_ERR_NULL, "topk_ids/topk_weights is NULL");
  MX_TRY(check_qweights(qw, true, false));
  MX_TRY(check_layer_saved(saved));
  LayerFwdWs w;
  const size_t need = carve_layer_fwd(nullptr, T, top_k, m_cap, D, E, F, &w);
  if (!workspace || workspace_bytes < need)
    return fail(MXMOE_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes, need);
  carve_layer_fwd(align_ws(workspace), T, top_k, m_cap, D, E, F, &w);
  const int32_t* rows_dev = saved->offsets + E;
  // routing -> padded expert-major layout
  MX_TRY(mxmoe_route(topk_ids, T, top_k, E, pad_multiple, m_cap, saved->offsets, saved->row_slot, saved->slot_row,
                     w.route_ws, size_t(route_chunks(T, top_k)) * E * 4 + 16, stream));
  // a1 fused with the gather: token rows -> x ROW (FC1) + COL (dW13, saved)
  GatherArgs g{saved->row_slot, nullptr, T * top_k, top_k};
  MX_TRY(launch_cast<kCastGather>(x_tokens, 1, m_cap, D, MXFP8_ROW | MXFP8_COL, MXFP8_SCALE_MMA, w.mlp.x_rc,
                                  w.mlp.x_rs, saved->mlp.x_col_codes, saved->mlp.x_col_scales, rows_dev, stream, &g));
  // a3, a4
  MX_TRY(gemm_swiglu(w.mlp.x_rc, w.mlp.x_rs, m_cap, D, qw->w13_codes, qw->w13_scales, E, F, saved->offsets,
                     pad_multiple, saved->mlp.h13, w.mlp.h_rc, w.mlp.h_rs, saved->mlp.h_col_codes,
                     saved->mlp.h_col_scales, stream));
  MX_TRY(gemm_ragged_m(w.mlp.h_rc, w.mlp.h_rs, m_cap, F, qw->w2_codes, qw->w2_scales, E, D, saved->offsets,
                       pad_multiple, saved->y, stream));
  // weighted combine back to token order
  return mxmoe_unpermute_combine(saved->y, m_cap, D, saved->slot_row, topk_weights, T, top_k, out_tokens, stream);
}

int moe_layer_bwd_q(const void* dout_tokens, int64_t T, int64_t D, const float* topk_weights, int top_k,
                    const mxmoe_qweights* qw, int E, int64_t F, int pad_multiple, const mxmoe_layer_saved* saved,
                    void* dx_tokens, void* dw13, void* dw2, float* dweights, void* workspace, size_t workspace_bytes,
                    cudaStream_t stream) {
  int64_t m_cap = 0;
  MX_TRY(check_layer_args(T, D, top_k, E, F, pad_multiple, &m_cap));
  MX_TRY(check_ptrs({{"dout_tokens", dout_tokens}, {"dx_tokens", dx_tokens}, {"dw13", dw13}, {"dw2", dw2}}));
  if (!topk_weights) return fail(MXMOE_ERR_NULL, "topk_weights is NULL");
  MX_TRY(check_qweights(qw, false, true));
  MX_TRY(check_layer_saved(saved));
  LayerBwdWs w;
  const size_t need = carve_layer_bwd(nullptr, m_cap, D, E, F, &w);
  if (!workspace || workspace_bytes < need)
    return fail(MXMOE_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes, need);
  carve_layer_bwd(align_ws(workspace), m_cap, D, E, F, &w);
  const int32_t* rows_dev = saved->offsets + E;
  // a5 fused with the gather: dY rows = bf16(w * dout[token]) -> ROW (dh) + COL (dW2)
  GatherArgs g{saved->row_slot, topk_weights, T * top_k, top_k};
  MX_TRY(launch_cast<kCastGather>(dout_tokens, 1, m_cap, D, MXFP8_ROW | MXFP8_COL, MXFP8_SCALE_MMA, w.mlp.dy_rc,
                                  w.mlp.dy_rs, w.mlp.dy_cc, w.mlp.dy_cs, rows_dev, stream, &g));
  const BwdWs& b = w.mlp;
  const mxmoe_saved* ms = &saved->mlp;
  // real rows per expert, from the route tables, for the weight gradients
  expert_rows_kernel<<<(E + 255) / 256, 256, 0, stream>>>(saved->offsets, saved->row_slot, E, m_cap, w.rows);
  MX_CHECK_CUDA(cudaGetLastError(), "expert rows launch");
  // a6 - a9
  MX_TRY(gemm_dswiglu(b.dy_rc, b.dy_rs, m_cap, D, qw->w2t_codes, qw->w2t_scales, E, F, saved->offsets, pad_multiple,
                      ms->h13, b.g_rc, b.g_rs, b.g_cc, b.g_cs, stream));
  MX_TRY(gemm_ragged_k(b.dy_cc, b.dy_cs, D, ms->h_col_codes, ms->h_col_scales, F, m_cap, saved->offsets, w.rows, E,
                       pad_multiple, dw2, stream));
  MX_TRY(gemm_ragged_m(b.g_rc, b.g_rs, m_cap, 2 * F, qw->w13t_codes, qw->w13t_scales, E, D, saved->offsets,
                       pad_multiple, w.dx_rows, stream));
  MX_TRY(gemm_ragged_k(b.g_cc, b.g_cs, 2 * F, ms->x_col_codes, ms->x_col_scales, D, m_cap, saved->offsets, w.rows, E,
                       pad_multiple, dw13, stream));
  // unpermute dx (sum over a token's copies) and the router-weight gradient
  MX_TRY(mxmoe_unpermute_combine(w.dx_rows, m_cap, D, saved->slot_row, nullptr, T, top_k, dx_tokens, stream));
  if (dweights)
    MX_TRY(mxmoe_combine_weight_grad(dout_tokens, saved->y, m_cap, D, saved->slot_row, T, top_k, dweights, stream));
  return MXMOE_OK;
}

}  // extern "C"
