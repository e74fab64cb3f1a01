// MXFP8 cast kernels: bf16 -> (E4M3 codes, E8M0 scales), row-wise and/or
// column-wise in one pass, plus the fused SwiGLU + dual quantization and the
// E8M0-endpoint-correct dequantization.
//
// Standalone casts: SwiGLU-boundary page, "Summary" (the unfused path's
// standalone cast kernels); A2E MXFP8 page ("the payload halves").
// Fused SwiGLU + dual quantization: SwiGLU-boundary page, "Summary".
// Dequantization: A2E transport page, review "[P2] Handle the two E8M0
// endpoint encodings before shifting".
//
// HBM-bound work: one 128 x 128 tile per CTA, 128-bit loads, the ROW pass in
// registers straight from the loads (4 lanes per 32-block, shuffle amax), the
// tile parked in shared memory for the COL pass (one thread per column block
// of 32 rows, stores of 32 contiguous codes).  With the MMA scale layout the
// tile's 512 scale bytes of each direction land in one contiguous atom.
#pragma once
#include "mx_common.cuh"

namespace mxmoe {

struct TileArgs {
  const uint16_t* in;   // bf16 input
  int64_t rows;         // rows of the (output) matrix per batch
  int64_t cols;         // columns of the quantized matrix (F for SwiGLU)
  int64_t ld_in;        // elements per input row (cols, or 2F for SwiGLU)
  int64_t up_off;       // SwiGLU: column offset of the up half (F)
  int modes;            // MXFP8_ROW | MXFP8_COL
  int mma_layout;       // 0 plain, 1 MMA
  uint8_t* row_codes;
  uint8_t* row_scales;
  uint8_t* col_codes;
  uint8_t* col_scales;
  const int32_t* dev_rows;  // optional: rows at or past *dev_rows are not read or written
};

constexpr int kTile = 128;
constexpr int kTileThreads = 256;

__device__ __forceinline__ uint4 ld_nc_v4(const uint16_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t swiglu_pair(uint32_t g, uint32_t u) {
  float h0 = silu_mul(bf16lo_to_f32(g), bf16lo_to_f32(u));
  float h1 = silu_mul(bf16hi_to_f32(g), bf16hi_to_f32(u));
  return pack_bf16x2(h0, h1);
}

template <bool kSwiglu>
__global__ void __launch_bounds__(kTileThreads)
mx_tile_kernel(TileArgs p) {
  __shared__ __align__(16) uint16_t tile[kTile][kTile];
  const int tid = threadIdx.x;
  const int64_t c0 = int64_t(blockIdx.x) * kTile;
  const int64_t r0 = int64_t(blockIdx.y) * kTile;
  const int64_t b = blockIdx.z;
  const int64_t rows = p.rows, cols = p.cols;
  const bool do_row = p.modes & 1;
  const bool do_col = p.modes & 2;
  const uint16_t* in = p.in + b * rows * p.ld_in;
  int64_t rows_lim = rows;
  if (p.dev_rows != nullptr) rows_lim = min(rows, int64_t(*p.dev_rows));

  // ---- load 8 chunks of 8 elements per thread (all loads first: ILP)
  uint4 v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int id = i * kTileThreads + tid;
    const int64_t row = r0 + (id >> 4);
    const int64_t col = c0 + (id & 15) * 8;
    if (row < rows_lim && col < cols) {
      v[i] = ld_nc_v4(in + row * p.ld_in + col);
    } else {
      v[i] = make_uint4(0, 0, 0, 0);
    }
  }
  if constexpr (kSwiglu) {
    uint4 u[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int id = i * kTileThreads + tid;
      const int64_t row = r0 + (id >> 4);
      const int64_t col = c0 + (id & 15) * 8;
      u[i] = (row < rows_lim && col < cols) ? ld_nc_v4(in + row * p.ld_in + p.up_off + col)
                                        : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[i].x = swiglu_pair(v[i].x, u[i].x);
      v[i].y = swiglu_pair(v[i].y, u[i].y);
      v[i].z = swiglu_pair(v[i].z, u[i].z);
      v[i].w = swiglu_pair(v[i].w, u[i].w);
    }
  }

  // ---- ROW pass (4 consecutive lanes hold one 32-block) + park in smem
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int id = i * kTileThreads + tid;
    const int rr = id >> 4, ch = id & 15;
    const int64_t row = r0 + rr;
    const int64_t col = c0 + ch * 8;
    if (do_row) {
      uint32_t am = absmax_bits8(v[i]);
      am = max(am, __shfl_xor_sync(0xffffffffu, am, 1));
      am = max(am, __shfl_xor_sync(0xffffffffu, am, 2));
      const uint32_t byte = scale_byte_from_bits(am);
      if (row < rows_lim && col < cols) {
        const int64_t R = b * rows + row;
        *reinterpret_cast<uint2*>(p.row_codes + R * cols + col) = encode8(v[i], byte);
        if ((ch & 3) == 0) {
          const int64_t off = p.mma_layout ? mma_scale_offset(R, col >> 5, cols)
                                           : R * (cols >> 5) + (col >> 5);
          p.row_scales[off] = uint8_t(byte);
        }
      }
    }
    if (do_col) *reinterpret_cast<uint4*>(&tile[rr][ch * 8]) = v[i];
  }
  if (!do_col) return;
  __syncthreads();

  // ---- COL pass: one thread per (column, 32-row block)
  const int64_t nrb = rows >> 5;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int task = i * kTileThreads + tid;
    const int c = task & 127, rb = task >> 7;
    const int64_t col = c0 + c;
    const int64_t rowb = r0 + rb * 32;
    if (col >= cols || rowb >= rows_lim) continue;
    uint4 w[4];
    uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
    for (int j = 0; j < 16; ++j)
      wp[j] = uint32_t(tile[rb * 32 + 2 * j][c]) | (uint32_t(tile[rb * 32 + 2 * j + 1][c]) << 16);
    uint32_t am = max(max(absmax_bits8(w[0]), absmax_bits8(w[1])),
                      max(absmax_bits8(w[2]), absmax_bits8(w[3])));
    const uint32_t byte = scale_byte_from_bits(am);
    const int64_t R = b * cols + col;
    uint2 q0 = encode8(w[0], byte), q1 = encode8(w[1], byte);
    uint2 q2 = encode8(w[2], byte), q3 = encode8(w[3], byte);
    uint8_t* dst = p.col_codes + R * rows + rowb;
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(q0.x, q0.y, q1.x, q1.y);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(q2.x, q2.y, q3.x, q3.y);
    const int64_t off = p.mma_layout ? mma_scale_offset(R, rowb >> 5, rows) : R * nrb + (rowb >> 5);
    p.col_scales[off] = uint8_t(byte);
  }
}

// Generic ROW cast for any column count (short last block): one warp per
// 32-element block, one element per lane.  Plain scale layout only.
__global__ void __launch_bounds__(256)
mx_row_generic_kernel(const uint16_t* __restrict__ in, int64_t R, int64_t cols,
                      uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t ncb = (cols + 31) >> 5;
  const int64_t w = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (w >= R * ncb) return;  // whole warp exits together
  const int64_t row = w / ncb, kb = w % ncb;
  const int64_t col = kb * 32 + lane;
  const bool valid = col < cols;
  const uint32_t bits = valid ? in[row * cols + col] : 0u;
  const uint32_t am = __reduce_max_sync(0xffffffffu, bits & 0x7FFFu);
  const uint32_t byte = scale_byte_from_bits(am);
  if (valid) {
    uint32_t code;
    if (byte == 0xFFu) {
      code = ((bits >> 8) & 0x80u) | 0x7Fu;
    } else {
      code = e4m3x2(__uint_as_float(bits << 16) * inv_scale_from_byte(byte), 0.f) & 0xFFu;
    }
    codes[row * cols + col] = uint8_t(code);
  }
  if (lane == 0) scales[row * ncb + kb] = uint8_t(byte);
}

// MXFP8 (ROW, plain scales) -> bf16: one thread per 8 elements where
// cols % 8 == 0, else per element.  E8M0 byte 0 decodes to 2^-127 and 0xFF
// to NaN.
__device__ __forceinline__ float e8m0_to_f32(uint32_t byte) {
  if (byte == 0xFFu) return __uint_as_float(0x7FC00000u);
  if (byte == 0u) return __uint_as_float(0x00400000u);  // 2^-127, an fp32 subnormal
  return __uint_as_float(byte << 23);
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  uint32_t h;
  asm("{ .reg .b16 c; cvt.u16.u32 c, %1; cvt.rn.f16x2.e4m3x2 %0, c; }" : "=r"(h) : "r"(code));
  return __half2float(__ushort_as_half(uint16_t(h & 0xFFFFu)));
}

__global__ void __launch_bounds__(256)
mx_dequant_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                  int64_t rows, int64_t cols, uint16_t* __restrict__ out) {
  const int64_t ncb = (cols + 31) >> 5;
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= rows * cols) return;
  const int64_t r = i / cols, c = i % cols;
  const float s = e8m0_to_f32(scales[r * ncb + (c >> 5)]);
  const float v = e4m3_to_f32(codes[i]) * s;
  out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

}  // namespace mxmoe
