// Device-side MXFP8 helpers shared by the cast and GEMM-epilogue kernels.
//
// MXFP8 block (A2E MXFP8 pages: E4M3 or E5M2 elements with an E8M0 block
// scale): 32 elements share one power-of-two scale 2^s with
// s = floor(log2(amax)) - emax (8 for E4M3, 15 for E5M2), stored as the byte
// s + 127 clamped to [0, 254]; elements are x / 2^s rounded to nearest-even
// and saturated (+-448, +-57344).  A block holding NaN/Inf gets byte 0xFF and
// codes 0x7F | sign.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace mxmoe {

constexpr int kBlock = 32;

// Device-side error word, one per device that loaded the library.
__device__ int g_device_error;

__device__ __forceinline__ void raise_device_error(int code) {
  atomicCAS(&g_device_error, 0, code);
}

// ---------------------------------------------------------------- bf16 bits
__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Round-to-nearest-even fp32 -> bf16 (hardware cvt), packed pair (lo = a).
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}

// max over |x| of eight packed bf16 (uint4) as a 15-bit magnitude pattern.
// For non-negative floats the integer order of the bit patterns is the
// numeric order, and NaN/Inf (>= 0x7F80) sort above every finite value.
__device__ __forceinline__ uint32_t absmax_bits8(uint4 v) {
  const uint32_t m = 0x7FFF7FFFu;
  uint32_t a = __vmaxu2(v.x & m, v.y & m);
  uint32_t b = __vmaxu2(v.z & m, v.w & m);
  a = __vmaxu2(a, b);
  return max(a & 0xFFFFu, a >> 16);
}

// E8M0 byte from the 15-bit magnitude pattern of the block maximum.
// floor(log2(amax)) is the unbiased exponent field, so the byte is
// max(expfield - 8, 0); subnormal or zero maxima land on 0 via the clamp.
// Returns 0xFF for NaN/Inf blocks.
__device__ __forceinline__ uint32_t scale_byte_from_bits(uint32_t amax_bits, int emax = 8) {
  if (amax_bits >= 0x7F80u) return 0xFFu;
  int e = int(amax_bits >> 7) - emax;
  return uint32_t(e < 0 ? 0 : e);
}

// 2^-(byte-127) as fp32 (exact; byte in [0, 254] -> exponent in [-127, 127]).
__device__ __forceinline__ float inv_scale_from_byte(uint32_t byte) {
  return __uint_as_float((254u - byte) << 23);
}

// Two fp32 -> two E4M3 codes (nearest-even, saturating), lo byte = a.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}
// Same for E5M2 (saturating at 57344).
__device__ __forceinline__ uint32_t e5m2x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}

// Element formats of an MXFP8 tensor: 0 = E4M3 (largest exponent 8),
// 1 = E5M2 (largest exponent 15).
template <int kElem>
__device__ __forceinline__ uint32_t fp8x2(float a, float b) {
  if constexpr (kElem == 0) return e4m3x2(a, b); else return e5m2x2(a, b);
}
template <int kElem>
__host__ __device__ constexpr int elem_emax() { return kElem == 0 ? 8 : 15; }

// Eight packed bf16 -> eight E4M3 codes (uint2), scaled by inv (a power of two).
__device__ __forceinline__ uint2 quant8_bf16(uint4 v, float inv) {
  uint2 out;
  out.x = e4m3x2(bf16lo_to_f32(v.x) * inv, bf16hi_to_f32(v.x) * inv) |
          (e4m3x2(bf16lo_to_f32(v.y) * inv, bf16hi_to_f32(v.y) * inv) << 16);
  out.y = e4m3x2(bf16lo_to_f32(v.z) * inv, bf16hi_to_f32(v.z) * inv) |
          (e4m3x2(bf16lo_to_f32(v.w) * inv, bf16hi_to_f32(v.w) * inv) << 16);
  return out;
}

// NaN codes (0x7F | sign) for eight packed bf16.
__device__ __forceinline__ uint2 nan8_bf16(uint4 v) {
  auto s = [](uint32_t w) {
    return ((w >> 8) & 0x80u) | ((w >> 16) & 0x8000u);
  };
  uint2 out;
  out.x = (s(v.x) | (s(v.y) << 16)) | 0x7F7F7F7Fu;
  out.y = (s(v.z) | (s(v.w) << 16)) | 0x7F7F7F7Fu;
  return out;
}

// Quantize 8 packed bf16 given the block's scale byte.
__device__ __forceinline__ uint2 encode8(uint4 v, uint32_t byte) {
  return byte == 0xFFu ? nan8_bf16(v) : quant8_bf16(v, inv_scale_from_byte(byte));
}

// ---------------------------------------------------------------- layouts
// Byte offset of the scale of row r, 32-column block kb in the MMA (tensor
// core) scale layout of a matrix with `kcols` columns (kcols % 128 == 0).
__device__ __forceinline__ int64_t mma_scale_offset(int64_t r, int64_t kb, int64_t kcols) {
  const int64_t atom = (r >> 7) * (kcols >> 7) + (kb >> 2);
  return atom * 512 + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (kb & 3);
}

// ---------------------------------------------------------------- SwiGLU
// sigmoid(a) = 1 / (1 + e^-a) with the fast exponential and division
// intrinsics (relative error a few fp32 ulp, far below the bf16 rounding the
// results go through; e^-a = inf gives exactly 0).
__device__ __forceinline__ float sigmoid_fast(float a) {
  return __fdividef(1.0f, 1.0f + __expf(-a));
}
// silu(a) * b in fp32 (rounded to bf16 by the caller).
__device__ __forceinline__ float silu_mul(float a, float b) {
  return a * sigmoid_fast(a) * b;
}

}  // namespace mxmoe
