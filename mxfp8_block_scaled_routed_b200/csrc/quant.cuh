// MXFP8 cast kernels: bf16 -> (E4M3 or E5M2 codes, E8M0 scales), row-wise
// and/or column-wise in one pass, plus the fused SwiGLU + dual quantization,
// the gather (token dispatcher) variant and the E8M0-endpoint-correct
// dequantization.
//
// Standalone casts: SwiGLU-boundary page, "Summary" (the unfused path's
// standalone cast kernels); A2E MXFP8 page ("the payload halves").
// Fused SwiGLU + dual quantization: SwiGLU-boundary page, "Summary".
// Dequantization: A2E transport page, review "[P2] Handle the two E8M0
// endpoint encodings before shifting".
//
// HBM-bound work: persistent CTAs, a TMA producer warp keeps 128 x 128 tiles
// streaming into shared memory while eight consumer warps quantize the
// previous ones (ROW pass: 4 lanes per 32-block, shuffle amax; COL pass: one
// thread per column pair of a 32-row block, stores of 32 contiguous codes).
// With the MMA scale layout the tile's 512 scale bytes of each direction land
// in one contiguous atom.
#pragma once
#include <cuda.h>
#include "mx_common.cuh"
#include "sm100.cuh"

namespace mxmoe {

struct CastArgs {
  int64_t rows;         // rows of the quantized matrix per batch
  int64_t cols;         // columns of the quantized matrix (F for SwiGLU)
  int64_t batch;
  int64_t up_off;       // SwiGLU: column offset of the up half in the input (F)
  int64_t tiles_c;      // 128-column tiles per row band
  int64_t tiles_r;      // 128-row tiles per batch
  int modes;            // MXFP8_ROW | MXFP8_COL
  int mma_layout;       // 0 plain, 1 MMA
  uint8_t* row_codes;
  uint8_t* row_scales;
  uint8_t* col_codes;
  uint8_t* col_scales;
  const int32_t* dev_rows;  // optional: rows at or past *dev_rows are neither read nor written
  // gather mode: row m of the quantized matrix is token row_slot[m] / top_k
  // of src ([*, cols] bf16, row stride cols), zero where row_slot[m] < 0;
  // with slot_weight, that row times slot_weight[row_slot[m]] rounded to bf16
  const uint16_t* src;
  const int32_t* row_slot;
  const float* slot_weight;
  int64_t n_slots;
  int top_k;
};

constexpr int kCastPlain = 0;    // TMA tiles of a [batch, rows, cols] tensor
constexpr int kCastSwiglu = 1;   // TMA gate + up tiles, h = silu(gate) * up
constexpr int kCastGather = 2;   // rows gathered by bulk copies through a slot table

constexpr int kTile = 128;
constexpr int kCastConsumers = 256;                 // 8 warps
constexpr int kCastThreads = kCastConsumers + 32;   // + 1 TMA producer warp
constexpr int kTileBytes = kTile * kTile * 2;       // one bf16 128 x 128 tile

template <int kMode>
struct CastCfg {
  static constexpr bool kSwiglu = kMode == kCastSwiglu;
  static constexpr int kStages = kSwiglu ? 1 : 2;       // SwiGLU: two CTAs per SM take turns instead
  static constexpr int kStageBytes = kSwiglu ? 2 * kTileBytes : kTileBytes;
  static constexpr int kOffColStage = kStages * kStageBytes;         // COL codes of one tile, 128 x 128 B
  static constexpr int kOffScales = kOffColStage + kTile * kTile;    // ROW then COL scale bytes, 512 B each
  static constexpr int kOffWeights = kOffScales + 1024;              // gather: per-row weights of each stage
  static constexpr int kOffPadMask = kOffWeights + (kMode == kCastGather ? kStages * kTile * 4 : 0);
  static constexpr int kOffBars = kOffPadMask + (kMode == kCastGather ? kStages * 16 : 0);
  static constexpr int kSmem = kOffBars + 2 * kStages * 8 + 128;     // + alignment slack
  static constexpr int kCtasPerSm = 2;
};

// bf16(w * x) for the two bf16 of a word (fp32 product, one rounding to bf16)
__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t x, float w) {
  return pack_bf16x2(w * bf16lo_to_f32(x), w * bf16hi_to_f32(x));
}

__device__ __forceinline__ uint32_t swiglu_pair(uint32_t g, uint32_t u) {
  float h0 = silu_mul(bf16lo_to_f32(g), bf16lo_to_f32(u));
  float h1 = silu_mul(bf16hi_to_f32(g), bf16hi_to_f32(u));
  return pack_bf16x2(h0, h1);
}

// The ROW and COL quantizers work on packed bf16 pairs.  The block maximum
// comes from max.NaN.xorsign.abs.bf16x2 (magnitude max of two bf16 pairs,
// NaN-propagating) on the bf16 bits, and the elements are scaled by the exact
// power of two 2^(127 - byte) in bf16x2 arithmetic: with byte <= 246 (every
// finite bf16 block) the factor is a bf16 normal and the product is exact
// unless it falls below 2^-126, where every E4M3/E5M2 code is +-0 anyway and
// the bf16 product keeps the sign.  The scaled pair is widened to fp32 and
// converted by cvt.rn.satfinite (nearest-even, saturating).
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
// bf16 bits of 2^(127 - byte) (byte <= 246).
__device__ __forceinline__ uint32_t bf16_inv_scale(uint32_t byte) { return (254u - byte) << 7; }

template <int kElem>
__device__ __forceinline__ uint2 row_quant8_packed(uint4 v, uint32_t* byte_out) {
  uint32_t a = bf16x2_absmax(bf16x2_absmax(v.x, v.y), bf16x2_absmax(v.z, v.w)) & 0x7FFF7FFFu;
  uint32_t m = max(a & 0xFFFFu, a >> 16);
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
  const uint32_t byte = scale_byte_from_bits(m, elem_emax<kElem>());
  *byte_out = byte;
  if (byte == 0xFFu) return nan8_bf16(v);
  const uint32_t s = bf16_inv_scale(byte) * 0x00010001u;
  const uint32_t x = bf16x2_mul(v.x, s), y = bf16x2_mul(v.y, s), z = bf16x2_mul(v.z, s), w = bf16x2_mul(v.w, s);
  uint2 o;
  auto cv = [](uint32_t t) { return fp8x2<kElem>(bf16lo_to_f32(t), bf16hi_to_f32(t)); };
  o.x = cv(x) | (cv(y) << 16);
  o.y = cv(z) | (cv(w) << 16);
  return o;
}

// Both columns of a 32-row block held as the two halves of w[0..31]: codes
// of the low-half column in q0, of the high-half column in q1; returns the
// two scale bytes (low | high << 8).
template <int kElem>
__device__ __forceinline__ uint32_t col_quant_pair32(const uint32_t (&w)[32], uint4 (&q0)[2], uint4 (&q1)[2]) {
  uint32_t a[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) a[j] = bf16x2_absmax(w[2 * j], w[2 * j + 1]);
#pragma unroll
  for (int st = 8; st >= 1; st >>= 1)
#pragma unroll
    for (int j = 0; j < st; ++j) a[j] = bf16x2_absmax(a[j], a[j + st]);
  const uint32_t m = a[0] & 0x7FFF7FFFu;
  const uint32_t b0 = scale_byte_from_bits(m & 0xFFFFu, elem_emax<kElem>());
  const uint32_t b1 = scale_byte_from_bits(m >> 16, elem_emax<kElem>());
  const uint32_t s = (b0 == 0xFFu ? 0u : bf16_inv_scale(b0)) | ((b1 == 0xFFu ? 0u : bf16_inv_scale(b1)) << 16);
  uint32_t c0[8], c1[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t x0 = bf16x2_mul(w[4 * k], s), x1 = bf16x2_mul(w[4 * k + 1], s);
    const uint32_t x2 = bf16x2_mul(w[4 * k + 2], s), x3 = bf16x2_mul(w[4 * k + 3], s);
    c0[k] = fp8x2<kElem>(bf16lo_to_f32(x0), bf16lo_to_f32(x1)) | (fp8x2<kElem>(bf16lo_to_f32(x2), bf16lo_to_f32(x3)) << 16);
    c1[k] = fp8x2<kElem>(bf16hi_to_f32(x0), bf16hi_to_f32(x1)) | (fp8x2<kElem>(bf16hi_to_f32(x2), bf16hi_to_f32(x3)) << 16);
  }
  if (b0 == 0xFFu || b1 == 0xFFu) {                 // NaN/Inf block: codes 0x7F | sign
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      uint32_t r0 = 0x7F7F7F7Fu, r1 = 0x7F7F7F7Fu;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        r0 |= ((w[4 * k + i] >> 15) & 1u) << (8 * i + 7);
        r1 |= (w[4 * k + i] >> 31) << (8 * i + 7);
      }
      if (b0 == 0xFFu) c0[k] = r0;
      if (b1 == 0xFFu) c1[k] = r1;
    }
  }
  q0[0] = make_uint4(c0[0], c0[1], c0[2], c0[3]);
  q0[1] = make_uint4(c0[4], c0[5], c0[6], c0[7]);
  q1[0] = make_uint4(c1[0], c1[1], c1[2], c1[3]);
  q1[1] = make_uint4(c1[4], c1[5], c1[6], c1[7]);
  return b0 | (b1 << 8);
}

// Persistent, TMA-fed cast.  Warp 8 streams 128 x 128 bf16 tiles (3-D tensor
// map [batch, rows, cols], zero fill past the edges) into a ring of shared
// memory stages; warps 0..7 quantize each tile straight from shared memory:
//  ROW: lane = 8 consecutive elements, 4 lanes = one 32-block (amax by two
//       shuffles), codes stored 8 bytes per lane (two 128-byte rows per warp
//       store);
//  COL: thread = two adjacent columns of one 32-row block (32 four-byte
//       shared loads), 32 codes per column stored as two 16-byte stores.
// SwiGLU: the gate and up tiles arrive together; the ROW pass computes
// h = bf16(silu(gate) * up), quantizes it and parks it over the gate tile
// for the COL pass (one barrier among the 256 consumer threads).
template <int kMode, int kElem = 0>
__global__ void __launch_bounds__(kCastThreads, CastCfg<kMode>::kCtasPerSm)
mx_cast_kernel(const __grid_constant__ CUtensorMap tin, const CastArgs p) {
  using C = CastCfg<kMode>;
  constexpr bool kSwiglu = kMode == kCastSwiglu, kGather = kMode == kCastGather;
  const bool weighted = kGather && p.slot_weight != nullptr;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint8_t* cstage = smem + C::kOffColStage;     // COL codes: column c at c*128, 16-byte chunk k at k ^ ((c>>1)&7)
  uint8_t* rsc = smem + C::kOffScales;          // ROW scales of the tile: [128 rows][4 blocks]
  uint8_t* csc = rsc + 512;                     // COL scales of the tile: [128 cols][4 blocks]
  float* wsm = reinterpret_cast<float*>(smem + C::kOffWeights);   // gather: [stage][row] weights
  uint32_t* padm = reinterpret_cast<uint32_t*>(smem + C::kOffPadMask);   // gather: [stage][4] pad-row bits
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t rows = p.rows, cols = p.cols;
  const int64_t ntiles = p.batch * p.tiles_r * p.tiles_c;
  int64_t rows_lim = rows;
  if (p.dev_rows != nullptr) rows_lim = min(rows, int64_t(*p.dev_rows));
  const bool do_row = p.modes & 1, do_col = p.modes & 2;
  // Tile sequence of this CTA.  TMA modes: grid stride.  Gather: a contiguous
  // run of the valid tiles (row bands below the device row limit), so that a
  // row band's slots are read once for all of its column tiles.
  int64_t t_begin = blockIdx.x, t_end = ntiles, t_step = gridDim.x;
  if constexpr (kGather) {
    const int64_t nvalid_tiles = min(ntiles, (max(rows_lim, int64_t(0)) + kTile - 1) / kTile * p.tiles_c);
    const int64_t per = (nvalid_tiles + gridDim.x - 1) / gridDim.x;
    t_begin = int64_t(blockIdx.x) * per;
    t_end = min(nvalid_tiles, t_begin + per);
    t_step = 1;
  }

  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      sm100::mbar_init(sm100::smem_u32(&bars[s]), 1);                                  // full
      sm100::mbar_init(sm100::smem_u32(&bars[C::kStages + s]), kCastConsumers / 32);  // empty
    }
    sm100::fence_mbar_init();
  }
  __syncthreads();

  const int64_t per_batch = p.tiles_r * p.tiles_c;
  if (kGather && warp == 8) {
    // ---------------- gather producer: lane g owns rows 4g..4g+3 of each
    // tile and fetches them with one four-row gather (tensor map over the
    // token matrix, box 128 x 1).  A pad row borrows a real row of its group
    // (the consumers zero it); a group without a real row is not fetched.
    if (lane == 0) sm100::prefetch_tmap(&tin);
    int stage = 0;
    uint32_t phase = 0;
    int64_t band = -1;
    int trow[4] = {0, 0, 0, 0};
    float wreg[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t padword = 0, ngroups = 0;
    bool fetch = false;
    for (int64_t t = t_begin; t < t_end; t += t_step) {
      const int64_t r0 = (t / p.tiles_c) * kTile, c0 = (t % p.tiles_c) * kTile;
      if (r0 >= rows_lim) continue;
      if (r0 != band) {                           // new row band: its slots, once
        band = r0;
        const int vrows = int(min(int64_t(kTile), rows_lim - r0));
        uint32_t pad = 0;
        int first = -1;
        int tok[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int rr = 4 * lane + i;
          int64_t sl = rr < vrows ? int64_t(p.row_slot[r0 + rr]) : -1;
          if (sl >= p.n_slots) {
            raise_device_error(4);
            sl = -1;
          }
          tok[i] = sl >= 0 ? int(sl / p.top_k) : -1;
          if (sl < 0) pad |= 1u << i;
          if (sl >= 0 && first < 0) first = tok[i];
          wreg[i] = (weighted && sl >= 0) ? p.slot_weight[sl] : 0.0f;
        }
        fetch = first >= 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) trow[i] = tok[i] >= 0 ? tok[i] : first;
        ngroups = __popc(__ballot_sync(0xffffffffu, fetch));
        // pad bits of rows 32w..32w+31 gathered into lane 8w
        uint32_t wd = pad << (4 * (lane & 7));
        wd |= __shfl_xor_sync(0xffffffffu, wd, 1);
        wd |= __shfl_xor_sync(0xffffffffu, wd, 2);
        wd |= __shfl_xor_sync(0xffffffffu, wd, 4);
        padword = wd;
      }
      bool ok = true;
      if (lane == 0) ok = sm100::mbar_wait(sm100::smem_u32(&bars[C::kStages + stage]), phase ^ 1);
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        if (lane == 0) raise_device_error(7);
        break;
      }
      if (weighted) {
#pragma unroll
        for (int i = 0; i < 4; ++i) wsm[stage * kTile + 4 * lane + i] = wreg[i];
      }
      if ((lane & 7) == 0) padm[stage * 4 + (lane >> 3)] = padword;
      __syncwarp();
      const uint32_t fb = sm100::smem_u32(&bars[stage]);
      if (lane == 0) sm100::mbar_arrive_expect_tx(fb, ngroups * 4u * kTile * 2u);
      __syncwarp();
      if (fetch)
        sm100::tma_gather4(sm100::smem_u32(smem + stage * C::kStageBytes + lane * 4 * 256), &tin, fb, int(c0),
                           trow[0], trow[1], trow[2], trow[3]);
      if (++stage == C::kStages) { stage = 0; phase ^= 1; }
    }
    return;
  }
  if (warp == 8) {
    // ---------------- producer
    if (lane == 0) {
      sm100::prefetch_tmap(&tin);
      int stage = 0;
      uint32_t phase = 0;
      for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
        const int64_t b = t / per_batch, rem = t - b * per_batch;
        const int64_t r0 = (rem / p.tiles_c) * kTile, c0 = (rem % p.tiles_c) * kTile;
        if (r0 >= rows_lim) continue;             // past the valid rows: never read
        if (!sm100::mbar_wait(sm100::smem_u32(&bars[C::kStages + stage]), phase ^ 1)) {
          raise_device_error(7);
          break;
        }
        const uint32_t fb = sm100::smem_u32(&bars[stage]);
        const uint32_t dst = sm100::smem_u32(smem + stage * C::kStageBytes);
        sm100::mbar_arrive_expect_tx(fb, C::kStageBytes);
        sm100::tma_load_3d(dst, &tin, fb, int(c0), int(r0), int(b));
        if constexpr (kSwiglu) sm100::tma_load_3d(dst + kTileBytes, &tin, fb, int(p.up_off + c0), int(r0), int(b));
        if (++stage == C::kStages) { stage = 0; phase ^= 1; }
      }
    }
    return;
  }

  // ---------------- consumers
  const int ch = tid & 15, rr0 = tid >> 4;      // ROW: chunk i = row i*16 + rr0, columns ch*8..ch*8+7
  const int cp = tid & 63, rb = tid >> 6;       // COL: columns 2cp, 2cp+1 of 32-row block rb
  const bool plain = p.mma_layout == 0;
  int stage = 0;
  uint32_t phase = 0;
  for (int64_t t = t_begin; t < t_end; t += t_step) {
    const int64_t b = t / per_batch, rem = t - b * per_batch;
    const int64_t r0 = (rem / p.tiles_c) * kTile, c0 = (rem % p.tiles_c) * kTile;
    if (r0 >= rows_lim) continue;
    if (!__all_sync(0xffffffffu, sm100::mbar_wait(sm100::smem_u32(&bars[stage]), phase))) {
      raise_device_error(7);
      break;
    }
    uint8_t* tile = smem + stage * C::kStageBytes;
    const int vrows = int(min(int64_t(kTile), rows_lim - r0));   // valid rows of the tile (multiple of 32 for COL)
    if constexpr (kGather) {
      // pad rows (and rows past the limit) hold a borrowed row or nothing: zero them
      const uint4 pm = *reinterpret_cast<const uint4*>(padm + stage * 4);
      if ((pm.x | pm.y | pm.z | pm.w) != 0u) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int idx = q * kCastConsumers + tid, row = idx >> 4;   // row = 8q + tid/16: word q/4
          const uint32_t w = q < 4 ? (q < 2 ? pm.x : pm.y) : (q < 6 ? pm.z : pm.w);
          if ((w >> (row & 31)) & 1u) reinterpret_cast<uint4*>(tile)[idx] = make_uint4(0u, 0u, 0u, 0u);
        }
        sm100::named_bar_sync(1, kCastConsumers);
      }
    }
    const int vcols = int(min(int64_t(kTile), cols - c0));       // valid columns (multiple of 32)

    // ---- ROW pass (and SwiGLU): codes straight to global, scales to shared
    if (do_row || kSwiglu || weighted) {
      const int64_t col = c0 + ch * 8;
      const int64_t Rb = b * rows + r0 + rr0;                    // matrix row of chunk 0
      uint8_t* rcode = p.row_codes + Rb * cols + col;            // advances 16 rows per chunk
#pragma unroll 2
      for (int i = 0; i < 8; ++i) {
        const int rr = i * 16 + rr0;
        uint8_t* srow = tile + rr * 256 + ch * 16;
        uint4 v = *reinterpret_cast<const uint4*>(srow);
        if constexpr (kSwiglu) {
          const uint4 u = *reinterpret_cast<const uint4*>(srow + kTileBytes);
          v.x = swiglu_pair(v.x, u.x);
          v.y = swiglu_pair(v.y, u.y);
          v.z = swiglu_pair(v.z, u.z);
          v.w = swiglu_pair(v.w, u.w);
          *reinterpret_cast<uint4*>(srow) = v;
        }
        if (weighted) {
          const float w = wsm[stage * kTile + rr];
          v.x = scale_bf16x2(v.x, w);
          v.y = scale_bf16x2(v.y, w);
          v.z = scale_bf16x2(v.z, w);
          v.w = scale_bf16x2(v.w, w);
          *reinterpret_cast<uint4*>(srow) = v;
        }
        if (do_row) {
          uint32_t byte;
          const uint2 q = row_quant8_packed<kElem>(v, &byte);
          if (rr < vrows && ch * 8 < vcols) {
            *reinterpret_cast<uint2*>(rcode + int64_t(i) * 16 * cols) = q;
            if ((ch & 3) == 0) rsc[rr * 4 + (ch >> 2)] = uint8_t(byte);
          }
        }
      }
    }
    if ((kSwiglu || weighted) && do_col) sm100::named_bar_sync(1, kCastConsumers);   // h parked for the COL pass

    // ---- COL pass: codes into the shared staging tile
    if (do_col) {
      if (rb * 32 < vrows && 2 * cp < vcols) {
        uint32_t w[32];
        const uint8_t* src = tile + (rb * 32) * 256 + cp * 4;
#pragma unroll
        for (int j = 0; j < 32; ++j) w[j] = *reinterpret_cast<const uint32_t*>(src + j * 256);
        uint4 qq[2][2];
        const uint32_t bytes = col_quant_pair32<kElem>(w, qq[0], qq[1]);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int c = 2 * cp + k;
          uint8_t* dst = cstage + c * 128;
          const int swz = cp & 7;
          *reinterpret_cast<uint4*>(dst + (((2 * rb) ^ swz) << 4)) = qq[k][0];
          *reinterpret_cast<uint4*>(dst + (((2 * rb + 1) ^ swz) << 4)) = qq[k][1];
          csc[c * 4 + rb] = uint8_t(bytes >> (8 * k));
        }
      }
    }
    // the input tile is no longer read: hand it back to the producer (after
    // ordering this thread's shared-memory writes into it, if any, before the
    // producer's next asynchronous copy into the same bytes)
    if constexpr (kSwiglu || kGather) sm100::fence_proxy_async();
    __syncwarp();
    if (lane == 0) sm100::mbar_arrive(sm100::smem_u32(&bars[C::kStages + stage]));
    if (++stage == C::kStages) { stage = 0; phase ^= 1; }
    sm100::named_bar_sync(1, kCastConsumers);                          // COL codes and scales staged

    // ---- write-out: whole 128-byte rows of COL codes, 16-byte scale stores
    if (do_col) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int qd = u * kCastConsumers + tid;                // 16-byte chunk id of the 16 KB tile
        const int c = qd >> 3, k = qd & 7;                      // output row (input column) c, chunk k
        if (c < vcols && k * 16 < vrows) {
          const uint4 v = *reinterpret_cast<const uint4*>(cstage + c * 128 + ((k ^ ((c >> 1) & 7)) << 4));
          *reinterpret_cast<uint4*>(p.col_codes + (b * cols + c0 + c) * rows + r0 + k * 16) = v;
        }
      }
    }
    if (do_row) {
      if (!plain) {
        // the tile's 128 rows x 4 blocks are exactly one 512-byte MMA atom:
        // atom byte (r%32)*16 + (r/32)*4 + kb  <-  staged byte r*4 + kb
        const int64_t atom = ((b * rows + r0) >> 7) * (cols >> 7) + (c0 >> 7);
        if (vrows == kTile) {
          if (tid < 32) {
            uint32_t wv[4];
#pragma unroll
            for (int g = 0; g < 4; ++g) wv[g] = *reinterpret_cast<const uint32_t*>(rsc + (g * 32 + tid) * 4);
            *reinterpret_cast<uint4*>(p.row_scales + atom * 512 + tid * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          }
        } else if (tid < vrows) {
          // a tile cut by the device row limit: only its valid rows' 4 bytes
          *reinterpret_cast<uint32_t*>(p.row_scales + atom * 512 + (tid & 31) * 16 + (tid >> 5) * 4) =
              *reinterpret_cast<const uint32_t*>(rsc + tid * 4);
        }
      } else if (tid < vrows) {
        const int nb = vcols >> 5;
        const int64_t R = b * rows + r0 + tid;
        uint8_t* d = p.row_scales + R * (cols >> 5) + (c0 >> 5);
        if (nb == 4 && (reinterpret_cast<uintptr_t>(d) & 3) == 0)
          *reinterpret_cast<uint32_t*>(d) = *reinterpret_cast<const uint32_t*>(rsc + tid * 4);
        else
          for (int kb = 0; kb < nb; ++kb) d[kb] = rsc[tid * 4 + kb];
      }
    }
    if (do_col) {
      if (!plain) {
        const int64_t atom = ((b * cols + c0) >> 7) * (rows >> 7) + (r0 >> 7);
        if (vrows == kTile) {
          if (tid >= 64 && tid < 96) {
            const int l = tid - 64;
            uint32_t wv[4];
#pragma unroll
            for (int g = 0; g < 4; ++g) wv[g] = *reinterpret_cast<const uint32_t*>(csc + (g * 32 + l) * 4);
            *reinterpret_cast<uint4*>(p.col_scales + atom * 512 + l * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          }
        } else if (tid >= 128) {
          // a tile cut by the device row limit: only the valid 32-row blocks
          const int c = tid - 128;
          for (int k = 0; k < (vrows >> 5); ++k) p.col_scales[atom * 512 + (c & 31) * 16 + (c >> 5) * 4 + k] = csc[c * 4 + k];
        }
      } else if (tid >= 128 && tid - 128 < vcols) {
        const int c = tid - 128;
        const int nb = vrows >> 5;
        const int64_t R = b * cols + c0 + c;
        uint8_t* d = p.col_scales + R * (rows >> 5) + (r0 >> 5);
        if (nb == 4 && (reinterpret_cast<uintptr_t>(d) & 3) == 0)
          *reinterpret_cast<uint32_t*>(d) = *reinterpret_cast<const uint32_t*>(csc + c * 4);
        else
          for (int k = 0; k < nb; ++k) d[k] = csc[c * 4 + k];
      }
    }
    // staging buffers are rewritten by the next tile
    sm100::named_bar_sync(1, kCastConsumers);
  }
}

// Generic ROW cast for any column count (short last block): one warp per
// 32-element block, one element per lane.  Plain scale layout only.
template <int kElem>
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
  const uint32_t byte = scale_byte_from_bits(am, elem_emax<kElem>());
  if (valid) {
    uint32_t code;
    if (byte == 0xFFu) {
      code = ((bits >> 8) & 0x80u) | 0x7Fu;
    } else {
      code = fp8x2<kElem>(__uint_as_float(bits << 16) * inv_scale_from_byte(byte), 0.f) & 0xFFu;
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

template <int kElem>
__device__ __forceinline__ float fp8_to_f32(uint32_t code) {
  uint32_t h;
  if constexpr (kElem == 0)
    asm("{ .reg .b16 c; cvt.u16.u32 c, %1; cvt.rn.f16x2.e4m3x2 %0, c; }" : "=r"(h) : "r"(code));
  else
    asm("{ .reg .b16 c; cvt.u16.u32 c, %1; cvt.rn.f16x2.e5m2x2 %0, c; }" : "=r"(h) : "r"(code));
  return __half2float(__ushort_as_half(uint16_t(h & 0xFFFFu)));
}

template <int kElem>
__global__ void __launch_bounds__(256)
mx_dequant_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                  int64_t rows, int64_t cols, uint16_t* __restrict__ out) {
  const int64_t ncb = (cols + 31) >> 5;
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= rows * cols) return;
  const int64_t r = i / cols, c = i % cols;
  const float s = e8m0_to_f32(scales[r * ncb + (c >> 5)]);
  const float v = fp8_to_f32<kElem>(codes[i]) * s;
  out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// Vector path (cols % 16 == 0, 16-B aligned codes and output): one thread
// per 16 codes, which share one scale.  The code's exponent and mantissa
// bits are placed in an fp32 word at the fp32 mantissa's top, so that the
// word reads as the code's value times 2^-120 (E4M3, exponent bias 7) or
// 2^-112 (E5M2, bias 15), normals and subnormals alike; multiplying by
// 2^(byte - bias) -- split in two factors when that power is not an fp32
// normal -- then rounds the exact product code * 2^(byte-127) once, exactly
// as the scalar path does.
template <int kElem>
struct Fp8Bits {
  static constexpr int kShift = kElem == 0 ? 20 : 21;     // code bit 0 -> fp32 bit
  static constexpr uint32_t kOff = kElem == 0 ? 120u : 112u;   // 127 - exponent bias
};

template <int kElem>
__device__ __forceinline__ uint32_t dequant_pair(uint32_t b0, uint32_t b1, float m1, float m2) {
  constexpr int sh = Fp8Bits<kElem>::kShift;
  const float y0 = __uint_as_float(((b0 & 0x80u) << 24) | ((b0 & 0x7Fu) << sh)) * m1 * m2;
  const float y1 = __uint_as_float(((b1 & 0x80u) << 24) | ((b1 & 0x7Fu) << sh)) * m1 * m2;
  const __nv_bfloat162 h = __floats2bfloat162_rn(y0, y1);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// bf16 of a code whose exponent field is all ones: E4M3 S.1111.111 is NaN;
// E5M2 S.11111.00 is +-infinity and S.11111.xx (xx != 0) NaN.
template <int kElem>
__device__ __forceinline__ uint32_t special_bf16(uint32_t c) {
  if constexpr (kElem == 0) return 0x7FFFu;
  else return (c & 3u) ? 0x7FFFu : (0x7F80u | ((c & 0x80u) << 8));
}

template <int kElem>
__device__ __forceinline__ void dequant_word(uint32_t w, float m1, float m2, uint32_t& lo, uint32_t& hi) {
  lo = dequant_pair<kElem>(w & 0xFFu, (w >> 8) & 0xFFu, m1, m2);
  hi = dequant_pair<kElem>((w >> 16) & 0xFFu, w >> 24, m1, m2);
  // bytes whose special-value field is all ones (E4M3: the low 7 bits; E5M2:
  // the 5 exponent bits) take their value from special_bf16
  constexpr uint32_t f = kElem == 0 ? 0x7Fu : 0x7Cu;
  constexpr uint32_t F4 = f * 0x01010101u, one = kElem == 0 ? 0x01010101u : 0x04040404u;
  if ((((w & F4) + one) & 0x80808080u) != 0u) {
    uint32_t v[4] = {lo & 0xFFFFu, lo >> 16, hi & 0xFFFFu, hi >> 16};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t c = (w >> (8 * j)) & 0xFFu;
      if ((c & f) == f) v[j] = special_bf16<kElem>(c);
    }
    lo = v[0] | (v[1] << 16);
    hi = v[2] | (v[3] << 16);
  }
}

template <typename Idx, int kElem>
__global__ void __launch_bounds__(256)
mx_dequant16_kernel(const uint4* __restrict__ codes, const uint8_t* __restrict__ scales, Idx n16, Idx chunks_per_row,
                    Idx ncb, uint4* __restrict__ out) {
  const Idx stride = Idx(gridDim.x) * blockDim.x;
  for (Idx i = Idx(blockIdx.x) * blockDim.x + threadIdx.x; i < n16; i += stride) {
    const Idx r = i / chunks_per_row, c = i - r * chunks_per_row;
    const uint32_t byte = __ldg(scales + r * ncb + (c >> 1));
    const uint4 q = __ldcs(codes + i);
    uint4 o0, o1;
    if (byte == 0xFFu) {
      o0 = o1 = make_uint4(0x7FFF7FFFu, 0x7FFF7FFFu, 0x7FFF7FFFu, 0x7FFF7FFFu);
    } else {
      constexpr uint32_t off = Fp8Bits<kElem>::kOff;
      const bool one = byte <= 254u - off;            // 2^(byte - bias) is an fp32 normal
      const float m1 = __uint_as_float(one ? (byte + off) << 23 : (byte + off - 127u) << 23);
      const float m2 = one ? 1.0f : __uint_as_float(254u << 23);
      dequant_word<kElem>(q.x, m1, m2, o0.x, o0.y);
      dequant_word<kElem>(q.y, m1, m2, o0.z, o0.w);
      dequant_word<kElem>(q.z, m1, m2, o1.x, o1.y);
      dequant_word<kElem>(q.w, m1, m2, o1.z, o1.w);
    }
    __stcs(out + 2 * i, o0);
    __stcs(out + 2 * i + 1, o1);
  }
}

}  // namespace mxmoe
