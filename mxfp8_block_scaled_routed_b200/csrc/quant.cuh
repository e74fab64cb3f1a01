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
// streaming into shared memory while consumer warps quantize the previous
// ones.  Each consumer warp owns a 32-row x 64-column sub-tile of a tile, so
// the warps never wait for each other: ROW blocks one per lane (no shuffles),
// COL blocks one column pair per lane, codes staged per warp and stored as
// whole 32-byte sectors, scale bytes written straight into their atoms.
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
constexpr int kCastGather = 2;   // rows gathered by four-row TMA gathers through a slot table

constexpr int kTile = 128;                          // tile columns (and rows, except SwiGLU)
constexpr int kTileBytes = kTile * kTile * 2;       // one bf16 128 x 128 tile
constexpr int kStagingBytes = 2048;                 // per consumer warp: 32 x 64 codes


// A tile is consumed by kWarpsPerTile warps, each owning a 32-row x
// 64-column sub-tile (rows 32*q.., columns 64*h..) from the moment the tile
// lands until it releases the stage: the warps never wait for one another.
// The 8 consumer warps of a CTA form groups that take tiles in turn (one
// group of 8 for 128-row tiles, two of 4 for the SwiGLU's 64-row tiles); two
// CTAs per SM with 2 stages each.  (One CTA per SM with 16 consumer warps and
// a 6-stage ring measured the same or slightly slower, interleaved in one
// process: 0.754 against 0.763 of HBM for the W13 dual cast.)
template <int kMode>
struct CastCfg {
  static constexpr bool kSwiglu = kMode == kCastSwiglu;
  static constexpr bool kGather = kMode == kCastGather;
  // plain / SwiGLU: each input tile arrives as two 64-column boxes in the
  // 128-byte TMA swizzle (16-byte chunk j of row r at chunk j ^ (r & 7)), so a
  // lane reading one row and a warp reading one column are both free of bank
  // conflicts.  Gather: 128 unswizzled rows of 256 bytes (four-row gathers).
  static constexpr bool kSwz = !kGather;
  static constexpr int kTileRows = kSwiglu ? 64 : 128;          // SwiGLU: gate + up of 64 rows per stage
  static constexpr int kQuarters = kTileRows / 32;
  static constexpr int kWarpsPerTile = 2 * kQuarters;
  static constexpr int kInputs = kSwiglu ? 2 : 1;
  static constexpr int kInputBytes = kTileRows * kTile * 2;     // one input tile
  static constexpr int kHalfBytes = kInputBytes / 2;            // one 64-column box of it
  static constexpr int kStageBytes = kInputs * kInputBytes;     // 32 KB
  // Gather: one CTA per SM with 16 consumer warps and 5 stages (160 KB of
  // token rows in flight per SM against the random-row DRAM latency; 15-17 %
  // faster than two CTAs of 8 warps and 2 stages at the DSv3 scale).  The TMA
  // casts keep two CTAs of 8 warps and 2 stages (the two configurations
  // measure within 1 % there).
  static constexpr bool kBig = kGather;
  static constexpr int kCtasPerSm = kBig ? 1 : 2;
  static constexpr int kConsumerWarps = kBig ? 16 : 8;
  static constexpr int kGroups = kConsumerWarps / kWarpsPerTile;
  static constexpr int kStages = kBig ? 5 : 2;
  static constexpr int kThreads = 32 * (kConsumerWarps + 1);   // + 1 producer warp
  static constexpr int kOffStaging = kStages * kStageBytes;
  static constexpr int kOffWeights = kOffStaging + kConsumerWarps * kStagingBytes;
  static constexpr int kOffPadMask = kOffWeights + (kGather ? kStages * kTile * 4 : 0);
  static constexpr int kOffBars = kOffPadMask + (kGather ? kStages * 16 : 0);
  static constexpr int kSmem = kOffBars + 2 * kStages * 8 + 1024;   // + 1024-byte alignment slack
  static_assert((kSmem + 1024) * kCtasPerSm <= 233472, "shared memory budget");
  static_assert(!kGather || kTileRows == 128, "the gather producer fetches 128-row tiles");
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
__device__ __forceinline__ uint32_t cvt_pair(uint32_t t) {
  return fp8x2<kElem>(bf16lo_to_f32(t), bf16hi_to_f32(t));
}

// One ROW block of 32 elements held by one lane as 16 packed bf16 words:
// returns the scale byte; c[j] holds the codes of elements 4j..4j+3.
template <int kElem>
__device__ __forceinline__ uint32_t quant_block32(const uint32_t (&w)[16], uint32_t (&c)[8]) {
  uint32_t a[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) a[j] = bf16x2_absmax(w[2 * j], w[2 * j + 1]);
#pragma unroll
  for (int st = 4; st >= 1; st >>= 1)
#pragma unroll
    for (int j = 0; j < st; ++j) a[j] = bf16x2_absmax(a[j], a[j + st]);
  const uint32_t m2 = a[0] & 0x7FFF7FFFu;
  const uint32_t byte = scale_byte_from_bits(max(m2 & 0xFFFFu, m2 >> 16), elem_emax<kElem>());
  if (byte == 0xFFu) {                               // NaN/Inf block: codes 0x7F | sign
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint2 n = nan8_bf16(make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]));
      c[2 * j] = n.x;
      c[2 * j + 1] = n.y;
    }
  } else {
    const uint32_t s = bf16_inv_scale(byte) * 0x00010001u;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      c[j] = cvt_pair<kElem>(bf16x2_mul(w[2 * j], s)) | (cvt_pair<kElem>(bf16x2_mul(w[2 * j + 1], s)) << 16);
  }
  return byte;
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

// Position (batch b, row tile tr, column tile tc) of tile t = t0 + i * step,
// advanced by additions: a 64-bit division per tile and thread would cost
// as much as quantizing a block.
struct TileWalk {
  int tc, tr, b;
  int dc, dr, db;
  int tiles_c, tiles_r;
  __device__ __forceinline__ TileWalk(int64_t t0, int64_t step, int64_t tiles_c_, int64_t tiles_r_)
      : tiles_c(int(tiles_c_)), tiles_r(int(tiles_r_)) {
    const int64_t per = tiles_c_ * tiles_r_;
    b = int(t0 / per);
    const int64_t rem = t0 - int64_t(b) * per;
    tr = int(rem / tiles_c_);
    tc = int(rem - int64_t(tr) * tiles_c_);
    db = int(step / per);
    const int64_t srem = step - int64_t(db) * per;
    dr = int(srem / tiles_c_);
    dc = int(srem - int64_t(dr) * tiles_c_);
  }
  __device__ __forceinline__ void next() {
    tc += dc;
    tr += dr;
    b += db;
    if (tc >= tiles_c) { tc -= tiles_c; ++tr; }
    if (tr >= tiles_r) { tr -= tiles_r; ++b; }
  }
};

// Per-warp staging buffer of 128 sixteen-byte chunks: chunk L at position
// L ^ ((L >> 3) & 3).  Written with chunk L = 4*lane + j (a lane's four
// chunks) and read with L = 32*k + lane, both patterns hit the 8 distinct
// 16-byte bank groups within every 8-lane phase.
__device__ __forceinline__ uint32_t staging_off(int L) { return uint32_t(L ^ ((L >> 3) & 3)) << 4; }

// Shared-memory accesses on 32-bit shared-window addresses (ld/st.shared,
// never the generic path).  volatile keeps them after the mbarrier waits.
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
// 32 words of one column pair, rows 0..31 of a 128-byte-swizzled sub-tile:
// row i's word sits at bases[i & 7] + 128 i, the row offset folded into the
// load's immediate.
template <int I = 0>
__device__ __forceinline__ void lds32_rows(uint32_t (&w)[32], const uint32_t (&bases)[8]) {
  asm volatile("ld.shared.u32 %0, [%1+%2];" : "=r"(w[I]) : "r"(bases[I & 7]), "n"(I * 128));
  if constexpr (I + 1 < 32) lds32_rows<I + 1>(w, bases);
}
__device__ __forceinline__ void sts64(uint32_t a, uint32_t x, uint32_t y) {
  asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// Persistent, TMA-fed cast.  The producer warp streams 128 x 128 bf16 tiles
// into a ring of shared-memory stages; each consumer warp quantizes its own
// 32 x 64 sub-tile of a tile and releases it, with no barrier among warps:
//  ROW: one lane per row, one 32-element block at a time (four 16-byte
//       loads, block maximum without shuffles), codes staged per warp and
//       stored as whole 32-byte sectors (8 rows x 64 bytes per store);
//  COL: one lane per column pair of the 32-row block (32 four-byte loads),
//       codes staged and stored as 16 columns x 32 bytes per store.
// SwiGLU: the ROW pass forms h = bf16(silu(gate) * up) from the gate and up
// tiles and parks it over the gate sub-tile for the COL pass.  Gather: rows
// arrive by four-row TMA gathers, unswizzled; the ROW pass there reads each
// lane's block in a rotated chunk order (conflict-free without the swizzle),
// zeroes pad rows and, with router weights, parks bf16(w * x) for the COL pass.
template <int kMode, int kElem>
__global__ void __launch_bounds__(CastCfg<kMode>::kThreads, CastCfg<kMode>::kCtasPerSm)
mx_cast_kernel(const __grid_constant__ CUtensorMap tin, const CastArgs p) {
  using C = CastCfg<kMode>;
  constexpr bool kSwiglu = C::kSwiglu, kGather = C::kGather;
  constexpr int S = C::kStages;
  const bool weighted = kGather && p.slot_weight != nullptr;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  float* wsm = reinterpret_cast<float*>(smem + C::kOffWeights);           // gather: [stage][row] weights
  uint32_t* padm = reinterpret_cast<uint32_t*>(smem + C::kOffPadMask);    // gather: [stage][4] pad-row bits
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t rows = p.rows, cols = p.cols;
  const int64_t ntiles = p.batch * p.tiles_r * p.tiles_c;
  int64_t rows_lim = rows;
  if (p.dev_rows != nullptr) rows_lim = min(rows, int64_t(*p.dev_rows));
  const bool do_row = p.modes & 1, do_col = p.modes & 2;
  // Tile order: a ROW-only cast walks the row tiles of a column band first
  // (measured 12 % faster on [8192, 7168]); the dual casts the column tiles
  // of a row band (the two orders measure the same), the gather its row bands.
  const bool row_fast = !kGather && !do_col;
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
    for (int s = 0; s < S; ++s) {
      sm100::mbar_init(sm100::smem_u32(&bars[s]), 1);        // full: the producer's arrival + bytes
      sm100::mbar_init(sm100::smem_u32(&bars[S + s]), C::kWarpsPerTile);   // empty: the consuming group's warps
    }
    sm100::fence_mbar_init();
  }
  __syncthreads();

  // Tiles past the valid rows are skipped by every role alike; n counts the
  // processed tiles: stage n % S (its (n / S)-th use), consumer group n % kGroups.
  if (kGather && warp == C::kConsumerWarps) {
    // ---------------- gather producer: lane g owns rows 4g..4g+3 of each
    // tile and fetches them with one four-row gather (tensor map over the
    // token matrix, box 128 x 1).  A pad row borrows a real row of its group
    // (the consumers zero it); a group without a real row is not fetched.
    if (lane == 0) sm100::prefetch_tmap(&tin);
    int64_t band = -1;
    int trow[4] = {0, 0, 0, 0};
    float wreg[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t padword = 0, ngroups = 0;
    bool fetch = false;
    int n = 0;
    TileWalk w(t_begin, t_step, p.tiles_c, p.tiles_r);
    for (int64_t t = t_begin; t < t_end; t += t_step, w.next()) {
      const int64_t r0 = int64_t(w.tr) * kTile, c0 = int64_t(w.tc) * kTile;
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
      const int s = n % S;
      const uint32_t ph = uint32_t(n / S) & 1u;
      ++n;
      bool ok = true;
      if (lane == 0) ok = sm100::mbar_wait(sm100::smem_u32(&bars[S + s]), ph ^ 1);
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        if (lane == 0) raise_device_error(7);
        break;
      }
      if (weighted) {
#pragma unroll
        for (int i = 0; i < 4; ++i) wsm[s * kTile + 4 * lane + i] = wreg[i];
      }
      if ((lane & 7) == 0) padm[s * 4 + (lane >> 3)] = padword;
      __syncwarp();
      const uint32_t fb = sm100::smem_u32(&bars[s]);
      if (lane == 0) sm100::mbar_arrive_expect_tx(fb, ngroups * 4u * kTile * 2u);
      __syncwarp();
      if (fetch)
        sm100::tma_gather4(sm100::smem_u32(smem + s * C::kStageBytes + lane * 4 * 256), &tin, fb, int(c0),
                           trow[0], trow[1], trow[2], trow[3]);
    }
    return;
  }
  if (warp == C::kConsumerWarps) {
    // ---------------- producer: two 64-column boxes per input tile
    if (lane == 0) {
      sm100::prefetch_tmap(&tin);
      int n = 0;
      TileWalk w(t_begin, t_step, row_fast ? p.tiles_r : p.tiles_c, row_fast ? p.tiles_c : p.tiles_r);
      for (int64_t t = t_begin; t < t_end; t += t_step, w.next()) {
        const int64_t b = w.b;
        const int64_t r0 = int64_t(row_fast ? w.tc : w.tr) * C::kTileRows, c0 = int64_t(row_fast ? w.tr : w.tc) * kTile;
        if (r0 >= rows_lim) continue;             // past the valid rows: never read
        const int s = n % S;
        const uint32_t ph = uint32_t(n / S) & 1u;
        ++n;
        if (!sm100::mbar_wait(sm100::smem_u32(&bars[S + s]), ph ^ 1)) {
          raise_device_error(7);
          break;
        }
        const uint32_t fb = sm100::smem_u32(&bars[s]);
        const uint32_t dst = sm100::smem_u32(smem + s * C::kStageBytes);
        sm100::mbar_arrive_expect_tx(fb, C::kStageBytes);
#pragma unroll
        for (int i = 0; i < C::kInputs; ++i)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
            sm100::tma_load_3d(dst + i * C::kInputBytes + hh * C::kHalfBytes, &tin, fb,
                               int((i ? p.up_off : 0) + c0 + 64 * hh), int(r0), int(b));
      }
    }
    return;
  }

  // ---------------- consumers
  const int grp = warp / C::kWarpsPerTile, wl = warp % C::kWarpsPerTile;
  const int q = wl % C::kQuarters, h = wl / C::kQuarters;   // rows 32q.., columns 64h.. of each tile
  const uint32_t sbase = sm100::smem_u32(smem);
  const uint32_t sb = sbase + C::kOffStaging + warp * kStagingBytes;
  const bool mma = p.mma_layout != 0;
  int n = 0;
  TileWalk w(t_begin, t_step, row_fast ? p.tiles_r : p.tiles_c, row_fast ? p.tiles_c : p.tiles_r);
  for (int64_t t = t_begin; t < t_end; t += t_step, w.next()) {
    const int64_t b = w.b;
    const int64_t r0 = int64_t(row_fast ? w.tc : w.tr) * C::kTileRows, c0 = int64_t(row_fast ? w.tr : w.tc) * kTile;
    if (r0 >= rows_lim) continue;
    const int s = n % S;
    const uint32_t ph = uint32_t(n / S) & 1u;
    const bool mine = (n % C::kGroups) == grp;
    ++n;
    if (!mine) continue;
    // lane 0 waits for the tile; __syncwarp orders the other lanes' reads after its acquire
    bool ok = true;
    if (lane == 0) ok = sm100::mbar_wait(sm100::smem_u32(&bars[s]), ph);
    __syncwarp();
    if (!__shfl_sync(0xffffffffu, ok, 0)) {
      if (lane == 0) raise_device_error(7);
      break;
    }
    const uint32_t tile = sbase + s * C::kStageBytes;
    const int vrows = int(min(int64_t(C::kTileRows), rows_lim - r0));   // valid rows of the tile (multiple of 32 for COL)
    const int vcols = int(min(int64_t(kTile), cols - c0));       // valid columns (multiple of 32)
    const int qrows = vrows - 32 * q;                            // valid rows of this warp's quarter (may exceed 32)
    const int hcols = vcols - 64 * h;                            // valid columns of this warp's half (may exceed 64)
    const bool active = qrows > 0 && hcols > 0;
    const int64_t R0 = b * rows + r0 + 32 * q;                   // matrix row of the sub-tile's first row
    const int qa = int((r0 & 127) >> 5) + q;                     // 32-row block of the sub-tile inside its 128-row MMA atom
    bool released = false;
    auto release = [&]() {
      // the stage is no longer read by this warp: hand it back (ordering this
      // warp's shared-memory writes into it, if any, before the producer's
      // next asynchronous copy into the same bytes)
      if constexpr (kSwiglu || kGather) sm100::fence_proxy_async();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(sm100::smem_u32(&bars[S + s]));
      released = true;
    };

    // ---- ROW pass (and the SwiGLU / gather transforms)
    if (active && (do_row || kSwiglu || kGather)) {
      if constexpr (C::kSwz) {
        const int rr = 32 * q + lane;            // tile row of this lane
        const uint32_t rp = tile + h * C::kHalfBytes + rr * 128;
        const int sw = rr & 7;
        const uint32_t rpx = rp | uint32_t(sw << 4);   // rp is 128-byte aligned
        uint32_t bytes = 0;
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          uint32_t w[16];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint4 v = lds128(rpx ^ uint32_t((4 * blk + k) << 4));
            w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
          }
          if constexpr (kSwiglu) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint4 u = lds128(rp + C::kInputBytes + (((4 * blk + k) ^ sw) << 4));
              w[4 * k] = swiglu_pair(w[4 * k], u.x);
              w[4 * k + 1] = swiglu_pair(w[4 * k + 1], u.y);
              w[4 * k + 2] = swiglu_pair(w[4 * k + 2], u.z);
              w[4 * k + 3] = swiglu_pair(w[4 * k + 3], u.w);
            }
            if (do_col) {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                sts128(rp + (((4 * blk + k) ^ sw) << 4), make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]));
            }
          }
          if (do_row) {
            uint32_t c[8];
            bytes |= quant_block32<kElem>(w, c) << (8 * blk);
            sts128(sb + staging_off(4 * lane + 2 * blk), make_uint4(c[0], c[1], c[2], c[3]));
            sts128(sb + staging_off(4 * lane + 2 * blk + 1), make_uint4(c[4], c[5], c[6], c[7]));
          }
        }
        if (!do_col) release();
        if (do_row) {
          // scales of this lane's row: blocks 2h, 2h+1 of the tile
          if (lane < qrows) {
            if (mma) {
              const int64_t atom = ((b * rows + r0) >> 7) * (cols >> 7) + (c0 >> 7);
              uint8_t* d = p.row_scales + atom * 512 + lane * 16 + qa * 4 + 2 * h;
              if (hcols >= 64) *reinterpret_cast<uint16_t*>(d) = uint16_t(bytes);
              else d[0] = uint8_t(bytes);
            } else {
              uint8_t* d = p.row_scales + (R0 + lane) * (cols >> 5) + (c0 >> 5) + 2 * h;
              d[0] = uint8_t(bytes);
              if (hcols >= 64) d[1] = uint8_t(bytes >> 8);
            }
          }
          __syncwarp();
          // staged codes -> 8 rows x 64 bytes per store
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int L = 32 * k + lane, sr = L >> 2, j = L & 3;
            if (sr < qrows && 16 * j < hcols)
              *reinterpret_cast<uint4*>(p.row_codes + (R0 + sr) * cols + c0 + 64 * h + 16 * j) = lds128(sb + staging_off(L));
          }
          __syncwarp();
        }
      } else {
        // gather: unswizzled 256-byte rows.  One lane per (row, 32-element
        // block): in pass it, lane l takes row 16*it + (l >> 1) of the quarter
        // and block l & 1 of the half, and reads the block's four 16-byte
        // chunks in the rotated order (j + rot) & 3, rot = (l >> 1) & 3, so the
        // 8 lanes of a phase hit 8 different bank groups.  The codes of each
        // chunk go to the staging buffer at that chunk's own position.
        const uint32_t pm = padm[s * 4 + q];
        const int blk = lane & 1, rot = (lane >> 1) & 3;
        const bool park = do_col;                 // pad zeros / weighted rows must be seen by the COL pass
#pragma unroll
        for (int it = 0; it < 2; ++it) {
          const int lr = 16 * it + (lane >> 1);
          const uint32_t rowa = tile + (32 * q + lr) * 256 + 128 * h + 64 * blk;
          uint32_t w[16];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 v = lds128(rowa + (((j + rot) & 3) << 4));
            w[4 * j] = v.x; w[4 * j + 1] = v.y; w[4 * j + 2] = v.z; w[4 * j + 3] = v.w;
          }
          const bool pad = (pm >> lr) & 1u;
          const uint32_t keep = pad ? 0u : 0xFFFFFFFFu;
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] &= keep;
          if (weighted) {
            const float wt = wsm[s * kTile + 32 * q + lr];
#pragma unroll
            for (int i = 0; i < 16; ++i) w[i] = scale_bf16x2(w[i], wt);
          }
          if (park && (pad || weighted)) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              sts128(rowa + (((j + rot) & 3) << 4), make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]));
          }
          if (do_row) {
            uint32_t c[8];
            const uint32_t byte = quant_block32<kElem>(w, c);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int jp = (j + rot) & 3;       // the chunk these 8 codes belong to
              sts64(sb + staging_off(4 * lr + 2 * blk + (jp >> 1)) + ((jp & 1) << 3), c[2 * j], c[2 * j + 1]);
            }
            if (lr < qrows && 32 * blk < hcols) {
              if (mma) {
                const int64_t atom = ((b * rows + r0) >> 7) * (cols >> 7) + (c0 >> 7);
                p.row_scales[atom * 512 + lr * 16 + qa * 4 + 2 * h + blk] = uint8_t(byte);
              } else {
                p.row_scales[(R0 + lr) * (cols >> 5) + (c0 >> 5) + 2 * h + blk] = uint8_t(byte);
              }
            }
          }
        }
        if (do_row) {
          __syncwarp();
          // staged codes -> 8 rows x 64 bytes per store
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int L = 32 * k + lane, sr = L >> 2, j = L & 3;
            if (sr < qrows && 16 * j < hcols)
              *reinterpret_cast<uint4*>(p.row_codes + (R0 + sr) * cols + c0 + 64 * h + 16 * j) = lds128(sb + staging_off(L));
          }
        }
        if (!do_col) release();
        __syncwarp();
      }
    }

    __syncwarp();                                  // parked rows visible to the whole warp

    // ---- COL pass: one lane per column pair (2*lane, 2*lane+1 of the half)
    if (active && do_col) {
      uint32_t w[32];
      if constexpr (C::kSwz) {
        const uint32_t cb = tile + h * C::kHalfBytes + 32 * q * 128 + ((lane & 3) << 2);
        uint32_t bases[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) bases[k] = cb + (((lane >> 2) ^ k) << 4);
        lds32_rows(w, bases);
      } else {
        const uint32_t cb = tile + 32 * q * 256 + 128 * h + 4 * lane;
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = lds32(cb + i * 256);
      }
      release();
      uint4 qq[2][2];
      const uint32_t bytes = col_quant_pair32<kElem>(w, qq[0], qq[1]);
#pragma unroll
      for (int k = 0; k < 2; ++k)
#pragma unroll
        for (int m = 0; m < 2; ++m) sts128(sb + staging_off(4 * lane + 2 * k + m), qq[k][m]);
      // scales of this lane's two columns, block q of the tile
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int ct = 64 * h + 2 * lane + k;    // tile column
        if (2 * lane + k < hcols) {
          const uint8_t v = uint8_t(bytes >> (8 * k));
          if (mma) {
            const int64_t atom = ((b * cols + c0) >> 7) * (rows >> 7) + (r0 >> 7);
            p.col_scales[atom * 512 + (ct & 31) * 16 + (ct >> 5) * 4 + qa] = v;
          } else {
            p.col_scales[(b * cols + c0 + ct) * (rows >> 5) + (r0 >> 5) + q] = v;
          }
        }
      }
      __syncwarp();
      // staged codes -> 16 columns x 32 bytes per store
      const int64_t cbase = b * cols + c0 + 64 * h;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int L = 32 * k + lane, c = L >> 1, m = L & 1;
        if (c < hcols)
          *reinterpret_cast<uint4*>(p.col_codes + (cbase + c) * rows + r0 + 32 * q + 16 * m) = lds128(sb + staging_off(L));
      }
      __syncwarp();
    }
    if (!released) release();
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
// per 16 codes, which share one scale.  Two codes at a time become f16 by
// cvt.rn.f16x2.{e4m3x2,e5m2x2} (exact: both formats fit in f16), then fp32,
// and one product with 2^(byte - 127) (exact, the subnormal 2^-127 included:
// the product of a code of at most 4 significant bits and a power of two is
// at least 2^-136) is rounded once to bf16 -- the correctly rounded value, as
// the scalar path gives.
template <int kElem>
__device__ __forceinline__ uint32_t fp8x2_to_f16x2(uint32_t pair) {
  uint32_t h;
  if constexpr (kElem == 0)
    asm("{ .reg .b16 c; cvt.u16.u32 c, %1; cvt.rn.f16x2.e4m3x2 %0, c; }" : "=r"(h) : "r"(pair));
  else
    asm("{ .reg .b16 c; cvt.u16.u32 c, %1; cvt.rn.f16x2.e5m2x2 %0, c; }" : "=r"(h) : "r"(pair));
  return h;
}

template <int kElem>
__device__ __forceinline__ uint32_t dequant_pair(uint32_t pair, float s) {
  const uint32_t h = fp8x2_to_f16x2<kElem>(pair);
  const float y0 = __half2float(__ushort_as_half(uint16_t(h & 0xFFFFu))) * s;
  const float y1 = __half2float(__ushort_as_half(uint16_t(h >> 16))) * s;
  const __nv_bfloat162 b = __floats2bfloat162_rn(y0, y1);
  return *reinterpret_cast<const uint32_t*>(&b);
}

// bf16 of a code whose exponent field is all ones: E4M3 S.1111.111 is NaN;
// E5M2 S.11111.00 is +-infinity and S.11111.xx (xx != 0) NaN.
template <int kElem>
__device__ __forceinline__ uint32_t special_bf16(uint32_t c) {
  if constexpr (kElem == 0) return 0x7FFFu;
  else return (c & 3u) ? 0x7FFFu : (0x7F80u | ((c & 0x80u) << 8));
}

template <int kElem>
__device__ __forceinline__ void dequant_word(uint32_t w, float s, uint32_t& lo, uint32_t& hi) {
  lo = dequant_pair<kElem>(w & 0xFFFFu, s);
  hi = dequant_pair<kElem>(w >> 16, s);
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

template <int kElem>
__device__ __forceinline__ void dequant16(const uint4 q, uint32_t byte, uint4& o0, uint4& o1) {
  if (byte == 0xFFu) {
    o0 = o1 = make_uint4(0x7FFF7FFFu, 0x7FFF7FFFu, 0x7FFF7FFFu, 0x7FFF7FFFu);
  } else {
    const float s = e8m0_to_f32(byte);
    dequant_word<kElem>(q.x, s, o0.x, o0.y);
    dequant_word<kElem>(q.y, s, o0.z, o0.w);
    dequant_word<kElem>(q.z, s, o1.x, o1.y);
    dequant_word<kElem>(q.w, s, o1.z, o1.w);
  }
}

// Grid-stride over 16-code chunks, four chunks per thread and iteration with
// their loads issued first, so each thread keeps 64 bytes of codes in flight.
template <typename Idx, int kElem>
__global__ void __launch_bounds__(256)
mx_dequant16_kernel(const uint4* __restrict__ codes, const uint8_t* __restrict__ scales, Idx n16, Idx chunks_per_row,
                    Idx ncb, uint4* __restrict__ out) {
  constexpr int kU = 4;
  const Idx stride = Idx(gridDim.x) * blockDim.x;
  for (Idx base = Idx(blockIdx.x) * blockDim.x + threadIdx.x; base < n16; base += kU * stride) {
    uint4 q[kU];
    uint32_t byte[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const Idx i = base + u * stride;
      if (i < n16) {
        const Idx r = i / chunks_per_row, c = i - r * chunks_per_row;
        byte[u] = __ldg(scales + r * ncb + (c >> 1));
        q[u] = __ldcs(codes + i);
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const Idx i = base + u * stride;
      if (i < n16) {
        uint4 o0, o1;
        dequant16<kElem>(q[u], byte[u], o0, o1);
        __stcs(out + 2 * i, o0);
        __stcs(out + 2 * i + 1, o1);
      }
    }
  }
}

}  // namespace mxmoe
