// Persistent MXFP8 grouped GEMM on the sm_100a tensor cores (tcgen05
// block-scaled MMA, fp32 accumulators in TMEM, TMA-fed shared-memory tiles).
//
// Covers the four grouped-GEMM ops of the fully-fused plan (torchtitan page
// "Wire the fully-fused grouped-GEMM MXFP8 plan behind fusion_plan", section
// "What it adds"): FC1 + SwiGLU + dual quantization, FC2, the dgrad with the
// fused dSwiGLU backward, and the wgrad over the ragged token dimension.
//
// Two schedules over the expert-major padded token layout:
//  * ragged M: out[m, :] = A[m, :] . B[e]^T for the rows m of expert e
//    (A = tokens x K, B = per-expert weights [E, N, K]); an M tile (128 rows,
//    256 on CTA pairs) never straddles two experts because segments are
//    padded to a multiple of it.  Zero-token experts own no M tile.
//  * ragged K: out[e] = A_e^T . B_e over expert e's token rows, with both
//    operands column-quantized and stored transposed ([N, M] and [Kx, M]) so
//    the token dimension is the contiguous contraction.  Experts without rows
//    write exact zeros.
//
// CTA = 12 warps: warp 0 issues TMA/bulk copies, warp 1 issues tcgen05.mma,
// warp 2 owns the TMEM allocation, warps 4..11 run the epilogue (warp 4+q and
// 8+q read TMEM lanes 32q..32q+31, i.e. rows 32q.. of the 128-row tile, each
// half of the columns).  Tile: 128 x BN x 128 (M x N x K bytes) per CTA,
// 128-byte swizzled K-major operands; on a CTA pair (cta_group::2) the two
// CTAs hold 128 rows each of a 256 x BN tile and one half of B each.
// The E8M0 scales arrive as 512-byte atoms (MMA scale layout), are copied to
// TMEM with tcgen05.cp and consumed by the block-scaled MMA (scale id = the
// 32-wide K step inside the 128-wide K block).
#pragma once
#include <cuda.h>
#include "mx_common.cuh"
#include "sm100.cuh"
#include "quant.cuh"

namespace mxmoe::gemm {

using namespace mxmoe::sm100;

enum Mode : int { kRaggedM = 0, kRaggedK = 1 };
enum Epi : int { kEpiBF16 = 0, kEpiSwiGLU = 1, kEpiDSwiGLU = 2 };

constexpr int kErrOffsets = 4;
constexpr int kErrTimeout = 7;

struct Params {
  int E;
  int64_t rows_a;     // ragged M: M (token rows); ragged K: N (rows of A^T)
  int64_t kext;       // K extent of A and B (ragged M: K; ragged K: M)
  int64_t n_out;      // ragged M: N (B rows per expert; 2F for SwiGLU); ragged K: Kx
  int64_t M;          // token rows of the buffer (bounds the offsets)
  const int32_t* offsets;
  const int32_t* rows;    // ragged K, optional: real (token) rows at the head of each expert's segment
  int pad;
  const uint8_t* a_scales;
  const uint8_t* b_scales;
  // epilogue
  uint16_t* out;          // bf16 output (BF16 epilogue), h13 out (SwiGLU, may be null)
  const uint16_t* h13;    // dSwiGLU input
  int64_t F;              // SwiGLU / dSwiGLU intermediate size
  uint8_t* row_codes;
  uint8_t* row_scales;
  uint8_t* col_codes;
  uint8_t* col_scales;
};

// kPair: the CTA pair (cluster of 2, cta_group::2) computes a 256 x BN tile;
// each CTA holds 128 rows of A, half of the BN rows of B and its own
// 128 x BN accumulator.
template <int kMode, int kEpi, int BN, bool kPair>
struct Cfg {
  static constexpr int BM = 128, BK = 128;
  static constexpr int kAcc = (BN == 256) ? 1 : 2;
  static constexpr int B_ROWS = kPair ? BN / 2 : BN;           // B rows loaded per CTA and stage
  static constexpr int A_BYTES = BM * BK;
  static constexpr int B_BYTES = B_ROWS * BK;
  static constexpr int SFA_BYTES = 512;
  static constexpr int SFB_BYTES = (BN / 128) * 512;          // scales of all BN rows of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  // (the dSwiGLU epilogue's larger staging tile costs one stage)
  static constexpr int kStages = (kPair ? ((BN == 256) ? 6 : 7) : ((BN == 256) ? 4 : 6)) - (kEpi == kEpiDSwiGLU ? 1 : 0);
  static constexpr int SF_COLS = 4 + BN / 32;           // TMEM columns for one SF buffer
  static constexpr int ACC_COLS = kAcc * BN;
  static constexpr int TMEM_COLS = 512;
  static_assert(ACC_COLS + 2 * SF_COLS <= TMEM_COLS, "TMEM budget");
  static_assert(!kPair || BN == 256 || BN == 128, "CTA pair tile widths");
  // shared memory map (offsets from a 1024-aligned base)
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + kStages * A_BYTES;
  static constexpr int OFF_SFA = OFF_B + kStages * B_BYTES;
  static constexpr int OFF_SFB = OFF_SFA + kStages * SFA_BYTES;
  static constexpr int OFF_EPI = OFF_SFB + kStages * SFB_BYTES;
  static constexpr int EPI_WARPS = 8;
  // per epilogue warp: 32x32 bf16 transpose / staging buffer; dSwiGLU: the
  // 32 x 64 bf16 dgate|dup tile (then its COL codes) and the ROW codes (512-aligned)
  static constexpr int EPI_WARP_BYTES = (kEpi == kEpiDSwiGLU) ? 6144 : 2560;
  static constexpr int EPI_BYTES = EPI_WARPS * EPI_WARP_BYTES;
  static constexpr int OFF_BAR = OFF_EPI + EPI_BYTES;
  static constexpr int NUM_BARS = 2 * kStages + 2 * kAcc;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_OFFS = OFF_MISC + 16;
  static constexpr int MAX_E = 1024;
  static constexpr int SMEM_BYTES = OFF_OFFS + (MAX_E + 1) * 4 + 1024;  // + alignment slack
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// ---------------------------------------------------------------- tile schedule
struct Tile {
  int e;
  int nk;           // K blocks of 128
  int64_t a_row;    // first A row loaded by this CTA
  int64_t b_row0;   // first B row of the tile's first 128-row box (scales)
  int64_t b_row1;   // first B row of the second box (BN == 256)
  int64_t b_mine;   // CTA pair: the B box this CTA loads
  int64_t k0;       // first K element
  int64_t out_r0;   // first output row of this CTA
  int64_t out_c0;   // first output column (SwiGLU: first f)
};

template <int kMode, int kEpi, int BN, bool kPair>
__device__ __forceinline__ int64_t num_tiles(const Params& p, const int32_t* offs) {
  constexpr int PM = kPair ? 256 : 128;
  if constexpr (kMode == kRaggedM) {
    const int64_t nt = (kEpi == kEpiSwiGLU) ? p.F / 128 : p.n_out / BN;
    return (int64_t(offs[p.E]) / PM) * nt;
  } else {
    return int64_t(p.E) * (p.rows_a / PM) * (p.n_out / BN);
  }
}

// The tiles t0, t0 + step, ... of one CTA (or CTA pair), in order.
//   ragged M: t = mt * nt + j (m tile, n tile), decoded per tile; e is the
//             last expert with offs[e] <= the tile's first row.  Its tiles
//             run the whole K extent, so the decode is a small part of one.
//   ragged K: t = (e * n1 + nt) * n2 + jt (expert, output row tile, column
//             tile); the coordinates advance by additions.  Decoding them
//             with 64-bit divisions took several hundred cycles per tile on
//             every role's thread, and the weight gradients run tiles of one
//             or two K blocks (~700 cycles each).
template <int kMode, int kEpi, int BN, bool kPair>
struct TileIter {
  static constexpr int PM = kPair ? 256 : 128;
  int64_t t, step;
  int64_t n1, n2;      // ragged K: output row tiles per expert, column tiles
  int64_t c1, c2;      // ragged K: (nt, jt)
  int64_t d1, d2, d0;  // per-step increments of c1, c2 and e
  int e;

  __device__ __forceinline__ TileIter(const Params& p, const int32_t* offs, int64_t t0, int64_t step_)
      : t(t0), step(step_) {
    if constexpr (kMode == kRaggedK) {
      // (extents clamped to 1 for the divisions: a zero extent means no tiles)
      n1 = max(int64_t(1), p.rows_a / PM);
      n2 = max(int64_t(1), p.n_out / BN);
      const int64_t q = t0 / n2, qs = step / n2;
      c2 = t0 % n2;
      c1 = q % n1;
      e = int(q / n1);
      d2 = step % n2;
      d1 = qs % n1;
      d0 = qs / n1;
    }
  }
  __device__ __forceinline__ void next(const Params&, const int32_t*) {
    t += step;
    if constexpr (kMode == kRaggedK) {
      c2 += d2;
      c1 += d1;
      if (c2 >= n2) { c2 -= n2; ++c1; }
      e += int(d0);
      if (c1 >= n1) { c1 -= n1; ++e; }
    }
  }
};

template <int kMode, int kEpi, int BN, bool kPair>
__device__ __forceinline__ Tile get_tile(const Params& p, const int32_t* offs, const TileIter<kMode, kEpi, BN, kPair>& it,
                                         int rank) {
  constexpr int PM = kPair ? 256 : 128;
  Tile T;
  if constexpr (kMode == kRaggedM) {
    const int64_t nt = (kEpi == kEpiSwiGLU) ? p.F / 128 : p.n_out / BN;
    const int64_t mt = it.t / nt, ntile = it.t % nt;
    const int64_t m0 = mt * PM;
    int lo = 0, hi = p.E;  // last e with offs[e] <= m0
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (offs[mid] <= m0) lo = mid; else hi = mid;
    }
    T.e = lo;
    T.nk = int(p.kext / 128);
    T.k0 = 0;
    T.a_row = m0 + rank * 128;
    T.out_r0 = T.a_row;
    if constexpr (kEpi == kEpiSwiGLU) {
      const int64_t f0 = ntile * 128;
      T.b_row0 = int64_t(T.e) * 2 * p.F + f0;          // gate rows
      T.b_row1 = int64_t(T.e) * 2 * p.F + p.F + f0;    // up rows
      T.out_c0 = f0;
    } else {
      T.b_row0 = int64_t(T.e) * p.n_out + ntile * BN;
      T.b_row1 = T.b_row0 + 128;
      T.out_c0 = ntile * BN;
    }
  } else {
    const int e = it.e;
    T.e = e;
    // low 7 bits of offs[e]: trailing 128-row K blocks of the segment that
    // hold only padding (set when the real row counts are given)
    T.k0 = offs[e] & ~127;
    T.nk = int(((offs[e + 1] & ~127) - T.k0) / 128) - (offs[e] & 127);
    T.a_row = it.c1 * PM + rank * 128;
    T.b_row0 = it.c2 * BN;
    T.b_row1 = it.c2 * BN + 128;
    T.out_r0 = T.a_row;
    T.out_c0 = it.c2 * BN;
  }
  if constexpr (kEpi == kEpiSwiGLU)
    T.b_mine = rank ? T.b_row1 : T.b_row0;          // gate rows on the even CTA, up rows on the odd one
  else
    T.b_mine = T.b_row0 + rank * (BN / 2);
  return T;
}

// ---------------------------------------------------------------- epilogue helpers
// Warp-level 32x32 transpose through shared memory: each lane gives one row
// of 16 packed bf16 pairs; each lane gets one column as 16 packed pairs.
// Row stride 17 words keeps both phases free of bank conflicts.
__device__ __forceinline__ void warp_transpose32(uint32_t* buf, const uint32_t* row, uint32_t (&col)[16],
                                                 int lane) {
#pragma unroll
  for (int j = 0; j < 16; ++j) buf[lane * 17 + j] = row[j];
  __syncwarp();
  const int w = lane >> 1, sh = (lane & 1) * 16;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t lo = (buf[(2 * j) * 17 + w] >> sh) & 0xFFFFu;
    const uint32_t hi = (buf[(2 * j + 1) * 17 + w] >> sh) & 0xFFFFu;
    col[j] = lo | (hi << 16);
  }
  __syncwarp();
}

// The warp's staging buffer may still be read by this warp's last TMA store:
// wait for that read before rewriting it.
__device__ __forceinline__ void sbuf_acquire(int lane) {
  if (lane == 0) bulk_wait_read_all();
  __syncwarp();
}

// Store a 32-row x 32-column bf16 block (one row per lane, 4 x 16 B in v) with
// one asynchronous TMA store: the block is written to the warp's staging
// buffer in the tensor map's 64-byte swizzle (16-byte chunk c of row r at
// chunk c ^ ((r >> 1) & 3), conflict-free) and lane 0 hands it to the TMA
// engine; the warp continues without waiting for the global write.
__device__ __forceinline__ void store_block_tma(uint8_t* sbuf, const uint32_t* v, const void* tmap, int x, int y,
                                                int lane) {
  sbuf_acquire(lane);
#pragma unroll
  for (int c = 0; c < 4; ++c)
    *reinterpret_cast<uint4*>(sbuf + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)) =
        make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
  fence_proxy_async();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tmap, smem_u32(sbuf), x, y);
    bulk_commit();
  }
}

// Same for a 32-row x 32-byte block (one row per lane, 2 x 16 B in v):
// chunk c of row r sits at chunk c ^ ((r >> 2) & 1); each store instruction
// writes 16 whole 32-byte row segments.
__device__ __forceinline__ void store_rows32(uint8_t* sbuf, const uint4 (&v)[2], uint8_t* dst0, int64_t ld,
                                             int lane) {
  sbuf_acquire(lane);
#pragma unroll
  for (int c = 0; c < 2; ++c)
    *reinterpret_cast<uint4*>(sbuf + lane * 32 + ((c ^ ((lane >> 2) & 1)) << 4)) = v[c];
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = 16 * i + (lane >> 1), c = lane & 1;
    const uint4 t = *reinterpret_cast<const uint4*>(sbuf + r * 32 + ((c ^ ((r >> 2) & 1)) << 4));
    *reinterpret_cast<uint4*>(dst0 + r * ld + c * 16) = t;
  }
  __syncwarp();
}

// Quantize 32 packed bf16 (16 words) of one block: returns the scale byte and
// the 32 codes.
__device__ __forceinline__ uint32_t quant32(const uint32_t* v, uint4 (&codes)[2]) {
  uint4 q[4];
  uint32_t am = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    q[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    am = max(am, absmax_bits8(q[i]));
  }
  const uint32_t byte = scale_byte_from_bits(am);
  uint2 c0 = encode8(q[0], byte), c1 = encode8(q[1], byte);
  uint2 c2 = encode8(q[2], byte), c3 = encode8(q[3], byte);
  codes[0] = make_uint4(c0.x, c0.y, c1.x, c1.y);
  codes[1] = make_uint4(c2.x, c2.y, c3.x, c3.y);
  return byte;
}

// ROW + COL quantization of a 32x32 bf16 block held one row per lane.
// ROW: codes of rows row0..row0+31, columns col0..col0+31 of a [*, ld_row]
// code matrix, scale (row, col0/32) in the MMA layout.  COL: codes of rows
// col0+lane, columns row0..row0+31 of the transposed [*, M] code matrix,
// scale (col0 + lane, row0/32).
__device__ __forceinline__ void dual_quant_block(const uint32_t* v, int lane, uint8_t* sbuf, int64_t row0,
                                                 int64_t col0, int64_t ld_row, int64_t M, uint8_t* row_codes,
                                                 uint8_t* row_scales, uint8_t* col_codes, uint8_t* col_scales) {
  uint4 q[2];
  const uint32_t rb = quant32(v, q);
  store_rows32(sbuf, q, row_codes + row0 * ld_row + col0, ld_row, lane);
  row_scales[mma_scale_offset(row0 + lane, col0 >> 5, ld_row)] = uint8_t(rb);
  uint32_t c[16];
  sbuf_acquire(lane);
  warp_transpose32(reinterpret_cast<uint32_t*>(sbuf), v, c, lane);
  const int64_t crow = col0 + lane;
  const uint32_t cb = quant32(c, q);
  uint4* dst = reinterpret_cast<uint4*>(col_codes + crow * M + row0);
  dst[0] = q[0];
  dst[1] = q[1];
  col_scales[mma_scale_offset(crow, row0 >> 5, M)] = uint8_t(cb);
}

__device__ __forceinline__ void load64(const uint16_t* src, uint32_t (&v)[16]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 t = s[i];
    v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
  }
}

// dSwiGLU outputs of one 32-column chunk, dgate (dg) and dup (du) of this
// lane's row (row0 + lane), dual-quantized to E4M3.  ROW: each lane
// quantizes its own two 32-element blocks (columns f.. and F + f.. of the
// [M, 2F] code matrix); the codes leave through 2 KB of staging as whole
// 32-byte row segments.  COL: the 32 x 64 bf16 tile dgate|dup is staged
// (16-byte piece j of row r at piece j ^ (r & 7)) and read back one column
// pair per lane, as the cast kernel's COL pass does (codes of columns f..
// and F + f.. of the [2F, M] code matrix, rows row0..row0+31), then leaves
// through the same 4 KB once it has been read.  tb: this warp's 6 KB of
// shared memory (tile, then ROW staging at +4096).
__device__ __forceinline__ void dswiglu_dual_quant(const uint32_t (&dg)[16], const uint32_t (&du)[16], int lane,
                                                   uint32_t tb, int64_t row0, int64_t f, int64_t F, int64_t M,
                                                   uint8_t* row_codes, uint8_t* row_scales, uint8_t* col_codes,
                                                   uint8_t* col_scales) {
  const uint32_t rs = tb + 4096;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    sts128(tb + lane * 128 + ((j ^ (lane & 7)) << 4), make_uint4(dg[4 * j], dg[4 * j + 1], dg[4 * j + 2], dg[4 * j + 3]));
    sts128(tb + lane * 128 + (((4 + j) ^ (lane & 7)) << 4),
           make_uint4(du[4 * j], du[4 * j + 1], du[4 * j + 2], du[4 * j + 3]));
  }
  // ROW: block g (0: dgate, 1: dup) of row r staged at 1024 g + 32 r, its two
  // 16-byte pieces swapped on (r >> 2) & 1
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    uint32_t cc[8];
    const uint32_t byte = quant_block32<0>(g ? du : dg, cc);
    row_scales[mma_scale_offset(row0 + lane, (g * F + f) >> 5, 2 * F)] = uint8_t(byte);
#pragma unroll
    for (int pc = 0; pc < 2; ++pc)
      sts128(rs + 1024 * g + lane * 32 + ((pc ^ ((lane >> 2) & 1)) << 4),
             make_uint4(cc[4 * pc], cc[4 * pc + 1], cc[4 * pc + 2], cc[4 * pc + 3]));
  }
  __syncwarp();
#pragma unroll
  for (int g = 0; g < 2; ++g)
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int r = 16 * i + (lane >> 1), pc = lane & 1;
      *reinterpret_cast<uint4*>(row_codes + (row0 + r) * 2 * F + g * F + f + 16 * pc) =
          lds128(rs + 1024 * g + r * 32 + ((pc ^ ((r >> 2) & 1)) << 4));
    }
  // COL
  uint32_t w[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) w[i] = lds32(tb + i * 128 + ((((lane >> 2) ^ (i & 7))) << 4) + ((lane & 3) << 2));
  __syncwarp();
  uint4 qq[2][2];
  const uint32_t cb = col_quant_pair32<0>(w, qq[0], qq[1]);
#pragma unroll
  for (int k = 0; k < 2; ++k) {
#pragma unroll
    for (int mm = 0; mm < 2; ++mm) sts128(tb + staging_off(4 * lane + 2 * k + mm), qq[k][mm]);
    const int L = 2 * lane + k;
    const int64_t gcol = (L < 32) ? f + L : F + f + (L - 32);
    col_scales[mma_scale_offset(gcol, row0 >> 5, M)] = uint8_t(cb >> (8 * k));
  }
  __syncwarp();
  // 16 columns x 32 bytes per store
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int L = 32 * k + lane, col = L >> 1, half = L & 1;
    const int64_t gcol = (col < 32) ? f + col : F + f + (col - 32);
    *reinterpret_cast<uint4*>(col_codes + gcol * M + row0 + 16 * half) = lds128(tb + staging_off(L));
  }
  __syncwarp();   // the staging is rewritten by the next chunk
}

// 32 TMEM columns of this lane's row -> 16 packed bf16 words (round to nearest even).
__device__ __forceinline__ void drain32_bf16(uint32_t taddr, uint32_t* w) {
  uint32_t r[32];
  tmem_ld_32x32b_x32(taddr, r);
  tmem_wait_ld();
#pragma unroll
  for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
}

// ---------------------------------------------------------------- the kernel
template <int kMode, int kEpi, int BN, bool kPair>
__global__ void __launch_bounds__(384, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                    const __grid_constant__ CUtensorMap tmap_sa, const __grid_constant__ CUtensorMap tmap_sb,
                    const __grid_constant__ CUtensorMap tmap_o, const Params p) {
  using C = Cfg<kMode, kEpi, BN, kPair>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTA pairs: the cluster is (2,1,1), so the rank in the pair is blockIdx.x & 1
  const int rank = kPair ? int(cluster_ctarank()) : 0;
  const int64_t unit = kPair ? (blockIdx.x >> 1) : blockIdx.x;       // tile-walker index of this CTA / pair
  const int64_t nunits = kPair ? (gridDim.x >> 1) : gridDim.x;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[C::kStages + s]); };
  auto tfull_bar = [&](int a) { return smem_u32(&bars[2 * C::kStages + a]); };
  auto tempty_bar = [&](int a) { return smem_u32(&bars[2 * C::kStages + C::kAcc + a]); };
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MISC);
  int32_t* offs = reinterpret_cast<int32_t*>(smem + C::OFF_OFFS);

  // ---- offsets into shared memory + validation (every CTA checks; both
  // CTAs of a pair see the same table, so they take the same decision)
  bool bad = p.E > C::MAX_E;
  if (!bad) {
    for (int i = threadIdx.x; i <= p.E; i += blockDim.x) offs[i] = p.offsets[i];
  }
  __syncthreads();
  if (!bad) {
    for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
      const int32_t o = offs[i];
      if (o < 0 || (o % p.pad) != 0 || int64_t(o) > p.M) bad = true;
      if (i == 0 && o != 0) bad = true;
      if (i < p.E && offs[i + 1] < o) bad = true;
    }
  }
  if constexpr (kMode == kRaggedK) {
    // real row counts: 0 <= rows[e] <= segment; the padded K blocks past the
    // last real row are skipped (their codes are zero, they add nothing).
    // Every thread reads the segments it owns first and tags them after a
    // barrier, so no read sees a tagged offset.
    constexpr int kPer = (C::MAX_E + 383) / 384;   // experts per thread (384 threads)
    int32_t skip[kPer];
    if (p.rows != nullptr) {
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = threadIdx.x + 384 * j;
        skip[j] = 0;
        if (!bad && i < p.E) {
          const int32_t seg = offs[i + 1] - offs[i], r = p.rows[i];
          if (r < 0 || r > seg) bad = true;
          else skip[j] = min((seg - ((r + 127) & ~127)) >> 7, 127);
        }
      }
    }
    if (__syncthreads_or(bad)) {
      if (threadIdx.x == 0 && blockIdx.x == 0) raise_device_error(kErrOffsets);
      return;
    }
    if (p.rows != nullptr) {
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = threadIdx.x + 384 * j;
        if (i < p.E) offs[i] |= skip[j];
      }
    }
  }
  if (__syncthreads_or(bad)) {
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_device_error(kErrOffsets);
    return;
  }

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    if constexpr (kPair) {
      prefetch_tmap(&tmap_sa);
      prefetch_tmap(&tmap_sb);
    }
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < C::kAcc; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), (kPair ? 2 : 1) * C::EPI_WARPS); // one arrival per epilogue warp
    }
    misc[1] = 0;  // abort flag
    fence_mbar_init();
  }
  if (warp == 2) {
    if constexpr (kPair) {
      tmem_alloc_pair(smem_u32(const_cast<uint32_t*>(misc)), C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(const_cast<uint32_t*>(misc)), C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (kPair) cluster_sync_all(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = misc[0];
  const int64_t ntiles = num_tiles<kMode, kEpi, BN, kPair>(p, offs);

  if (warp == 0) {
    // ================= producer (every CTA loads its own operand halves)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (TileIter<kMode, kEpi, BN, kPair> it(p, offs, unit, nunits); it.t < ntiles && ok; it.next(p, offs)) {
        const Tile T = get_tile(p, offs, it, rank);
        for (int kb = 0; kb < T.nk; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1)) { ok = false; break; }
          const int64_t k = T.k0 + int64_t(kb) * 128;
          const int64_t katoms = p.kext / 128, kat = k / 128;
          if constexpr (kPair) {
            // both CTAs' loads are credited to the even CTA's full barrier,
            // which expects the bytes of the whole pair
            const uint32_t fb = mapa_cluster(full_bar(stage), 0);
            if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 2 * C::STAGE_BYTES);
            tma_load_2d_pair(sbase + C::OFF_A + stage * C::A_BYTES, &tmap_a, fb, int(k), int(T.a_row));
            tma_load_2d_pair(sbase + C::OFF_B + stage * C::B_BYTES, &tmap_b, fb, int(k), int(T.b_mine));
            // scale atoms: a 512-byte atom is two 256-byte rows of the scale map
            tma_load_2d_pair(sbase + C::OFF_SFA + stage * C::SFA_BYTES, &tmap_sa, fb, 0,
                             int(((T.a_row / 128) * katoms + kat) * 2));
            tma_load_2d_pair(sbase + C::OFF_SFB + stage * C::SFB_BYTES, &tmap_sb, fb, 0,
                             int(((T.b_row0 / 128) * katoms + kat) * 2));
            if constexpr (BN == 256)
              tma_load_2d_pair(sbase + C::OFF_SFB + stage * C::SFB_BYTES + 512, &tmap_sb, fb, 0,
                               int(((T.b_row1 / 128) * katoms + kat) * 2));
          } else {
            const uint32_t fb = full_bar(stage);
            mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
            tma_load_2d(sbase + C::OFF_A + stage * C::A_BYTES, &tmap_a, fb, int(k), int(T.a_row));
            tma_load_2d(sbase + C::OFF_B + stage * C::B_BYTES, &tmap_b, fb, int(k), int(T.b_row0));
            if constexpr (BN == 256)
              tma_load_2d(sbase + C::OFF_B + stage * C::B_BYTES + 16384, &tmap_b, fb, int(k), int(T.b_row1));
            bulk_load(sbase + C::OFF_SFA + stage * C::SFA_BYTES,
                      p.a_scales + ((T.a_row / 128) * katoms + kat) * 512, 512, fb);
            bulk_load(sbase + C::OFF_SFB + stage * C::SFB_BYTES,
                      p.b_scales + ((T.b_row0 / 128) * katoms + kat) * 512, 512, fb);
            if constexpr (BN == 256)
              bulk_load(sbase + C::OFF_SFB + stage * C::SFB_BYTES + 512,
                        p.b_scales + ((T.b_row1 / 128) * katoms + kat) * 512, 512, fb);
          }
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) { misc[1] = 1; raise_device_error(kErrTimeout); }
    }
  } else if (warp == 1) {
    // ================= MMA issuer (the even CTA of a pair issues for both)
    if (lane == 0 && rank == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      uint32_t sfbuf = 0;
      bool ok = true;
      const uint32_t sf_col0 = C::ACC_COLS;
      constexpr uint32_t kMmaM = kPair ? 256 : 128;
      for (TileIter<kMode, kEpi, BN, kPair> it(p, offs, unit, nunits); it.t < ntiles && ok; it.next(p, offs)) {
        const Tile T = get_tile(p, offs, it, 0);
        if (T.nk == 0) continue;
        if (!(kPair ? mbar_wait_cluster(tempty_bar(acc), acc_phase ^ 1) : mbar_wait(tempty_bar(acc), acc_phase ^ 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < T.nk; ++kb) {
          if (!(kPair ? mbar_wait_cluster(full_bar(stage), phase) : mbar_wait(full_bar(stage), phase))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_t = tmem_base + sf_col0 + sfbuf * C::SF_COLS;
          const uint32_t sfb_t = sfa_t + 4;
          const uint32_t sfa_s = sbase + C::OFF_SFA + stage * C::SFA_BYTES;
          const uint32_t sfb_s = sbase + C::OFF_SFB + stage * C::SFB_BYTES;
          if constexpr (kPair) {
            utccp_32x128b_warpx4_pair(sfa_t, smem_desc(sfa_s, 0, 128, 0));
#pragma unroll
            for (int j = 0; j < BN / 128; ++j)
              utccp_32x128b_warpx4_pair(sfb_t + 4 * j, smem_desc(sfb_s + 512 * j, 0, 128, 0));
          } else {
            utccp_32x128b_warpx4(sfa_t, smem_desc(sfa_s, 0, 128, 0));
#pragma unroll
            for (int j = 0; j < BN / 128; ++j)
              utccp_32x128b_warpx4(sfb_t + 4 * j, smem_desc(sfb_s + 512 * j, 0, 128, 0));
          }
          const uint32_t a_s = sbase + C::OFF_A + stage * C::A_BYTES;
          const uint32_t b_s = sbase + C::OFF_B + stage * C::B_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = smem_desc(a_s + k * 32, 0, 1024, 2);
            const uint64_t bd = smem_desc(b_s + k * 32, 0, 1024, 2);
            if constexpr (kPair)
              mma_mxf8_pair(d_tmem, ad, bd, mxf8_idesc(kMmaM, BN, k), sfa_t, sfb_t, (kb | k) != 0);
            else
              mma_mxf8(d_tmem, ad, bd, mxf8_idesc(kMmaM, BN, k), sfa_t, sfb_t, (kb | k) != 0);
          }
          if constexpr (kPair) mma_commit_pair(empty_bar(stage)); else mma_commit(empty_bar(stage));
          sfbuf ^= 1;
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if constexpr (kPair) mma_commit_pair(tfull_bar(acc)); else mma_commit(tfull_bar(acc));
        if (++acc == C::kAcc) { acc = 0; acc_phase ^= 1; }
      }
      if (!ok) { misc[1] = 1; raise_device_error(kErrTimeout); }
    }
  } else if (warp >= 4) {
    // ================= epilogue =================
    // Warp 4+e (e = 0..7) reads TMEM lane quarter q = warp % 4 (rows 32q..)
    // and handles column half h = e / 4 of the tile.  The accumulator is
    // drained into packed bf16 registers and TMEM is released before any
    // math, so the next tile's MMAs overlap this tile's epilogue.
    const int q = warp & 3;
    const int h = (warp - 4) >> 2;
    uint8_t* sbuf = smem + C::OFF_EPI + (warp - 4) * C::EPI_WARP_BYTES;
    constexpr int kHalf = (kEpi == kEpiSwiGLU) ? 64 : BN / 2;   // accumulator columns per thread (per operand)
    constexpr int kChunks = kHalf / 32;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (TileIter<kMode, kEpi, BN, kPair> it(p, offs, unit, nunits); it.t < ntiles; it.next(p, offs)) {
      const Tile T = get_tile(p, offs, it, rank);
      const int64_t row0 = T.out_r0 + q * 32;              // first row of this warp's 32-row slab
      if constexpr (kMode == kRaggedK) {
        if (T.nk == 0) {
          // expert without rows: its weight gradient is exactly zero
          uint32_t z[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) z[j] = 0u;
#pragma unroll 1
          for (int c = 0; c < kChunks; ++c)
            store_block_tma(sbuf, z, &tmap_o, int(T.out_c0 + h * kHalf + 32 * c), int(int64_t(T.e) * p.rows_a + row0),
                            lane);
          continue;
        }
      }
      // warp-uniform outcome: the tcgen05.ld below are .sync.aligned
      if (!__all_sync(0xffffffffu, mbar_wait(tfull_bar(acc), acc_phase))) {
        raise_device_error(kErrTimeout);
        break;
      }
      tc_fence_after();
      const uint32_t t_row = tmem_base + (uint32_t(q * 32) << 16) + acc * BN;
      uint32_t va[kChunks * 16];
      uint32_t vb[(kEpi == kEpiSwiGLU) ? kChunks * 16 : 1];
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (kPair) mbar_arrive_remote(tempty_bar(acc), 0); else mbar_arrive(tempty_bar(acc));
        }
        if (++acc == C::kAcc) { acc = 0; acc_phase ^= 1; }
      };
      if constexpr (kEpi == kEpiBF16) {
        // all of this warp's columns in flight at once, one wait, and the
        // accumulator goes back to the MMA warp before any conversion: with a
        // single accumulator the next tile's MMAs start that much sooner
        uint32_t r[kChunks][32];
#pragma unroll
        for (int c = 0; c < kChunks; ++c) tmem_ld_32x32b_x32(t_row + h * kHalf + 32 * c, r[c]);
        tmem_wait_ld();
        release();
#pragma unroll
        for (int c = 0; c < kChunks; ++c)
#pragma unroll
          for (int j = 0; j < 16; ++j)
            va[16 * c + j] = pack_bf16x2(__uint_as_float(r[c][2 * j]), __uint_as_float(r[c][2 * j + 1]));
      } else {
        // the same for the SwiGLU / dSwiGLU epilogues: every TMEM load in
        // flight, one wait, TMEM handed back, then the bf16 rounding
        constexpr int kLoads = (kEpi == kEpiSwiGLU) ? 2 * kChunks : kChunks;
        uint32_t r[kLoads][32];
#pragma unroll
        for (int c = 0; c < kChunks; ++c) tmem_ld_32x32b_x32(t_row + h * kHalf + 32 * c, r[c]);
        if constexpr (kEpi == kEpiSwiGLU) {
#pragma unroll
          for (int c = 0; c < kChunks; ++c) tmem_ld_32x32b_x32(t_row + 128 + h * kHalf + 32 * c, r[kChunks + c]);
        }
        tmem_wait_ld();
        release();
#pragma unroll
        for (int c = 0; c < kChunks; ++c)
#pragma unroll
          for (int j = 0; j < 16; ++j)
            va[16 * c + j] = pack_bf16x2(__uint_as_float(r[c][2 * j]), __uint_as_float(r[c][2 * j + 1]));
        if constexpr (kEpi == kEpiSwiGLU) {
#pragma unroll
          for (int c = 0; c < kChunks; ++c)
#pragma unroll
            for (int j = 0; j < 16; ++j)
              vb[16 * c + j] = pack_bf16x2(__uint_as_float(r[kChunks + c][2 * j]),
                                           __uint_as_float(r[kChunks + c][2 * j + 1]));
        }
      }

      if constexpr (kEpi == kEpiBF16) {
        const int64_t orow = (kMode == kRaggedK) ? int64_t(T.e) * p.rows_a + row0 : row0;
#pragma unroll
        for (int c = 0; c < kChunks; ++c)
          store_block_tma(sbuf, va + 16 * c, &tmap_o, int(T.out_c0 + h * kHalf + 32 * c), int(orow), lane);
      } else if constexpr (kEpi == kEpiSwiGLU) {
        const int64_t F = p.F;
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          const int64_t f = T.out_c0 + h * kHalf + 32 * c;
          const uint32_t* a2 = va + 16 * c;
          const uint32_t* b2 = vb + 16 * c;
          if (p.out != nullptr) {
            store_block_tma(sbuf, a2, &tmap_o, int(f), int(row0), lane);
            store_block_tma(sbuf, b2, &tmap_o, int(F + f), int(row0), lane);
          }
          uint32_t h2[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            h2[j] = pack_bf16x2(silu_mul(bf16lo_to_f32(a2[j]), bf16lo_to_f32(b2[j])),
                                silu_mul(bf16hi_to_f32(a2[j]), bf16hi_to_f32(b2[j])));
          dual_quant_block(h2, lane, sbuf, row0, f, F, p.M, p.row_codes, p.row_scales, p.col_codes, p.col_scales);
        }
      } else {  // kEpiDSwiGLU
        const int64_t F = p.F;
        const int64_t m = row0 + lane;
        const uint32_t tb = smem_u32(sbuf);
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          const int64_t f = T.out_c0 + h * kHalf + 32 * c;
          // h13 gate (hw[0..15]) and up (hw[16..31]) words of this row; dgate
          // and dup are written over them
          uint32_t hw[32];
          load64(p.h13 + m * 2 * F + f, *reinterpret_cast<uint32_t(*)[16]>(&hw[0]));
          load64(p.h13 + m * 2 * F + F + f, *reinterpret_cast<uint32_t(*)[16]>(&hw[16]));
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const uint32_t dw = va[16 * c + j];
            float d[2], a[2], b[2], og[2], ou[2];
            d[0] = bf16lo_to_f32(dw); d[1] = bf16hi_to_f32(dw);
            a[0] = bf16lo_to_f32(hw[j]); a[1] = bf16hi_to_f32(hw[j]);
            b[0] = bf16lo_to_f32(hw[16 + j]); b[1] = bf16hi_to_f32(hw[16 + j]);
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const float s = sigmoid_fast(a[i]);
              og[i] = d[i] * b[i] * s * (1.0f + a[i] * (1.0f - s));
              ou[i] = d[i] * a[i] * s;
            }
            hw[j] = pack_bf16x2(og[0], og[1]);        // dgate
            hw[16 + j] = pack_bf16x2(ou[0], ou[1]);   // dup
          }
          dswiglu_dual_quant(*reinterpret_cast<const uint32_t(*)[16]>(&hw[0]),
                             *reinterpret_cast<const uint32_t(*)[16]>(&hw[16]), lane, tb, row0, f, F, p.M, p.row_codes, p.row_scales, p.col_codes,
                             p.col_scales);
        }
      }
    }
  }

  // outstanding TMA stores of the epilogue warps complete before the CTA exits
  if (warp >= 4 && lane == 0) bulk_wait_all();

  // ---- teardown: every role has left its loop (all waits are bounded); in a
  // pair, neither CTA frees its TMEM or exits while the other may still
  // arrive on its barriers or run MMAs into its TMEM
  tc_fence_before();
  if constexpr (kPair) cluster_sync_all(); else __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    if constexpr (kPair) tmem_dealloc_pair(tmem_base, C::TMEM_COLS); else tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace mxmoe::gemm
