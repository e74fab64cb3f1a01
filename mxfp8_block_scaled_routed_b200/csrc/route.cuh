// Token dispatcher around the routed-experts MLP: the padded expert-major
// layout (routing -> offsets and the row <-> slot tables), and the weighted
// combine back to token order with its weight gradient.
//
// The fully-fused plan page ("What it adds") installs a dispatcher whose
// per-expert segments are padded to pad_multiple rows, and the
// SwiGLU-boundary page ("Usage") has that dispatcher produce the padded
// expert-major layout the kernels consume.  Slot s = t*k + j is token t's
// j-th routed copy; an expert's segment lists its slots in ascending order,
// then zero pad rows.  The gather into that layout is fused with the MXFP8
// cast (mx_cast_kernel<kCastGather> in quant.cuh).
//
// Layout construction is a deterministic counting sort in three launches:
// per-chunk histograms, one block that scans them into padded offsets and
// per-(chunk, expert) base rows, and a pass that ranks every slot inside its
// chunk (warp match + per-warp prefix counts) so the order is stable.
#pragma once
#include "mx_common.cuh"

namespace mxmoe {

constexpr int kRouteChunk = 4096;      // slots per chunk: 32 warps x 128
constexpr int kRouteThreads = 1024;
constexpr int kRouteMaxE = 1024;

// chunk_counts[c][e] = slots of chunk c routed to expert e.
__global__ void __launch_bounds__(kRouteThreads)
route_count_kernel(const int32_t* __restrict__ topk, int64_t n, int E, int32_t* __restrict__ chunk_counts) {
  __shared__ int hist[kRouteMaxE];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int64_t s0 = int64_t(blockIdx.x) * kRouteChunk;
  for (int i = threadIdx.x; i < kRouteChunk; i += blockDim.x) {
    const int64_t s = s0 + i;
    if (s >= n) break;
    const int e = topk[s];
    if (e >= 0 && e < E)
      atomicAdd(&hist[e], 1);
    else
      raise_device_error(9);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_counts[int64_t(blockIdx.x) * E + e] = hist[e];
}

// One block: totals per expert, padded exclusive scan -> offsets, chunk
// counts -> absolute base row of (chunk, expert), -1 into every pad row and
// every row of [offsets[E], m_cap).
__global__ void __launch_bounds__(kRouteThreads)
route_scan_kernel(int32_t* __restrict__ chunk_counts, int nchunks, int E, int pad, int64_t m_cap,
                  int32_t* __restrict__ offsets, int32_t* __restrict__ row_slot) {
  __shared__ int64_t scan[kRouteThreads];
  __shared__ int32_t tot_sh[kRouteMaxE];
  __shared__ int32_t off_sh[kRouteMaxE + 1];
  const int e = threadIdx.x;
  int64_t tot = 0;
  if (e < E)
    for (int c = 0; c < nchunks; ++c) tot += chunk_counts[int64_t(c) * E + e];
  const int64_t padded = (tot + pad - 1) / pad * pad;
  scan[e] = e < E ? padded : 0;
  __syncthreads();
  for (int off = 1; off < kRouteThreads; off <<= 1) {
    const int64_t v = e >= off ? scan[e - off] : 0;
    __syncthreads();
    scan[e] += v;
    __syncthreads();
  }
  const int64_t excl = scan[e] - padded;
  const int64_t total = scan[kRouteThreads - 1];
  if (total > m_cap) {
    if (e == 0) raise_device_error(2);
  }
  if (e < E) {
    offsets[e] = int32_t(excl);
    off_sh[e] = int32_t(excl);
    tot_sh[e] = int32_t(tot);
    int64_t run = excl;
    for (int c = 0; c < nchunks; ++c) {
      const int64_t i = int64_t(c) * E + e;
      const int32_t cnt = chunk_counts[i];
      chunk_counts[i] = int32_t(run);
      run += cnt;
    }
  }
  if (e == 0) {
    offsets[E] = int32_t(total);
    off_sh[E] = int32_t(total);
  }
  __syncthreads();
  for (int x = 0; x < E; ++x) {
    const int64_t end = min(int64_t(off_sh[x + 1]), m_cap);
    for (int64_t r = int64_t(off_sh[x]) + tot_sh[x] + e; r < end; r += kRouteThreads) row_slot[r] = -1;
  }
  for (int64_t r = total + e; r < m_cap; r += kRouteThreads) row_slot[r] = -1;
}

// Stable rank of every slot: warp w of block c owns slots
// [c*4096 + w*128, +128) in four batches of 32.  Rows past m_cap are not
// written (the scan kernel has flagged the overflow).
__global__ void __launch_bounds__(kRouteThreads)
route_assign_kernel(const int32_t* __restrict__ topk, int64_t n, int E, const int32_t* __restrict__ chunk_base,
                    int64_t m_cap, int32_t* __restrict__ row_slot, int32_t* __restrict__ slot_row) {
  extern __shared__ __align__(16) uint8_t route_smem[];
  int32_t* base = reinterpret_cast<int32_t*>(route_smem);              // [E]
  uint16_t* pre = reinterpret_cast<uint16_t*>(route_smem + E * 4);     // [32 warps][E]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < E; e += kRouteThreads) base[e] = chunk_base[int64_t(blockIdx.x) * E + e];
  for (int i = tid; i < 32 * E; i += kRouteThreads) pre[i] = 0;
  __syncthreads();
  const int64_t s0 = int64_t(blockIdx.x) * kRouteChunk + warp * 128;
  auto expert_of = [&](int64_t s) {
    if (s >= n) return -1;
    const int e = topk[s];
    return (e >= 0 && e < E) ? e : -1;
  };
  // per-warp counts
  for (int b = 0; b < 4; ++b) {
    const int e = expert_of(s0 + b * 32 + lane);
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) pre[warp * E + e] += uint16_t(__popc(peers));
    __syncwarp();
  }
  __syncthreads();
  // exclusive prefix over warps, per expert
  for (int e = tid; e < E; e += kRouteThreads) {
    uint32_t run = 0;
    for (int w = 0; w < 32; ++w) {
      const uint32_t v = pre[w * E + e];
      pre[w * E + e] = uint16_t(run);
      run += v;
    }
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  for (int b = 0; b < 4; ++b) {
    const int64_t s = s0 + b * 32 + lane;
    const int e = expert_of(s);
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (s < n) {
      if (e >= 0) {
        const int64_t row = int64_t(base[e]) + pre[warp * E + e] + __popc(peers & lt);
        slot_row[s] = int32_t(row);
        if (row < m_cap) row_slot[row] = int32_t(s);
      } else {
        slot_row[s] = -1;
      }
    }
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) pre[warp * E + e] += uint16_t(__popc(peers));
    __syncwarp();
  }
}

// out[t] = bf16( sum_j w[t*k+j] * y[slot_row[t*k+j]] ), fp32 accumulation in
// j order (w = 1 without weights).  One block per token, 8 bf16 per thread
// and step.
__global__ void __launch_bounds__(256)
combine_kernel(const uint16_t* __restrict__ y, int64_t m_rows, const int32_t* __restrict__ slot_row,
               const float* __restrict__ w, int k, int64_t D, uint16_t* __restrict__ out) {
  __shared__ int64_t rows[64];
  __shared__ float ws[64];
  const int64_t t = blockIdx.x;
  if (threadIdx.x < k) {
    int64_t r = slot_row[t * k + threadIdx.x];
    if (r >= m_rows) {
      raise_device_error(4);
      r = -1;
    }
    rows[threadIdx.x] = r;
    ws[threadIdx.x] = w ? w[t * k + threadIdx.x] : 1.0f;
  }
  __syncthreads();
  const int64_t nv = D >> 3;
  for (int64_t c = threadIdx.x; c < nv; c += blockDim.x) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    for (int j = 0; j < k; ++j) {
      const int64_t r = rows[j];
      if (r < 0) continue;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(y + r * D) + c);
      const float wj = ws[j];
      acc[0] = fmaf(wj, bf16lo_to_f32(v.x), acc[0]);
      acc[1] = fmaf(wj, bf16hi_to_f32(v.x), acc[1]);
      acc[2] = fmaf(wj, bf16lo_to_f32(v.y), acc[2]);
      acc[3] = fmaf(wj, bf16hi_to_f32(v.y), acc[3]);
      acc[4] = fmaf(wj, bf16lo_to_f32(v.z), acc[4]);
      acc[5] = fmaf(wj, bf16hi_to_f32(v.z), acc[5]);
      acc[6] = fmaf(wj, bf16lo_to_f32(v.w), acc[6]);
      acc[7] = fmaf(wj, bf16hi_to_f32(v.w), acc[7]);
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    __stcs(reinterpret_cast<uint4*>(out + t * D) + c, o);
  }
}

// Real (token) rows of each expert's padded segment.  The route lays out a
// segment's token rows first and its pad rows (row_slot < 0) after them, so
// the count is the position of the first pad row: a binary search per expert.
// A segment outside [0, m_rows] counts 0 rows (the GEMMs reject its offsets).
__global__ void __launch_bounds__(256)
expert_rows_kernel(const int32_t* __restrict__ offsets, const int32_t* __restrict__ row_slot, int E, int64_t m_rows,
                   int32_t* __restrict__ rows) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  const int64_t base = offsets[e], end = offsets[e + 1];
  if (base < 0 || end > m_rows || end < base) {
    rows[e] = 0;
    return;
  }
  int64_t lo = base, hi = end;     // first pad row in [base, end]
  while (lo < hi) {
    const int64_t mid = (lo + hi) >> 1;
    if (row_slot[mid] >= 0) lo = mid + 1; else hi = mid;
  }
  rows[e] = int32_t(lo - base);
}

// dw[t*k+j] = <dout[t], y[slot_row[t*k+j]]> in fp32 (0 for an invalid slot).
__global__ void __launch_bounds__(256)
combine_weight_grad_kernel(const uint16_t* __restrict__ dout, const uint16_t* __restrict__ y, int64_t m_rows,
                           const int32_t* __restrict__ slot_row, int k, int64_t D, float* __restrict__ dw) {
  __shared__ float red[8];
  const int64_t t = blockIdx.x;
  const int64_t nv = D >> 3;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint4* d4 = reinterpret_cast<const uint4*>(dout + t * D);
  for (int j = 0; j < k; ++j) {
    int64_t r = slot_row[t * k + j];
    if (r >= m_rows) {
      if (threadIdx.x == 0) raise_device_error(4);
      r = -1;
    }
    float part = 0.0f;
    if (r >= 0) {
      const uint4* y4 = reinterpret_cast<const uint4*>(y + r * D);
      for (int64_t c = threadIdx.x; c < nv; c += blockDim.x) {
        const uint4 a = __ldg(d4 + c), b = __ldg(y4 + c);
        part = fmaf(bf16lo_to_f32(a.x), bf16lo_to_f32(b.x), part);
        part = fmaf(bf16hi_to_f32(a.x), bf16hi_to_f32(b.x), part);
        part = fmaf(bf16lo_to_f32(a.y), bf16lo_to_f32(b.y), part);
        part = fmaf(bf16hi_to_f32(a.y), bf16hi_to_f32(b.y), part);
        part = fmaf(bf16lo_to_f32(a.z), bf16lo_to_f32(b.z), part);
        part = fmaf(bf16hi_to_f32(a.z), bf16hi_to_f32(b.z), part);
        part = fmaf(bf16lo_to_f32(a.w), bf16lo_to_f32(b.w), part);
        part = fmaf(bf16hi_to_f32(a.w), bf16hi_to_f32(b.w), part);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) red[warp] = part;
    __syncthreads();
    if (threadIdx.x == 0) {
      float s = 0.0f;
      for (int i = 0; i < (int)(blockDim.x >> 5); ++i) s += red[i];
      dw[t * k + j] = s;
    }
    __syncthreads();
  }
}

}  // namespace mxmoe
