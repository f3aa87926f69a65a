// Packed-layout helpers: unpadding a masked batch into the packed stream the
// attention kernel reads, the row gather / scatter between the padded and
// packed layouts, and the fold of one per-pair bias row into a per-key bias.
//
// All of them are memory-bound copies or scans: coalesced 16-byte accesses,
// grid-stride loops over a grid sized from the SM count, no shared-memory
// staging beyond the block scans. Indices and boundaries read from device
// memory are bounds-checked; a bad one raises kErrBadSeqlens in the device
// error word and the offending row is skipped, never accessed.
#pragma once
#include <cstdint>
#include "common.cuh"

namespace va {

constexpr int kLayoutThreads = 256;

// Inclusive warp scan then block-wide exclusive offset (blockDim = 256).
__device__ __forceinline__ int block_scan_256(int x, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = lane < kLayoutThreads / 32 ? warp_sums[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < kLayoutThreads / 32) warp_sums[lane] = wi - w;
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  const int r = warp_sums[warp] + incl - x;
  __syncthreads();
  return r;
}

// counts[b] = number of nonzero mask bytes in row b (one block per row).
__global__ void __launch_bounds__(kLayoutThreads) mask_count_kernel(const uint8_t* mask, int S,
                                                                    int32_t* counts) {
  __shared__ int s_sum;
  if (threadIdx.x == 0) s_sum = 0;
  __syncthreads();
  const uint8_t* row = mask + (long long)blockIdx.x * S;
  int n = 0;
  for (int s = threadIdx.x; s < S; s += kLayoutThreads) n += row[s] != 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
  if ((threadIdx.x & 31) == 0) atomicAdd(&s_sum, n);
  __syncthreads();
  if (threadIdx.x == 0) counts[blockIdx.x] = s_sum;
}

// cu[0] = 0, cu[b + 1] = cu[b] + counts[b] (counts stored in cu[1..B]),
// *max_len = max counts. One block.
__global__ void __launch_bounds__(kLayoutThreads) seqlens_scan_kernel(int32_t* cu, int B,
                                                                      int32_t* max_len) {
  __shared__ int s_warp[kLayoutThreads / 32];
  __shared__ int s_total, s_max;
  if (threadIdx.x == 0) s_max = 0;
  int carry = 0, mx = 0;
  for (int base = 0; base < B; base += kLayoutThreads) {
    const int b = base + threadIdx.x;
    const int c = b < B ? cu[b + 1] : 0;
    mx = max(mx, c);
    const int off = carry + block_scan_256(c, s_warp, &s_total);
    if (b < B) cu[b + 1] = off + c;
    carry += s_total;
  }
  atomicMax(&s_max, mx);
  __syncthreads();
  if (threadIdx.x == 0) {
    cu[0] = 0;
    *max_len = s_max;
  }
}

// indices[cu[b] + j] = b * S + s for the j-th nonzero s of row b, in order
// (one block per row).
__global__ void __launch_bounds__(kLayoutThreads) mask_indices_kernel(const uint8_t* mask, int S,
                                                                      const int32_t* cu,
                                                                      int32_t* indices) {
  __shared__ int s_warp[kLayoutThreads / 32];
  __shared__ int s_total;
  const int b = blockIdx.x;
  const uint8_t* row = mask + (long long)b * S;
  int carry = cu[b];
  for (int base = 0; base < S; base += kLayoutThreads) {
    const int s = base + threadIdx.x;
    const int v = (s < S && row[s] != 0) ? 1 : 0;
    const int off = carry + block_scan_256(v, s_warp, &s_total);
    if (v) indices[off] = (int32_t)((long long)b * S + s);
    carry += s_total;
  }
}

// dst[t] = src[indices[t]] for t < cu[B]: 16-byte units, grid-stride.
__global__ void __launch_bounds__(kLayoutThreads) gather_rows_kernel(
    const uint4* src, long long src_rows, long long row_units, const int32_t* indices,
    const int32_t* cu, int B, uint4* dst, long long dst_rows, int* error) {
  const long long T = cu[B];
  if (T < 0 || T > dst_rows) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicCAS(error, 0, kErrBadSeqlens);
    return;
  }
  const long long n = T * row_units;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const long long t = e / row_units, u = e - t * row_units;
    const long long sr = indices[t];
    if (sr < 0 || sr >= src_rows) {
      if (u == 0) atomicCAS(error, 0, kErrBadSeqlens);
      continue;
    }
    dst[t * row_units + u] = src[sr * row_units + u];
  }
}

// dst[indices[t]] = src[t] for t < cu[B] (dst zeroed beforehand).
__global__ void __launch_bounds__(kLayoutThreads) scatter_rows_kernel(
    const uint4* src, long long src_rows, long long row_units, const int32_t* indices,
    const int32_t* cu, int B, uint4* dst, long long dst_rows, int* error) {
  const long long T = cu[B];
  if (T < 0 || T > src_rows) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicCAS(error, 0, kErrBadSeqlens);
    return;
  }
  const long long n = T * row_units;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const long long t = e / row_units, u = e - t * row_units;
    const long long dr = indices[t];
    if (dr < 0 || dr >= dst_rows) {
      if (u == 0) atomicCAS(error, 0, kErrBadSeqlens);
      continue;
    }
    dst[dr * row_units + u] = src[t * row_units + u];
  }
}

// out[cu_k[i] + c, h] = in[cu_k[i] + c, h] (or 0) +
//   grid[i*sb + (h / head_div)*sh + row*sr + c*sc] for c < Lk_i.
__global__ void __launch_bounds__(kLayoutThreads) fold_pair_row_kernel(
    const float* grid, long long sb, long long sh, long long sr, long long sc, int row, int head_div,
    const int32_t* cu_k, int B, int total_k, int H, const float* in, float* out, int* error) {
  const int T = cu_k[B];
  if (T < 0 || T > total_k || cu_k[0] != 0) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicCAS(error, 0, kErrBadSeqlens);
    return;
  }
  const long long n = (long long)T * H;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(e / H), h = (int)(e - (long long)t * H);
    // sequence of key row t: the last i with cu_k[i] <= t (binary search)
    int lo = 0, hi = B;  // invariant: cu_k[lo] <= t < cu_k[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (cu_k[mid] <= t) lo = mid;
      else hi = mid;
    }
    const int c = t - cu_k[lo];
    if (c < 0 || t >= cu_k[lo + 1]) {  // boundaries not non-decreasing
      atomicCAS(error, 0, kErrBadSeqlens);
      continue;
    }
    const float g = grid[(long long)lo * sb + (long long)(h / head_div) * sh + (long long)row * sr +
                         (long long)c * sc];
    out[e] = (in ? in[e] : 0.f) + g;
  }
}

}  // namespace va
