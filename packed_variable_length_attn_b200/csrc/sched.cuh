// Schedule kernel: validates cu_seqlens and builds the work list of the
// persistent attention kernel, longest job first (LPT).
//
// One CTA of 1024 threads:
//   1. validate the boundaries (cu[0] = 0, non-decreasing, lengths within
//      the caller's max_seqlen, cu[B] within the totals). On failure the
//      error word gets kErrBadSeqlens and the work count is 0, so the
//      attention kernel does nothing and reads nothing out of range;
//   2. enumerate the (sequence, group) pairs with a block-wide prefix sum;
//   3. order them with an in-shared-memory bitonic sort of 64-bit keys:
//      sequences by size, largest first, and within a sequence the pairs by
//      K/V tiles to visit, descending (ties by position in the stream);
//   4. publish the list, the item count and a zeroed fetch counter.
// Each pair expands to n_hg consecutive work items (head groups), so the
// heads of one q-block run side by side and share K/V and bias tiles in L2.
// Grouping by sequence keeps the CTAs that run at the same time on the K/V
// of one sequence (a few tens of MB at most), which then stays in L2
// instead of being fetched from HBM again for every q-block; largest first
// within and across sequences keeps the longest items away from the end.
#pragma once
#include "common.cuh"

namespace va {

constexpr int kSchedThreads = 1024;
constexpr int kSortCap = 8192;  // pairs sorted in shared memory; beyond: stream order
static_assert(kSortCap <= (1 << 20), "stream position must fit the low 20 bits of a sort key");

__device__ __forceinline__ int block_exclusive_scan(int x, int* warp_sums, int* total) {
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
    int w = warp_sums[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    warp_sums[lane] = wi - w;  // exclusive prefix of warp totals
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  const int r = warp_sums[warp] + incl - x;
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kSchedThreads, 1) schedule_kernel(SchedParams p) {
  extern __shared__ unsigned long long sort_keys[];
  __shared__ int s_bad;
  __shared__ int s_warp[32];
  __shared__ int s_total;
  const int tid = threadIdx.x;
  if (tid == 0) s_bad = 0;
  __syncthreads();

  // 1. validation
  int bad = 0;
  for (int i = tid; i <= p.batch; i += kSchedThreads) {
    const int cq = p.cu_q[i], ck = p.cu_k[i];
    if (i == 0 && (cq != 0 || ck != 0)) bad = 1;
    if (i < p.batch) {
      const int lq = p.cu_q[i + 1] - cq, lk = p.cu_k[i + 1] - ck;
      if (lq < 0 || lk < 0 || lq > p.max_q || lk > p.max_k) bad = 1;
    } else if (cq > p.total_q || ck > p.total_k) {
      bad = 1;
    }
  }
  if (bad) atomicOr(&s_bad, 1);
  __syncthreads();
  if (s_bad) {
    if (tid == 0) {
      atomicCAS(p.error, 0, kErrBadSeqlens);
      *p.ws.count = 0;
      *p.ws.counter = 0;
    }
    return;
  }
  if (p.pairing < 0) {  // validate only
    if (tid == 0) {
      *p.ws.count = 1;
      *p.ws.counter = 0;
    }
    return;
  }

  // 2. enumerate pairs
  int carry = 0;
  for (int base = 0; base < p.batch; base += kSchedThreads) {
    const int i = base + tid;
    int ng = 0;
    if (i < p.batch) ng = seq_groups(p.cu_q[i + 1] - p.cu_q[i], p.pairing);
    const int off = carry + block_exclusive_scan(ng, s_warp, &s_total);
    if (i < p.batch) {
      for (int g = 0; g < ng && off + g < p.ws.capacity; ++g) p.ws.tmp[off + g] = make_int2(i, g);
    }
    carry += s_total;
    __syncthreads();
  }
  const int P = carry;
  if (P > p.ws.capacity) {  // cannot happen once lengths <= max_q (checked above)
    if (tid == 0) {
      atomicCAS(p.error, 0, kErrBadSeqlens);
      *p.ws.count = 0;
      *p.ws.counter = 0;
    }
    return;
  }
  __syncthreads();

  // 3. LPT order
  if (P <= kSortCap) {
    int N = 1;
    while (N < P) N <<= 1;
    for (int k = tid; k < N; k += kSchedThreads) {
      unsigned long long key = ~0ull;
      if (k < P) {
        const int2 pr = p.ws.tmp[k];
        const int i = pr.x, g = pr.y;
        Item it;
        it.Lq = p.cu_q[i + 1] - p.cu_q[i];
        it.Lk = p.cu_k[i + 1] - p.cu_k[i];
        int work = 0;
        for (int s = 0; s < 2; ++s) {
          const int q_loc0 = p.pairing == kPairHeads ? g * BM : (2 * g + s) * BM;
          int rows = it.Lq - q_loc0;
          rows = rows < 0 ? 0 : (rows > BM ? BM : rows);
          work += slot_tiles(q_loc0, rows, it.Lq, it.Lk, p.causal);
        }
        // key: [63:40] sequence size (descending), [39:20] item work
        // (descending), [19:0] stream position (k < kSortCap <= 2^20).
        long long sk = (long long)ceil_div(it.Lq, BM) * ceil_div(it.Lk, BN);
        sk = sk > 0xFFFFFF ? 0xFFFFFF : sk;
        const int wk = work > 0xFFFFF ? 0xFFFFF : work;
        key = ((unsigned long long)(0xFFFFFF - sk) << 40) |
              ((unsigned long long)(0xFFFFF - wk) << 20) | (unsigned)k;
      }
      sort_keys[k] = key;
    }
    __syncthreads();
    for (int k = 2; k <= N; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int idx = tid; idx < N; idx += kSchedThreads) {
          const int ixj = idx ^ j;
          if (ixj > idx) {
            const unsigned long long a = sort_keys[idx], b = sort_keys[ixj];
            const bool up = (idx & k) == 0;
            if ((a > b) == up) {
              sort_keys[idx] = b;
              sort_keys[ixj] = a;
            }
          }
        }
        __syncthreads();
      }
    }
    for (int k = tid; k < P; k += kSchedThreads)
      p.ws.list[k] = p.ws.tmp[(int)(sort_keys[k] & 0xFFFFFu)];
  } else {
    for (int k = tid; k < P; k += kSchedThreads) p.ws.list[k] = p.ws.tmp[k];
  }
  __syncthreads();
  if (tid == 0) {
    *p.ws.count = P * p.n_hg;
    *p.ws.counter = 0;
  }
}

}  // namespace va
