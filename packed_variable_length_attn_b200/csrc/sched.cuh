// Schedule kernel: validates cu_seqlens and builds the work list of the
// persistent attention kernel, longest job first (LPT).
//
// One CTA of 1024 threads:
//   1. validate the boundaries (cu[0] = 0, non-decreasing, lengths within
//      the caller's max_seqlen, cu[B] within the totals). On failure the
//      error word gets kErrBadSeqlens and the work count is 0, so the
//      attention kernel does nothing and reads nothing out of range;
//   2. order the sequences by size, largest first (ties: stream order), with
//      a bitonic sort of 64-bit keys in shared memory; beyond kSeqSortCap
//      sequences, runs of kSeqSortCap are sorted there and merged in global
//      memory (each key finds its place in the partner run by binary search),
//      so every batch size gets the same order;
//   3. give each sequence its range of the list (prefix sum of its pair
//      counts in that order) and place its (sequence, group) pairs there by
//      K/V tiles to visit, descending: for a causal mask the work of a
//      q-block never decreases along the sequence, so the pairs go last
//      first (a lone last unit of an odd number of units is put where its
//      work falls); without a mask every full pair has the same work and
//      they keep stream order;
//   4. publish the item count and a zeroed fetch counter.
// Each pair expands to n_hg consecutive work items (head groups), so the
// heads of one q-block run side by side and share K/V and bias tiles in L2.
// Grouping by sequence keeps the CTAs that run at the same time on the K/V
// of one sequence (a few tens of MB at most), which then stays in L2
// instead of being fetched from HBM again for every q-block; largest first
// within and across sequences keeps the longest items away from the end.
// The order only decides when an item runs, never what it computes.
// With key ranges (a decode step whose sequences are cut into ranges of the
// cache, see SchedParams) steps 2-4 run over the virtual sequences, one per
// (sequence, range), each sized by its own keys.
#pragma once
#include "common.cuh"

namespace va {

constexpr int kSchedThreads = 1024;
constexpr int kSeqSortCap = 16384;  // sequence keys sorted in one shared-memory pass
constexpr int kSchedSmemBytes = kSeqSortCap * 8;

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

// Sort key of sequence i: size (q-blocks x K/V blocks) descending in the
// high bits, the index (ascending) in the low 32 bits; keys are unique.
__device__ __forceinline__ unsigned long long seq_key(const SchedParams& p, int i) {
  const int lq = range_lq(p, i), lk = range_lk(p, i);
  long long sk = (long long)ceil_div(lq, BM) * ceil_div(lk, BN);
  sk = sk > 0xFFFFFF ? 0xFFFFFF : sk;
  return ((unsigned long long)(0xFFFFFF - sk) << 32) | (unsigned)i;
}

// Ascending bitonic sort of n keys (n a power of two) in shared memory.
__device__ void bitonic_sort_smem(unsigned long long* keys, int n) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int idx = threadIdx.x; idx < n; idx += kSchedThreads) {
        const int ixj = idx ^ j;
        if (ixj > idx) {
          const unsigned long long a = keys[idx], b = keys[ixj];
          const bool up = (idx & k) == 0;
          if ((a > b) == up) {
            keys[idx] = b;
            keys[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
}

// Number of keys of the sorted run [a, a + n) that are below `key`.
__device__ __forceinline__ int count_below(const unsigned long long* run, int n,
                                           unsigned long long key) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (run[mid] < key) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// Work (K/V tiles over both slots) of pair g of a sequence.
__device__ __forceinline__ int pair_work(int g, int Lq, int Lk, int pairing, int group,
                                         int causal) {
  int work = 0;
  for (int s = 0; s < 2; ++s) {
    int q_loc0, hl;
    slot_unit(g, s, pairing, group, q_loc0, hl);
    int rows = Lq - q_loc0;
    rows = rows < 0 ? 0 : (rows > BM ? BM : rows);
    work += slot_tiles(q_loc0, rows, Lq, Lk, causal);
  }
  return work;
}

__global__ void __launch_bounds__(kSchedThreads, 1) schedule_kernel(SchedParams p) {
  extern __shared__ unsigned long long sort_keys[];
  __shared__ int s_bad;
  __shared__ int s_warp[32];
  __shared__ int s_total;
  const int tid = threadIdx.x;
  // The attention kernel launched after this one may begin its set-up now;
  // it reads the work list only after this grid has completed.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid == 0) s_bad = 0;
  __syncthreads();

  // 1. validation
  int bad = 0;
  for (int i = tid; i <= p.batch; i += kSchedThreads) {
    const int cq = p.cu_q[i];
    const bool cache = p.cache_seqlens != nullptr;
    const int ck = cache ? 0 : p.cu_k[i];
    if (i == 0 && (cq != 0 || ck != 0)) bad = 1;
    if (i < p.batch) {
      const int lq = p.cu_q[i + 1] - cq;
      const int lk = cache ? seq_lk(p, i) : p.cu_k[i + 1] - ck;
      if (lq < 0 || lk < 0 || lq > p.max_q || lk > (cache ? p.cache_len : p.max_k)) bad = 1;
      if (cache && p.cache_seqlens[i] < 0) bad = 1;
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

  // 2. sequences by size. `ord` ends up holding, per rank, the sequence index
  // (x) and, after step 3, the first list position of its pairs (y).
  const int B = p.batch * (p.cache_ranges > 1 ? p.cache_ranges : 1);
  int2* ord;
  if (B <= kSeqSortCap) {
    int n = 1;
    while (n < B) n <<= 1;
    for (int k = tid; k < n; k += kSchedThreads) sort_keys[k] = k < B ? seq_key(p, k) : ~0ull;
    __syncthreads();
    bitonic_sort_smem(sort_keys, n);
    ord = reinterpret_cast<int2*>(sort_keys);  // in place: entry r read and written by one thread
    for (int r = tid; r < B; r += kSchedThreads) {
      const unsigned long long key = sort_keys[r];
      ord[r] = make_int2((int)(unsigned)(key & 0xFFFFFFFFu), 0);
    }
  } else {
    // runs of kSeqSortCap sorted in shared memory, then merged pairwise; the
    // buffers (list and tmp hold >= B entries of 8 bytes) alternate so that
    // the sorted keys end in tmp, which step 3 turns into `ord`.
    unsigned long long* buf[2] = {reinterpret_cast<unsigned long long*>(p.ws.tmp),
                                  reinterpret_cast<unsigned long long*>(p.ws.list)};
    const int runs = ceil_div(B, kSeqSortCap);
    int passes = 0;
    while ((1 << passes) < runs) ++passes;
    int cur = passes & 1;  // buffer holding the current runs
    for (int r0 = 0; r0 < B; r0 += kSeqSortCap) {
      const int len = min(kSeqSortCap, B - r0);
      for (int k = tid; k < kSeqSortCap; k += kSchedThreads)
        sort_keys[k] = k < len ? seq_key(p, r0 + k) : ~0ull;
      __syncthreads();
      bitonic_sort_smem(sort_keys, kSeqSortCap);
      for (int k = tid; k < len; k += kSchedThreads) buf[cur][r0 + k] = sort_keys[k];
      __syncthreads();
    }
    for (int w = kSeqSortCap; w < B; w <<= 1) {
      const unsigned long long* src = buf[cur];
      unsigned long long* dst = buf[cur ^ 1];
      for (int idx = tid; idx < B; idx += kSchedThreads) {
        const int run = idx / w;
        const int base = (run & ~1) * w;  // first key of the run pair
        const unsigned long long key = src[idx];
        const int a_len = min(w, B - base);
        const int b_len = max(0, min(w, B - base - w));
        int pos;
        if ((run & 1) == 0) pos = (idx - base) + count_below(src + base + w, b_len, key);
        else pos = (idx - base - w) + count_below(src + base, a_len, key);
        dst[base + pos] = key;
      }
      __threadfence_block();
      __syncthreads();
      cur ^= 1;
    }
    ord = p.ws.tmp;  // cur == 0: the sorted keys are in tmp
    for (int r = tid; r < B; r += kSchedThreads) {
      const unsigned long long key = buf[0][r];
      ord[r] = make_int2((int)(unsigned)(key & 0xFFFFFFFFu), 0);
    }
    __threadfence_block();
  }
  __syncthreads();

  // 3. list ranges in that order
  int carry = 0;
  for (int base = 0; base < B; base += kSchedThreads) {
    const int r = base + tid;
    int ng = 0, i = 0;
    if (r < B) {
      i = ord[r].x;
      ng = seq_groups(range_lq(p, i), p.pairing, p.group);
    }
    const int off = carry + block_exclusive_scan(ng, s_warp, &s_total);
    if (r < B) ord[r].y = off;
    carry += s_total;
  }
  const int P = carry;
  __threadfence_block();
  __syncthreads();
  if (P > p.ws.capacity) {  // cannot happen once lengths <= max_q (checked above)
    if (tid == 0) {
      atomicCAS(p.error, 0, kErrBadSeqlens);
      *p.ws.count = 0;
      *p.ws.counter = 0;
    }
    return;
  }

  // 4. pairs of each sequence (one warp per sequence, lanes over its pairs)
  const int lane = tid & 31, warp = tid >> 5;
  for (int r = warp; r < B; r += kSchedThreads / 32) {
    const int2 o = ord[r];
    const int i = o.x;
    const int Lq = range_lq(p, i), Lk = range_lk(p, i);
    const int ng = seq_groups(Lq, p.pairing, p.group);
    // a pair whose second unit does not exist (the last pair of an odd
    // number of units) may do less work than the pairs before it
    const int units = p.pairing == kPairHeads ? p.group * ceil_div(Lq, BM) : ceil_div(Lq, BM);
    const bool lone = p.pairing != kPackGQA && (units & 1);
    const int m = lone ? ng - 1 : ng;  // full pairs: work non-decreasing in g
    int cnt = m;                         // place of the lone pair
    if (lone) {
      const int e = pair_work(ng - 1, Lq, Lk, p.pairing, p.group, p.causal);
      if (p.causal) {  // full pairs in descending order: the lone one follows those with more work
        int lo = 0, hi = m;  // first full g with work > e
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (pair_work(mid, Lq, Lk, p.pairing, p.group, p.causal) > e) hi = mid;
          else lo = mid + 1;
        }
        cnt = m - lo;
      }
    }
    for (int g = lane; g < ng; g += 32) {
      int pos;
      if (lone && g == ng - 1) {
        pos = cnt;
      } else {
        const int rank = p.causal ? m - 1 - g : g;
        pos = rank + (rank >= cnt ? 1 : 0);
      }
      p.ws.list[o.y + pos] = make_int2(i, g);
    }
  }
  __syncthreads();
  if (tid == 0) {
    *p.ws.count = P * p.n_hg;
    *p.ws.counter = 0;
  }
}

}  // namespace va
