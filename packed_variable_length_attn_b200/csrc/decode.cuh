// Decode attention over a per-sequence K/V cache (q_len small), split over
// the keys.
//
// Decode reads every cached key and value once and does ~4 FLOP per byte of
// them (G query heads x q_len rows per K/V head), far below the tensor-core
// ridge, so this path runs on the CUDA cores in fp32 and is written for HBM
// bandwidth: one CTA per (key split, K/V head, sequence) streams its split of
// the cache through a double-buffered cp.async ring, and the query rows of
// all G query heads of that K/V head share every key block. With more than
// one split, each CTA writes a normalised partial output and its LSE, and a
// combine kernel merges the splits (O = sum_s exp(LSE_s - LSE) O_s,
// LSE = ln sum_s exp(LSE_s)).
//
// Cache layout: [batch, cache_len, n_kv_heads, D] bf16 (sequence i's rows are
// i*cache_len .. i*cache_len + cache_seqlens[i] - 1). Optional new K/V rows
// (packed like q, [total_q, n_kv_heads, D]) are first written into the cache
// after the cached ones and are then attended to as well.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "common.cuh"

namespace va {

constexpr int kDecThreads = 256;
constexpr int kDecKeys = 64;     // keys per block of the ring
constexpr int kDecMaxRows = 32;  // q_len x G rows per CTA
constexpr int kDecMaxOut = kDecMaxRows * 128 / kDecThreads;  // O accumulators per thread

struct DecodeParams {
  const __nv_bfloat16* q;       // [Tq, Hq, D]
  const int* cu_q;              // [B+1]
  __nv_bfloat16* k_cache;       // [B, S, Hkv, D]
  __nv_bfloat16* v_cache;
  const int* cache_seqlens;     // [B]
  const __nv_bfloat16* k_new;   // [Tq, Hkv, D] or null
  const __nv_bfloat16* v_new;
  int batch, total_q, cache_len, n_heads, n_kv_heads, group, causal, n_splits;
  float scale_log2;             // softmax_scale * log2(e)
  __nv_bfloat16* out;           // [Tq, Hq, D]
  float* lse;                   // [Hq, Tq] or null
  float* part_o;                // [n_splits, Tq, Hq, D] (n_splits > 1)
  float* part_lse;              // [n_splits, Hq, Tq]
  int* error;
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Writes the new K/V rows of every sequence into its cache rows
// [cache_seqlens[i], cache_seqlens[i] + Lq_i); 16-byte units, grid-stride.
template <int D>
__global__ void __launch_bounds__(kDecThreads) decode_append_kernel(DecodeParams p) {
  const int units = p.n_kv_heads * D / 8;  // 16-byte units per token row
  const long long n = (long long)p.total_q * units;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(e / units), u = (int)(e - (long long)t * units);
    if (t >= p.cu_q[p.batch]) continue;
    int lo = 0, hi = p.batch;  // sequence of query row t: cu_q[lo] <= t < cu_q[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.cu_q[mid] <= t) lo = mid;
      else hi = mid;
    }
    const int r = t - p.cu_q[lo];
    const int pos = p.cache_seqlens[lo] + r;
    if (r < 0 || t >= p.cu_q[lo + 1] || pos < 0 || pos >= p.cache_len) {
      if (u == 0) atomicCAS(p.error, 0, kErrBadSeqlens);
      continue;
    }
    const long long dst = ((long long)lo * p.cache_len + pos) * units + u;
    reinterpret_cast<uint4*>(p.k_cache)[dst] = reinterpret_cast<const uint4*>(p.k_new)[e];
    reinterpret_cast<uint4*>(p.v_cache)[dst] = reinterpret_cast<const uint4*>(p.v_new)[e];
  }
}

template <int D>
struct DecSmem {
  static constexpr int kKV = kDecKeys * D;                   // bf16 elements per block
  static constexpr int kBytes = 2 * 2 * kKV * 2              // K and V, double-buffered
                                + kDecMaxRows * D * 4        // Q (fp32)
                                + kDecMaxRows * kDecKeys * 4 // scores / P
                                + 3 * kDecMaxRows * 4;       // m, l, rescale factor
};

template <int D>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(DecodeParams p) {
  extern __shared__ __align__(16) uint8_t dsm[];
  using S = DecSmem<D>;
  __nv_bfloat16* kbuf = reinterpret_cast<__nv_bfloat16*>(dsm);            // [2][64][D]
  __nv_bfloat16* vbuf = kbuf + 2 * S::kKV;                                 // [2][64][D]
  float* qs = reinterpret_cast<float*>(vbuf + 2 * S::kKV);                 // [R][D]
  float* ps = qs + kDecMaxRows * D;                                        // [R][64]
  float* m_s = ps + kDecMaxRows * kDecKeys;
  float* l_s = m_s + kDecMaxRows;
  float* f_s = l_s + kDecMaxRows;

  const int split = blockIdx.x, g = blockIdx.y, i = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q0 = p.cu_q[i], Lq = p.cu_q[i + 1] - q0;
  const int G = p.group;
  const int R = Lq * G;
  if (Lq <= 0) return;
  const int Lk = p.cache_seqlens[i] + (p.k_new ? Lq : 0);
  if (R > kDecMaxRows || Lk > p.cache_len || Lk < 0) {
    if (tid == 0) atomicCAS(p.error, 0, kErrBadSeqlens);
    return;
  }
  // this split's keys, in whole blocks
  const int nblk_all = (Lk + kDecKeys - 1) / kDecKeys;
  const int per = (nblk_all + p.n_splits - 1) / p.n_splits;
  const int b0 = split * per, b1 = min(nblk_all, b0 + per);

  // rows: rho = r * G + hl (query token r, query head g*G + hl)
  for (int e = tid; e < R * D; e += kDecThreads) {
    const int rho = e / D, d = e - rho * D;
    const int r = rho / G, hl = rho - r * G;
    qs[e] = __bfloat162float(p.q[((long long)(q0 + r) * p.n_heads + g * G + hl) * D + d]);
  }
  for (int rho = tid; rho < kDecMaxRows; rho += kDecThreads) {
    m_s[rho] = -INFINITY;
    l_s[rho] = 0.f;
  }
  float acc[kDecMaxOut];
#pragma unroll
  for (int j = 0; j < kDecMaxOut; ++j) acc[j] = 0.f;

  const long long row_stride = (long long)p.n_kv_heads * D;  // elements between cache rows
  const __nv_bfloat16* kbase = p.k_cache + (long long)i * p.cache_len * row_stride + (long long)g * D;
  const __nv_bfloat16* vbase = p.v_cache + (long long)i * p.cache_len * row_stride + (long long)g * D;
  constexpr int kUnitsPerRow = D / 8;  // 16-byte units per key row
  auto load_block = [&](int blk, int buf) {
    const int k0 = blk * kDecKeys;
    for (int e = tid; e < kDecKeys * kUnitsPerRow; e += kDecThreads) {
      const int kr = e / kUnitsPerRow, u = e - kr * kUnitsPerRow;
      __nv_bfloat16* kd = kbuf + buf * S::kKV + kr * D + u * 8;
      __nv_bfloat16* vd = vbuf + buf * S::kKV + kr * D + u * 8;
      if (k0 + kr < Lk) {
        cp_async16(kd, kbase + (long long)(k0 + kr) * row_stride + u * 8);
        cp_async16(vd, vbase + (long long)(k0 + kr) * row_stride + u * 8);
      } else {  // past the end: zeros (masked anyway, and keep P V finite)
        *reinterpret_cast<uint4*>(kd) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(vd) = make_uint4(0, 0, 0, 0);
      }
    }
  };
  if (b0 < b1) load_block(b0, 0);
  cp_async_commit();
  __syncthreads();  // Q, m, l visible

  for (int blk = b0; blk < b1; ++blk) {
    const int buf = (blk - b0) & 1;
    if (blk + 1 < b1) load_block(blk + 1, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const __nv_bfloat16* kb = kbuf + buf * S::kKV;
    const __nv_bfloat16* vb = vbuf + buf * S::kKV;
    const int k0 = blk * kDecKeys;
    // scores (log2 domain): thread -> (row, key); the d loop starts at a
    // key-dependent offset so that the 32 keys of a warp hit 32 banks.
    for (int e = tid; e < R * kDecKeys; e += kDecThreads) {
      const int rho = e / kDecKeys, kr = e - rho * kDecKeys;
      const int r = rho / G;
      const int c = k0 + kr;
      float s = -INFINITY;
      const bool visible = c < Lk && (!p.causal || c <= r + Lk - Lq);
      if (visible) {
        const __nv_bfloat162* krow = reinterpret_cast<const __nv_bfloat162*>(kb + kr * D);
        const float2* qrow = reinterpret_cast<const float2*>(qs + rho * D);
        float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
        for (int m = 0; m < D / 2; ++m) {
          const int mm = (m + kr) & (D / 2 - 1);
          const float2 kv = __bfloat1622float2(krow[mm]);
          const float2 qv = qrow[mm];
          a0 = fmaf(qv.x, kv.x, a0);
          a1 = fmaf(qv.y, kv.y, a1);
        }
        s = (a0 + a1) * p.scale_log2;
      }
      ps[rho * kDecKeys + kr] = s;
    }
    __syncthreads();
    // online softmax: one warp per row, two keys per lane
    for (int rho = warp; rho < R; rho += kDecThreads / 32) {
      const float s0 = ps[rho * kDecKeys + lane], s1 = ps[rho * kDecKeys + lane + 32];
      float mx = fmaxf(s0, s1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_old = m_s[rho];
      const float m_new = fmaxf(m_old, mx);
      const float mb = m_new == -INFINITY ? 0.f : m_new;
      const float e0 = exp2f(s0 - mb), e1 = exp2f(s1 - mb);
      ps[rho * kDecKeys + lane] = e0;
      ps[rho * kDecKeys + lane + 32] = e1;
      float sum = e0 + e1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) {
        const float fac = m_old == -INFINITY ? 0.f : exp2f(m_old - mb);
        f_s[rho] = fac;
        l_s[rho] = l_s[rho] * fac + sum;
        m_s[rho] = m_new;
      }
    }
    __syncthreads();
    // O = O * fac + P V: thread -> outputs (row, d) = e, e + 256, ...
#pragma unroll
    for (int j = 0; j < kDecMaxOut; ++j) {
      const int e = tid + j * kDecThreads;
      if (e < R * D) {
        const int rho = e / D, d = e - rho * D;
        float a = acc[j] * f_s[rho];
        const float* prow = ps + rho * kDecKeys;
#pragma unroll 8
        for (int kr = 0; kr < kDecKeys; ++kr) a = fmaf(prow[kr], __bfloat162float(vb[kr * D + d]), a);
        acc[j] = a;
      }
    }
    __syncthreads();  // the buffer is reloaded two blocks later; ps, f_s reused
  }
  cp_async_wait<0>();

  // epilogue: normalise; one split writes the result, several write partials
#pragma unroll
  for (int j = 0; j < kDecMaxOut; ++j) {
    const int e = tid + j * kDecThreads;
    if (e < R * D) {
      const int rho = e / D, d = e - rho * D;
      const int r = rho / G, h = g * G + (rho - r * G);
      const float l = l_s[rho];
      const float o = l > 0.f ? acc[j] / l : 0.f;
      const long long oi = ((long long)(q0 + r) * p.n_heads + h) * D + d;
      if (p.n_splits == 1)
        p.out[oi] = __float2bfloat16_rn(o);
      else
        p.part_o[(long long)split * p.total_q * p.n_heads * D + oi] = o;
    }
  }
  for (int rho = tid; rho < R; rho += kDecThreads) {
    const int r = rho / G, h = g * G + (rho - r * G);
    const float l = l_s[rho];
    const float lse = l > 0.f ? (m_s[rho] + __log2f(l)) * 0.6931471805599453f : -INFINITY;
    const long long li = (long long)h * p.total_q + q0 + r;
    if (p.n_splits == 1) {
      if (p.lse) p.lse[li] = lse;
    } else {
      p.part_lse[(long long)split * p.n_heads * p.total_q + li] = lse;
    }
  }
}

// Merge the splits: per (query row, head), LSE = ln sum_s exp(LSE_s) and
// O = sum_s exp(LSE_s - LSE) O_s (rows that see no key: O = 0, LSE = -inf).
template <int D>
__global__ void __launch_bounds__(kDecThreads) decode_combine_kernel(DecodeParams p) {
  const long long rows = (long long)p.total_q * p.n_heads;
  const int q_end = p.cu_q[p.batch];
  for (long long e = (long long)blockIdx.x * (kDecThreads / 32) + (threadIdx.x >> 5); e < rows;
       e += (long long)gridDim.x * (kDecThreads / 32)) {
    const int t = (int)(e / p.n_heads), h = (int)(e - (long long)t * p.n_heads);
    if (t >= q_end) continue;
    const int lane = threadIdx.x & 31;
    float mx = -INFINITY;
    for (int s = 0; s < p.n_splits; ++s)
      mx = fmaxf(mx, p.part_lse[(long long)s * p.n_heads * p.total_q + (long long)h * p.total_q + t]);
    float wsum = 0.f;
    float o[D / 32];
#pragma unroll
    for (int j = 0; j < D / 32; ++j) o[j] = 0.f;
    if (mx != -INFINITY) {
      for (int s = 0; s < p.n_splits; ++s) {
        const float ls = p.part_lse[(long long)s * p.n_heads * p.total_q + (long long)h * p.total_q + t];
        const float wgt = __expf(ls - mx);
        wsum += wgt;
        const float* po = p.part_o + ((long long)s * p.total_q * p.n_heads + e) * D;
#pragma unroll
        for (int j = 0; j < D / 32; ++j) o[j] = fmaf(wgt, po[lane + 32 * j], o[j]);
      }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
    for (int j = 0; j < D / 32; ++j) p.out[e * D + lane + 32 * j] = __float2bfloat16_rn(o[j] * inv);
    if (lane == 0 && p.lse)
      p.lse[(long long)h * p.total_q + t] = wsum > 0.f ? mx + __logf(wsum) : -INFINITY;
  }
}

}  // namespace va
