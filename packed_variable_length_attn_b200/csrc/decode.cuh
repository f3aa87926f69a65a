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
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include "attn_sm100.cuh"  // Ctl, bounded barrier waits
#include "common.cuh"
#include "ptx.cuh"

namespace va {

constexpr int kDecThreads = 256;
constexpr int kDecKeys = 32;     // keys per block of the ring (one per lane in the softmax)
constexpr int kDecStages = 2;    // ring depth: one block in flight while one is used
constexpr int kDecMaxRows = 32;  // q_len x G rows per CTA

struct DecodeParams {
  const __nv_bfloat16* q;       // [Tq, Hq, D]
  const int* cu_q;              // [B+1]
  __nv_bfloat16* k_cache;       // [B, S, Hkv, D]
  __nv_bfloat16* v_cache;
  const int* cache_seqlens;     // [B]
  const __nv_bfloat16* k_new;   // [Tq, Hkv, D] or null
  const __nv_bfloat16* v_new;
  int batch, total_q, cache_len, n_heads, n_kv_heads, group, causal, n_splits;
  int split_blocks;             // key blocks per split, the same for every sequence
  float scale_log2;             // softmax_scale * log2(e)
  __nv_bfloat16* out;           // [Tq, Hq, D]
  float* lse;                   // [Hq, Tq] or null
  float* part_o;                // [n_splits, Tq, Hq, D] (n_splits > 1)
  float* part_lse;              // [n_splits, Hq, Tq]
  int* error;
};

// bf16 -> fp32 is exact: the bf16 bits are the upper half of the fp32 bits.
// Integer shifts / masks keep the conversions off the XU pipe.
__device__ __forceinline__ float bf16_lo(uint32_t two) { return __uint_as_float(two << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t two) { return __uint_as_float(two & 0xffff0000u); }

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Key blocks [b0, b1) of split `split` of a sequence with nblk_all blocks: the
// splits are fixed ranges of the cache (split_blocks blocks each), so a split
// costs the same in every sequence and the shorter sequences leave their last
// splits empty. An empty split (with more than one split) only marks its rows'
// partial LSE as -inf, which the combine skips.
__device__ __forceinline__ bool split_range(const DecodeParams& p, int split, int nblk_all, int q0,
                                            int R, int g, int& b0, int& b1) {
  b0 = split * p.split_blocks;
  b1 = min(nblk_all, b0 + p.split_blocks);
  if (b1 > b0 || p.n_splits == 1) return true;
  for (int rho = threadIdx.x; rho < R; rho += blockDim.x) {
    const int r = rho / p.group, h = g * p.group + (rho - r * p.group);
    p.part_lse[(long long)split * p.n_heads * p.total_q + (long long)h * p.total_q + q0 + r] = -INFINITY;
  }
  return false;
}

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

template <int D, int RT>
struct DecSmem {
  // K rows are padded by 64 bytes: with the interleaved dim slices of the
  // score pass (thread c of a key reads dims 32m + 4c .. +3), the four keys a
  // warp covers then fall on alternate bank halves and each 8-byte load
  // instruction takes the minimum two wavefronts.
  static constexpr int kKS = D + 32;        // K row stride (bf16 elements)
  static constexpr int kKV = kDecKeys * kKS;  // bf16 elements per K (or V) block slot
  // K and V ring (kDecStages blocks) | Q [RT][D] fp32 | P [kDecKeys][RT] fp32 | m, l, f [RT]
  static constexpr int kKVBytes = kDecStages * 2 * kKV * 2;
  static constexpr int kBytes = kKVBytes + RT * D * 4 + kDecKeys * RT * 4 + 3 * RT * 4;
  static_assert(RT * D * 4 <= kKVBytes, "the final O reduction reuses the K/V buffers");
};

// One CTA: key split blockIdx.x of K/V head blockIdx.y of sequence blockIdx.z;
// RT >= q_len * G query rows (rho = r * G + hl: query token r, head g*G + hl).
// Per 64-key block:
//   scores  8 threads per key, each a D/8 slice of the dot products of all
//           rows with that key (the key is read once and used RT times),
//           reduced over the 8 threads with shuffles;
//   softmax one warp per row (online max / sum over the block);
//   P V     each thread two output dims of every row, over its group of
//           keys; the key groups' partial O are added once at the end.
template <int D, int RT>
__global__ void __launch_bounds__(kDecThreads, RT <= 8 ? 4 : 2) decode_kernel(DecodeParams p) {
  extern __shared__ __align__(16) uint8_t dsm[];
  using S = DecSmem<D, RT>;
  constexpr int kTPK = 8;                       // threads per key (scores)
  constexpr int kDPT = D / kTPK;                // dims per thread (16 or 8)
  constexpr int kKPP = kDecThreads / kTPK;      // keys per score pass (32)
  constexpr int kNPair = D / 2;                 // output dim pairs (64 or 32)
  constexpr int kNKG = kDecThreads / kNPair;    // key groups in P V (4 or 8)
  constexpr int kKPG = kDecKeys / kNKG;         // keys per group (16 or 8)
  __nv_bfloat16* kbuf = reinterpret_cast<__nv_bfloat16*>(dsm);            // [stages][64][D]
  __nv_bfloat16* vbuf = kbuf + kDecStages * S::kKV;                        // [stages][64][D]
  float* qs = reinterpret_cast<float*>(vbuf + kDecStages * S::kKV);        // [RT][D]
  float* ps = qs + RT * D;                                                 // [64][RT]
  float* m_s = ps + kDecKeys * RT;
  float* l_s = m_s + RT;
  float* f_s = l_s + RT;

  const int split = blockIdx.x, g = blockIdx.y, i = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q0 = p.cu_q[i], Lq = p.cu_q[i + 1] - q0;
  const int G = p.group;
  const int R = Lq * G;
  if (Lq <= 0) return;
  const int Lk = p.cache_seqlens[i] + (p.k_new ? Lq : 0);
  if (R > RT || Lk > p.cache_len || Lk < 0) {
    if (tid == 0) atomicCAS(p.error, 0, kErrBadSeqlens);
    return;
  }
  // this split's keys, in whole blocks
  const int nblk_all = (Lk + kDecKeys - 1) / kDecKeys;
  int b0, b1;
  if (!split_range(p, split, nblk_all, q0, R, g, b0, b1)) return;

  for (int e = tid; e < RT * D; e += kDecThreads) {
    const int rho = e / D, d = e - rho * D;
    float v = 0.f;
    if (rho < R) {
      const int r = rho / G, hl = rho - r * G;
      v = __bfloat162float(p.q[((long long)(q0 + r) * p.n_heads + g * G + hl) * D + d]);
    }
    qs[e] = v;
  }
  for (int rho = tid; rho < RT; rho += kDecThreads) {
    m_s[rho] = -INFINITY;
    l_s[rho] = 0.f;
  }
  const int dp = tid % kNPair, kg = tid / kNPair;  // P V: dims 2dp, 2dp+1; key group kg
  // O accumulators: dims 2dp and 2dp + 1 of the row pairs (2i, 2i + 1), as
  // packed fp32 pairs (one packed FMA updates two rows)
  uint64_t ax[RT / 2], ay[RT / 2];
#pragma unroll
  for (int i = 0; i < RT / 2; ++i) ax[i] = ay[i] = 0ull;

  const long long row_stride = (long long)p.n_kv_heads * D;  // elements between cache rows
  const __nv_bfloat16* kbase = p.k_cache + (long long)i * p.cache_len * row_stride + (long long)g * D;
  const __nv_bfloat16* vbase = p.v_cache + (long long)i * p.cache_len * row_stride + (long long)g * D;
  constexpr int kUnitsPerRow = D / 8;  // 16-byte units per key row
  auto load_block = [&](int blk, int buf) {
    const int k0 = blk * kDecKeys;
    for (int e = tid; e < kDecKeys * kUnitsPerRow; e += kDecThreads) {
      const int kr = e / kUnitsPerRow, u = e - kr * kUnitsPerRow;
      __nv_bfloat16* kd = kbuf + buf * S::kKV + kr * S::kKS + u * 8;
      __nv_bfloat16* vd = vbuf + buf * S::kKV + kr * S::kKS + u * 8;
      if (k0 + kr < Lk) {
        cp_async16(kd, kbase + (long long)(k0 + kr) * row_stride + u * 8);
        cp_async16(vd, vbase + (long long)(k0 + kr) * row_stride + u * 8);
      } else {  // past the end: zeros (masked anyway, and keep P V finite)
        *reinterpret_cast<uint4*>(kd) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(vd) = make_uint4(0, 0, 0, 0);
      }
    }
  };
#pragma unroll
  for (int st = 0; st < kDecStages - 1; ++st) {
    if (b0 + st < b1) load_block(b0 + st, st);
    cp_async_commit();
  }
  __syncthreads();  // Q, m, l visible

  for (int blk = b0; blk < b1; ++blk) {
    const int buf = (blk - b0) % kDecStages;
    const int ahead = blk + kDecStages - 1;
    if (ahead < b1) load_block(ahead, (ahead - b0) % kDecStages);
    cp_async_commit();
    cp_async_wait<kDecStages - 1>();  // block blk has landed
    __syncthreads();
    const __nv_bfloat16* kb = kbuf + buf * S::kKV;
    const __nv_bfloat16* vb = vbuf + buf * S::kKV;
    const int k0 = blk * kDecKeys;
    // scores (log2 domain); thread c of a key holds dims 32m + 4c .. 32m + 4c + 3
#pragma unroll
    for (int pass = 0; pass < kDecKeys / kKPP; ++pass) {
      const int kr = pass * kKPP + tid / kTPK, c = tid % kTPK;
      uint64_t kf[kDPT / 2];  // dim pairs (4c + 32m, +1) and (+2, +3)
#pragma unroll
      for (int m = 0; m < D / 32; ++m) {
        const uint2 raw = *reinterpret_cast<const uint2*>(kb + kr * S::kKS + 32 * m + 4 * c);
        kf[2 * m] = ptx::f2(bf16_lo(raw.x), bf16_hi(raw.x));
        kf[2 * m + 1] = ptx::f2(bf16_lo(raw.y), bf16_hi(raw.y));
      }
      const int key = k0 + kr;
#pragma unroll 1
      for (int r0 = 0; r0 < RT; r0 += 4) {  // four rows at a time (bounded registers)
        float part[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float* qrow = qs + (r0 + j) * D + 4 * c;
          uint64_t ab = 0ull;  // even dims | odd dims
#pragma unroll
          for (int m = 0; m < D / 32; ++m) {
            const ulonglong2 qv = *reinterpret_cast<const ulonglong2*>(qrow + 32 * m);
            ab = ptx::ffma2(qv.x, kf[2 * m], ab);
            ab = ptx::ffma2(qv.y, kf[2 * m + 1], ab);
          }
          float a, b;
          ptx::f2_split(ab, a, b);
          part[j] = a + b;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
          for (int o = 1; o < kTPK; o <<= 1) part[j] += __shfl_xor_sync(0xffffffffu, part[j], o);
        }
        if (c == 0) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int rho = r0 + j, r = rho / G;
            const bool vis = rho < R && key < Lk && (!p.causal || key <= r + Lk - Lq);
            ps[kr * RT + rho] = vis ? part[j] * p.scale_log2 : -INFINITY;
          }
        }
      }
    }
    __syncthreads();
    // online softmax: one warp per row, one key per lane
    static_assert(kDecKeys == 32, "one key per lane");
    for (int rho = warp; rho < R; rho += kDecThreads / 32) {
      const float s0 = ps[lane * RT + rho];
      float mx = s0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_old = m_s[rho];
      const float m_new = fmaxf(m_old, mx);
      const float mb = m_new == -INFINITY ? 0.f : m_new;
      const float e0 = exp2f(s0 - mb);
      ps[lane * RT + rho] = e0;
      float sum = e0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) {
        const float fac = m_old == -INFINITY ? 0.f : exp2f(m_old - mb);
        f_s[rho] = fac;
        l_s[rho] = l_s[rho] * fac + sum;
        m_s[rho] = m_new;
      }
    }
    for (int rho = R + tid; rho < RT; rho += kDecThreads) {  // rows past R: no contribution
      f_s[rho] = 0.f;
      for (int kk = 0; kk < kDecKeys; ++kk) ps[kk * RT + rho] = 0.f;
    }
    __syncthreads();
    // O = O * fac + P V over this thread's key group
#pragma unroll
    for (int i = 0; i < RT / 2; ++i) {
      const uint64_t f = *reinterpret_cast<const uint64_t*>(f_s + 2 * i);
      ax[i] = ptx::ffma2(ax[i], f, 0ull);
      ay[i] = ptx::ffma2(ay[i], f, 0ull);
    }
#pragma unroll 4
    for (int kk = 0; kk < kKPG; ++kk) {
      const int key = kg * kKPG + kk;
      const uint32_t vraw = *reinterpret_cast<const uint32_t*>(vb + key * S::kKS + 2 * dp);
      const float vx = bf16_lo(vraw), vy = bf16_hi(vraw);
      const uint64_t vx2 = ptx::f2(vx, vx), vy2 = ptx::f2(vy, vy);
      const ulonglong2* prow = reinterpret_cast<const ulonglong2*>(ps + key * RT);
#pragma unroll
      for (int r4 = 0; r4 < RT / 4; ++r4) {
        const ulonglong2 pp = prow[r4];  // rows (4r4, 4r4 + 1) | (4r4 + 2, 4r4 + 3)
        ax[2 * r4] = ptx::ffma2(pp.x, vx2, ax[2 * r4]);
        ay[2 * r4] = ptx::ffma2(pp.x, vy2, ay[2 * r4]);
        ax[2 * r4 + 1] = ptx::ffma2(pp.y, vx2, ax[2 * r4 + 1]);
        ay[2 * r4 + 1] = ptx::ffma2(pp.y, vy2, ay[2 * r4 + 1]);
      }
    }
    __syncthreads();  // this stage is reloaded by the next iteration; ps, f_s reused
  }
  cp_async_wait<0>();
  __syncthreads();

  // add the key groups' partial O in a fixed order (deterministic), in the
  // now free K/V buffers: O [RT][D] fp32
  float* osum = reinterpret_cast<float*>(dsm);
  for (int grp = 0; grp < kNKG; ++grp) {
    if (kg == grp) {
#pragma unroll
      for (int i = 0; i < RT / 2; ++i) {
        float x0, x1, y0, y1;
        ptx::f2_split(ax[i], x0, x1);
        ptx::f2_split(ay[i], y0, y1);
        float2* d0 = reinterpret_cast<float2*>(osum + (2 * i) * D + 2 * dp);
        float2* d1 = reinterpret_cast<float2*>(osum + (2 * i + 1) * D + 2 * dp);
        const float2 p0 = grp == 0 ? make_float2(0.f, 0.f) : *d0;
        const float2 p1 = grp == 0 ? make_float2(0.f, 0.f) : *d1;
        *d0 = make_float2(p0.x + x0, p0.y + y0);
        *d1 = make_float2(p1.x + x1, p1.y + y1);
      }
    }
    __syncthreads();
  }

  // epilogue: normalise; one split writes the result, several write partials
  for (int e = tid; e < R * D; e += kDecThreads) {
    const int rho = e / D, d = e - rho * D;
    const int r = rho / G, h = g * G + (rho - r * G);
    const float l = l_s[rho];
    const float o = l > 0.f ? osum[e] / l : 0.f;
    const long long oi = ((long long)(q0 + r) * p.n_heads + h) * D + d;
    if (p.n_splits == 1)
      p.out[oi] = __float2bfloat16_rn(o);
    else
      p.part_o[(long long)split * p.total_q * p.n_heads * D + oi] = o;
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
        if (ls == -INFINITY) continue;  // an empty split (its O was never written)
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

// ---------------------------------------------------------------------------
// Decode with a TMA ring and warp-owned key blocks, for up to kDec2MaxRows
// query rows per (sequence, K/V head) (q_len x G; a decode step with G <= 8).
//
// One CTA per (key split, K/V head, sequence), five warps:
//   warp 4      producer: one lane issues the TMA tile loads of each 32-key
//               block (K then V, 64-column 128-byte-swizzled boxes of the
//               cache [batch * cache_len, n_kv_heads, D]) into a kDec2Stages
//               mbarrier ring;
//   warps 0-3   consumers: warp w takes blocks w, w + 4, ... of the split and
//               keeps its own online softmax (max, sum, O) for every row:
//               scores with one key per lane (the key's row is read once and
//               used for every query row), the block's max and sum by warp
//               shuffles, P V with four (head_dim 128) or two (64) output
//               dims per lane and P broadcast from shared memory.
// No CTA barrier runs inside the loop; at the end the four warps' states are
// merged in a fixed order (deterministic), as several key splits are by the
// combine kernel. Keys at or past the sequence's length are masked in the
// scores and skipped in P V, so whatever the cache holds there (old rows,
// NaN) never reaches the output. Every barrier wait is bounded (Ctl): on
// expiry the error word gets kErrTimeout and the CTA returns.
constexpr int kDec2Consumers = 4;
constexpr int kDec2Threads = 32 * (kDec2Consumers + 1);
constexpr int kDec2Stages = 4;
constexpr int kDec2MaxRows = 16;
// Block t goes to stage t % kDec2Stages and consumer warp t % kDec2Consumers.
// A consumer reaches block t only after block t - kDec2Consumers, so with at
// least as many stages as consumers the stage's previous fill (block
// t - kDec2Stages) has already landed and a parity wait can never match an
// older phase of the barrier.
static_assert(kDec2Consumers <= kDec2Stages, "a consumer must never run two fills ahead");

template <int D, int RT>
struct Dec2Cfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kBox = kDecKeys * 128;        // 32 rows x 128 B (64 dims)
  static constexpr int kTile = kChunks * kBox;       // K (or V) of one block
  static constexpr int kStage = 2 * kTile;           // K then V
  static constexpr int kQOff = kDec2Stages * kStage;             // q [RT][D] fp32
  static constexpr int kPOff = kQOff + RT * D * 4;               // P [warp][32][RT] fp32
  static constexpr int kBarOff = kPOff + kDec2Consumers * kDecKeys * RT * 4;
  static constexpr int kMiscOff = kBarOff + 2 * kDec2Stages * 8;  // abort flag
  static constexpr int kBytes = kMiscOff + 16 + 1024;             // + alignment slack
  // the merge at the end reuses the ring: per warp m, l [RT] and O [RT][D]
  static_assert(kDec2Consumers * RT * (D + 2) * 4 <= kDec2Stages * kStage, "merge area");
};

template <int D, int RT>
__global__ void __launch_bounds__(kDec2Threads) decode_tma_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    DecodeParams p, long long wait_limit) {
  extern __shared__ uint8_t dsm_raw[];
  using C = Dec2Cfg<D, RT>;
  constexpr int kDPL = D / 32;  // output dims per lane in P V
  uint8_t* sm;
  {
    const uint32_t a = ptx::smem_u32(dsm_raw);
    sm = dsm_raw + ((1024 - (a & 1023)) & 1023);  // 128-byte swizzle: 1024-byte aligned
  }
  float* qs = reinterpret_cast<float*>(sm + C::kQOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + C::kBarOff);
  uint64_t* empty = full + kDec2Stages;
  int* abort_flag = reinterpret_cast<int*>(sm + C::kMiscOff);

  const int split = blockIdx.x, g = blockIdx.y, i = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q0 = p.cu_q[i], Lq = p.cu_q[i + 1] - q0;
  const int G = p.group;
  const int R = Lq * G;
  if (Lq <= 0) return;
  const int Lk = p.cache_seqlens[i] + (p.k_new ? Lq : 0);
  if (R > RT || Lk > p.cache_len || Lk < 0) {
    if (tid == 0) atomicCAS(p.error, 0, kErrBadSeqlens);
    return;
  }
  const int nblk_all = (Lk + kDecKeys - 1) / kDecKeys;
  int b0, b1;
  if (!split_range(p, split, nblk_all, q0, R, g, b0, b1)) return;
  const int nblk = max(0, b1 - b0);

  if (tid == 0) {
    for (int st = 0; st < kDec2Stages; ++st) {
      ptx::mbar_init(full + st, 1);
      ptx::mbar_init(empty + st, 1);
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  for (int e = tid; e < RT * D; e += kDec2Threads) {
    const int rho = e / D, d = e - rho * D;
    float v = 0.f;
    if (rho < R) {
      const int r = rho / G, hl = rho - r * G;
      v = __bfloat162float(p.q[((long long)(q0 + r) * p.n_heads + g * G + hl) * D + d]);
    }
    qs[e] = v;
  }
  __syncthreads();
  const Ctl ctl{abort_flag, p.error, wait_limit};
  const long long row0 = (long long)i * p.cache_len;  // first cache row of sequence i

  float m[RT], l[RT];
  float o[RT][kDPL];
#pragma unroll
  for (int r = 0; r < RT; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int d = 0; d < kDPL; ++d) o[r][d] = 0.f;
  }

  if (warp == kDec2Consumers) {
    // ---- producer
    int t = 0;
    for (; t < nblk; ++t) {
      const int st = t % kDec2Stages;
      if (!__all_sync(0xffffffffu, wait_bar(empty + st, ((t / kDec2Stages) & 1) ^ 1, ctl))) break;
      if (ptx::elect_one()) {
        uint8_t* dst = sm + st * C::kStage;
        const int row = (int)(row0 + (long long)(b0 + t) * kDecKeys);
        ptx::mbar_arrive_expect_tx(full + st, C::kStage);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c) {
          ptx::tma_load_3d(dst + c * C::kBox, &tm_k, full + st, c * 64, g, row);
          ptx::tma_load_3d(dst + C::kTile + c * C::kBox, &tm_v, full + st, c * 64, g, row);
        }
      }
      __syncwarp();
    }
    // wait (bounded) for every copy issued into each stage
    for (int st = 0; st < kDec2Stages && st < t; ++st) {
      const int uses = (t - 1 - st) / kDec2Stages + 1;
      drain_bar(full + st, (uses - 1) & 1);
    }
  } else {
    // ---- consumer warp: blocks t = warp, warp + 4, ...
    float* pw = reinterpret_cast<float*>(sm + C::kPOff) + warp * kDecKeys * RT;  // [32][RT]
    const int q_last = Lk - Lq;  // bottom-right causal: row r sees keys <= r + q_last
    for (int t = warp; t < nblk; t += kDec2Consumers) {
      const int st = t % kDec2Stages;
      if (!__all_sync(0xffffffffu, wait_bar(full + st, (t / kDec2Stages) & 1, ctl))) break;
      const uint8_t* kt = sm + st * C::kStage;
      const uint8_t* vt = kt + C::kTile;
      const int k0 = (b0 + t) * kDecKeys;
      const int key = k0 + lane;
      // scores: this lane's key against every row (row `lane` of each box,
      // 16-byte unit u stored at unit u ^ (lane & 7))
      uint64_t acc[RT];
#pragma unroll
      for (int r = 0; r < RT; ++r) acc[r] = 0ull;
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 kv = ptx::ld_shared_v4(ptx::smem_u32(kt + c * C::kBox + lane * 128 +
                                                           ((u ^ (lane & 7)) << 4)));
          const uint64_t k01 = ptx::f2(bf16_lo(kv.x), bf16_hi(kv.x));
          const uint64_t k23 = ptx::f2(bf16_lo(kv.y), bf16_hi(kv.y));
          const uint64_t k45 = ptx::f2(bf16_lo(kv.z), bf16_hi(kv.z));
          const uint64_t k67 = ptx::f2(bf16_lo(kv.w), bf16_hi(kv.w));
          const int d0 = c * 64 + u * 8;
#pragma unroll
          for (int r = 0; r < RT; ++r) {
            const ulonglong2 qa = *reinterpret_cast<const ulonglong2*>(qs + r * D + d0);
            const ulonglong2 qb = *reinterpret_cast<const ulonglong2*>(qs + r * D + d0 + 4);
            acc[r] = ptx::ffma2(qa.x, k01, acc[r]);
            acc[r] = ptx::ffma2(qa.y, k23, acc[r]);
            acc[r] = ptx::ffma2(qb.x, k45, acc[r]);
            acc[r] = ptx::ffma2(qb.y, k67, acc[r]);
          }
        }
      }
      // online softmax per row (log2 domain); masked keys give P = 0 exactly
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        float lo, hi;
        ptx::f2_split(acc[r], lo, hi);
        const bool vis = r < R && key < Lk && (!p.causal || key <= r / G + q_last);
        const float s = vis ? (lo + hi) * p.scale_log2 : -INFINITY;
        float mx = s;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_new = fmaxf(m[r], mx);
        const float mb = m_new == -INFINITY ? 0.f : m_new;
        const float pr = ptx::ex2(s - mb);
        float sum = pr;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        const float fac = ptx::ex2(m[r] - mb);  // 0 while m[r] is -inf
        l[r] = l[r] * fac + sum;
        m[r] = m_new;
#pragma unroll
        for (int d = 0; d < kDPL; ++d) o[r][d] *= fac;
        pw[lane * RT + r] = pr;
      }
      __syncwarp();
      // P V: this lane's output dims d0 .. d0 + kDPL - 1 over the block's keys
      const int d0 = lane * kDPL;
      const int vc = d0 / 64, vb = (d0 % 64) * 2;  // chunk, byte offset in the 128-byte row
      const int nk = min(kDecKeys, Lk - k0);       // keys past the length are skipped
      for (int kk = 0; kk < nk; ++kk) {
        const uint32_t va = ptx::smem_u32(vt + vc * C::kBox + kk * 128) +
                            (uint32_t)(((((vb >> 4) ^ (kk & 7)) << 4)) | (vb & 15));
        float v[kDPL];
        if constexpr (kDPL == 4) {
          uint32_t x, y;
          asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(x), "=r"(y) : "r"(va));
          v[0] = bf16_lo(x); v[1] = bf16_hi(x); v[2] = bf16_lo(y); v[3] = bf16_hi(y);
        } else {
          uint32_t x;
          asm volatile("ld.shared.b32 %0, [%1];" : "=r"(x) : "r"(va));
          v[0] = bf16_lo(x); v[1] = bf16_hi(x);
        }
        const float* prow = pw + kk * RT;
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          const float pr = prow[r];
#pragma unroll
          for (int d = 0; d < kDPL; ++d) o[r][d] = fmaf(pr, v[d], o[r][d]);
        }
      }
      __syncwarp();  // pw is rewritten by the next block
      if (lane == 0) ptx::mbar_arrive(empty + st);
    }
  }
  __syncthreads();  // every copy has landed and every block has been read

  // merge the consumer warps' states (fixed order) in the ring's space
  float* mm = reinterpret_cast<float*>(sm);                    // [warp][RT]
  float* ll = mm + kDec2Consumers * RT;                        // [warp][RT]
  float* oo = ll + kDec2Consumers * RT;                        // [warp][RT][D]
  if (warp < kDec2Consumers) {
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      if (lane == 0) {
        mm[warp * RT + r] = m[r];
        ll[warp * RT + r] = l[r];
      }
#pragma unroll
      for (int d = 0; d < kDPL; ++d) oo[(warp * RT + r) * D + lane * kDPL + d] = o[r][d];
    }
  }
  __syncthreads();
  for (int e = tid; e < R * D; e += kDec2Threads) {
    const int rho = e / D, d = e - rho * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDec2Consumers; ++w) M = fmaxf(M, mm[w * RT + rho]);
    const float mb = M == -INFINITY ? 0.f : M;
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kDec2Consumers; ++w) {
      const float f = ptx::ex2(mm[w * RT + rho] - mb);
      L += ll[w * RT + rho] * f;
      O += oo[(w * RT + rho) * D + d] * f;
    }
    const int r = rho / G, h = g * G + (rho - r * G);
    const float val = L > 0.f ? O / L : 0.f;
    const long long oi = ((long long)(q0 + r) * p.n_heads + h) * D + d;
    if (p.n_splits == 1)
      p.out[oi] = __float2bfloat16_rn(val);
    else
      p.part_o[(long long)split * p.total_q * p.n_heads * D + oi] = val;
    if (d == 0) {
      const float lse = L > 0.f ? (M + __log2f(L)) * 0.6931471805599453f : -INFINITY;
      const long long li = (long long)h * p.total_q + q0 + r;
      if (p.n_splits == 1) {
        if (p.lse) p.lse[li] = lse;
      } else {
        p.part_lse[(long long)split * p.n_heads * p.total_q + li] = lse;
      }
    }
  }
}

}  // namespace va
