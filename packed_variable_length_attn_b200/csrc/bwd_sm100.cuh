// Backward pass of packed variable-length attention for sm_100a.
//
// With P the forward's probabilities (recomputed from Q, K, the biases and
// the forward's LSE), dO the output gradient and delta = rowsum(dO * O):
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - delta),
//   dQ = scale dS K,  dK = scale dS^T Q,  dbias_key = colsum(dS),  dbias_pair = dS
// (the chain rule through the forward definition; the GiGL PR 858 page,
// "Approach", notes that a varlen kernel with a per-sequence bias lacks this
// backward, and the ASpec PR 25 page, "Verification", bounds Q/K/V gradient
// errors at 1% relative L2 against a dense math backend).
//
// Two kernels, one CTA per SM; dQ, dK and dV are computed without atomics,
// so they do not depend on scheduling:
//   attn_bwd_dkdv_sm100: one CTA per (sequence, K/V head, 128-key block).
//     K and V stay in shared memory; for every query head of the group and
//     every 128-row query block that can see the keys, Q and dO arrive by
//     TMA (a ring each) and the tensor cores compute
//       S^T  = K Q^T       (tensor memory cols [0,128): keys are the lanes)
//       dP^T = V dO^T      (cols [128,256))
//     the sixteen compute warps (four per lane quarter, 32 columns each)
//     turn them into P^T and dS^T (bf16, written back over each part's own
//     S^T and dP^T columns), and
//       dV  += P^T dO      (cols [256, 256+D), P^T read from tensor memory)
//       dK  += dS^T Q      (cols [256+D, 256+2D))
//     Each thread owns one key, so the per-key bias gradient is a register
//     sum per part (the four parts add atomically) and the pair-grid gradient
//     rows are written coalesced.
//   attn_bwd_dq_sm100: one CTA per (sequence, query head, 128-row block).
//     Q and dO stay; K and V stream in rings of their own; S = Q K^T,
//     dP = dO V^T, dS as above (one thread per query row and column part),
//     dQ += dS K.
// The pair of kernels recomputes S and dP once more than a single fused
// kernel with atomic dQ accumulation would; in exchange nothing of Q, K, V's
// gradients is reduced across CTAs.
#pragma once
#include <type_traits>

#include "attn_sm100.cuh"

namespace va {

struct BwdParams {
  const int* cu_q;
  const int* cu_k;
  const int* valid;               // 1 when the validation kernel accepted cu_seqlens
  int total_q, total_k;
  int n_heads, n_kv_heads, group;
  int causal;
  float scale;                    // softmax_scale
  const float* lse;               // [Hq, Tq] natural log (forward output)
  const float* delta;             // [Hq, Tq] rowsum(dO * O)
  const float* bias_key;          // [Tk, Hq] or null
  const float* bias_pair;         // strided grid or null
  long long sb, sh, sr, sc;
  int bias_head_div;
  float* dbias_key;               // [Tk, Hq] or null
  float* dbias_pair;              // [B, Hq, R, C] (column stride 1) or null
  long long dsb, dsh, dsr;
  void* dq;                       // bf16 [Tq, Hq, D]
  void* dk;                       // bf16 [Tk, Hkv, D]
  void* dv;                       // bf16 [Tk, Hkv, D]
  int* error;
  long long wait_limit;           // cycles a bounded wait may take
  int test_stall;                 // test hook: the MMA warp first waits on a barrier
                                  // phase nothing completes (its wait runs out)
};

// Compute warps 0-15: warp w reads tensor-memory lanes 32(w % 4) .. +31 and
// the 32 columns 32(w / 4) .. +31 of each 128-column tile (four warps per SM
// sub-partition, for latency hiding). MMA warp 16, load warp 17.
constexpr int kBwdParts = 4;
constexpr int kBwdCompute = 128 * kBwdParts;
constexpr int kBwdThreads = kBwdCompute + 64;
constexpr int kBwdMmaWarp = kBwdCompute / 32;
constexpr int kBwdLoadWarp = kBwdMmaWarp + 1;

// Stages of the two streamed-operand rings (see BwdCfg): 192 KB of shared
// memory in all at head_dim 128, 160 KB at 64.
template <int D>
constexpr int kBwdRingA = D == 64 ? 4 : 3;
template <int D>
constexpr int kBwdRingB = D == 64 ? 4 : 1;

template <int D>
struct BwdCfg {
  static constexpr int kChunk = 128 * 128;               // 128 rows x 64 bf16 (128 B)
  static constexpr int kTile = (D / 64) * kChunk;         // 128 rows x D bf16
  // Two streamed operands with rings of their own: A is read by the first
  // and the last product of a tile (Q in dK/dV: S^T and dK; K in dQ: S and
  // dQ), so its stage is freed late and it gets the deeper ring; B is read
  // by products in the middle (dO: dP^T, dV; V: dP) and is freed earlier.
  static constexpr int kNA = kBwdRingA<D>;
  static constexpr int kNB = kBwdRingB<D>;
  static constexpr int kFixedOff = 0;                     // two resident tiles
  static constexpr int kAOff = 2 * kTile;
  static constexpr int kBOff = kAOff + kNA * kTile;
  static constexpr int kRowOff = kBOff + kNB * kTile;     // float [2 buf][2][128]
  static constexpr int kBarOff = kRowOff + 2 * 2 * 128 * 4;
  // fixed_full, s_full, p_full, o_full, rows_full[2], dp_full, ds_full,
  // a_full[kNA], a_empty[kNA], b_full[kNB], b_empty[kNB]
  static constexpr int kNumBars = 8 + 2 * kNA + 2 * kNB;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem slot, abort flag
  static constexpr int kUsed = kMiscOff + 16 + 1024;       // + alignment slack
  // At least 120 KB so that one CTA (holding all 512 tensor-memory columns)
  // runs per SM.
  static constexpr int kSmemBytes = kUsed < 120 * 1024 ? 120 * 1024 : kUsed;
};

template <int D>
struct BwdSmem {
  uint8_t* base;
  __device__ uint8_t* fixed(int i) const { return base + BwdCfg<D>::kFixedOff + i * BwdCfg<D>::kTile; }
  __device__ uint8_t* ring_a(int st) const { return base + BwdCfg<D>::kAOff + st * BwdCfg<D>::kTile; }
  __device__ uint8_t* ring_b(int st) const { return base + BwdCfg<D>::kBOff + st * BwdCfg<D>::kTile; }
  __device__ float* rows(int b, int i) const {
    return reinterpret_cast<float*>(base + BwdCfg<D>::kRowOff) + (2 * b + i) * 128;
  }
  __device__ uint64_t* bars() const { return reinterpret_cast<uint64_t*>(base + BwdCfg<D>::kBarOff); }
  __device__ uint64_t* fixed_full() const { return bars(); }
  __device__ uint64_t* s_full() const { return bars() + 1; }
  __device__ uint64_t* p_full() const { return bars() + 2; }
  __device__ uint64_t* o_full() const { return bars() + 3; }
  __device__ uint64_t* rows_full(int b) const { return bars() + 4 + b; }
  __device__ uint64_t* dp_full() const { return bars() + 6; }
  __device__ uint64_t* ds_full() const { return bars() + 7; }
  __device__ uint64_t* a_full(int st) const { return bars() + 8 + st; }
  __device__ uint64_t* a_empty(int st) const { return bars() + 8 + BwdCfg<D>::kNA + st; }
  __device__ uint64_t* b_full(int st) const { return bars() + 8 + 2 * BwdCfg<D>::kNA + st; }
  __device__ uint64_t* b_empty(int st) const {
    return bars() + 8 + 2 * BwdCfg<D>::kNA + BwdCfg<D>::kNB + st;
  }
  __device__ uint32_t* tmem_slot() const { return reinterpret_cast<uint32_t*>(base + BwdCfg<D>::kMiscOff); }
  __device__ int* abort_flag() const { return reinterpret_cast<int*>(base + BwdCfg<D>::kMiscOff + 4); }
};

// delta[h, t] = sum_d dO[t, h, d] * O[t, h, d] (fp32 from bf16), one thread
// per (token, head), 16-byte loads.
template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const __nv_bfloat16* __restrict__ out,
                                                        const __nv_bfloat16* __restrict__ dout,
                                                        int total_q, int n_heads,
                                                        float* __restrict__ delta) {
  const long long n = (long long)total_q * n_heads;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const uint4* o = reinterpret_cast<const uint4*>(out + i * D);
    const uint4* g = reinterpret_cast<const uint4*>(dout + i * D);
    float acc = 0.f;
#pragma unroll 4
    for (int u = 0; u < D / 8; ++u) {
      const uint4 a = __ldg(o + u), b = __ldg(g + u);
      const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc = fmaf(__uint_as_float(av[e] << 16), __uint_as_float(bv[e] << 16), acc);
        acc = fmaf(__uint_as_float(av[e] & 0xffff0000u), __uint_as_float(bv[e] & 0xffff0000u), acc);
      }
    }
    const long long t = i / n_heads, h = i % n_heads;
    delta[h * total_q + t] = acc;
  }
}

// Shared setup of both kernels: barriers, tensor memory, smem base.
template <int D>
__device__ __forceinline__ uint32_t bwd_setup(BwdSmem<D>& sm, uint8_t* smem_raw) {
  {
    const uint32_t a = ptx::smem_u32(smem_raw);
    sm.base = smem_raw + ((1024 - (a & 1023)) & 1023);
  }
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    ptx::mbar_init(sm.fixed_full(), 1);
    for (int st = 0; st < BwdCfg<D>::kNA; ++st) {
      ptx::mbar_init(sm.a_full(st), 1);
      ptx::mbar_init(sm.a_empty(st), 1);
    }
    for (int st = 0; st < BwdCfg<D>::kNB; ++st) {
      ptx::mbar_init(sm.b_full(st), 1);
      ptx::mbar_init(sm.b_empty(st), 1);
    }
    ptx::mbar_init(sm.s_full(), 1);
    ptx::mbar_init(sm.p_full(), kBwdCompute);
    ptx::mbar_init(sm.o_full(), 1);
    ptx::mbar_init(sm.rows_full(0), kBwdCompute);
    ptx::mbar_init(sm.rows_full(1), kBwdCompute);
    ptx::mbar_init(sm.dp_full(), 1);
    ptx::mbar_init(sm.ds_full(), kBwdCompute);
    *sm.abort_flag() = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kBwdMmaWarp) {
    ptx::tmem_alloc(sm.tmem_slot(), 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  return *sm.tmem_slot();
}

template <int D>
__device__ __forceinline__ void bwd_teardown(const BwdSmem<D>& sm, uint32_t tmem) {
  ptx::tc_fence_before();
  __syncthreads();
  if ((threadIdx.x >> 5) == kBwdMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// D[tmem] (+)= A[tmem] * B[smem], K = 128 in steps of 16, with A written by
// the four column parts: part p's 32 rows of K (bf16 pairs) sit in columns
// a_base + 32p .. +15, i.e. K step k16 at a_base + 32(k16 / 2) + 8(k16 % 2).
template <int D>
__device__ __forceinline__ void issue_ts_parts(uint32_t d_tmem, uint32_t a_base, uint64_t b_desc,
                                               bool acc) {
  constexpr uint32_t idesc = idesc_bf16(D, true);
#pragma unroll
  for (int k16 = 0; k16 < 8; ++k16)
    ptx::mma_ts(d_tmem, a_base + 32 * (k16 >> 1) + 8 * (k16 & 1),
                b_desc + (uint64_t)((k16 * 16 * 128) >> 4), idesc, (acc || k16 > 0) ? 1u : 0u);
}

// Position of use u in a ring of N stages: stage and mbarrier parity.
template <int N>
__device__ __forceinline__ int ring_stage(int u) { return u % N; }
template <int N>
__device__ __forceinline__ uint32_t ring_parity(int u) { return (uint32_t)((u / N) & 1); }

// Loads a 128-row x D tile (D/64 swizzled chunks) at (head, row).
template <int D>
__device__ __forceinline__ void bwd_load_tile(uint8_t* dst, const CUtensorMap* tm, uint64_t* bar,
                                              int head, int row) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c)
    ptx::tma_load_3d(dst + c * BwdCfg<D>::kChunk, tm, bar, c * 64, head, row);
}

// Accumulator rows of tensor memory (D fp32 columns at `t`) -> bf16 row of
// `dst` times `mul`, or zeros when `have` is false.
template <int C0, int C1>
__device__ __forceinline__ void bwd_store_row(uint32_t t, bool have, float mul, __nv_bfloat16* dst,
                                              bool ok) {
  for (int c = C0; c < C1; ++c) {
    uint32_t v[32];
    if (have) {
      ptx::tmem_ld32(t + c * 32, v);
      ptx::tmem_wait_ld();
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = 0u;
    }
    if (ok) {
      uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint4 w;
        w.x = ptx::pack_bf16x2(__uint_as_float(v[8 * u + 0]) * mul, __uint_as_float(v[8 * u + 1]) * mul);
        w.y = ptx::pack_bf16x2(__uint_as_float(v[8 * u + 2]) * mul, __uint_as_float(v[8 * u + 3]) * mul);
        w.z = ptx::pack_bf16x2(__uint_as_float(v[8 * u + 4]) * mul, __uint_as_float(v[8 * u + 5]) * mul);
        w.w = ptx::pack_bf16x2(__uint_as_float(v[8 * u + 6]) * mul, __uint_as_float(v[8 * u + 7]) * mul);
        d4[u] = w;
      }
    }
  }
}

// The load warp's stream: for t = 0 .. n-1, tile t of operand A (ring A)
// then of operand B (ring B), each once its stage is free; `where(t, head,
// row)` gives the tensor-map coordinates. Afterwards, waits (bounded,
// ignoring an abort) for the last copy into every stage it used.
template <int D, typename Where>
__device__ __forceinline__ void bwd_stream(const BwdSmem<D>& sm, const CUtensorMap* tm_a,
                                           const CUtensorMap* tm_b, int n, const Ctl& ctl,
                                           Where where) {
  using C = BwdCfg<D>;
  const unsigned FULL = 0xffffffffu;
  int na = 0, nb = 0;  // copies issued per ring
  for (int t = 0; t < n; ++t) {
    int head, row;
    where(t, head, row);
    const int sa = ring_stage<C::kNA>(t), sb = ring_stage<C::kNB>(t);
    if (!__all_sync(FULL, wait_bar(sm.a_empty(sa), ring_parity<C::kNA>(t) ^ 1, ctl))) break;
    if (ptx::elect_one()) {
      ptx::mbar_arrive_expect_tx(sm.a_full(sa), C::kTile);
      bwd_load_tile<D>(sm.ring_a(sa), tm_a, sm.a_full(sa), head, row);
    }
    __syncwarp();
    ++na;
    if (!__all_sync(FULL, wait_bar(sm.b_empty(sb), ring_parity<C::kNB>(t) ^ 1, ctl))) break;
    if (ptx::elect_one()) {
      ptx::mbar_arrive_expect_tx(sm.b_full(sb), C::kTile);
      bwd_load_tile<D>(sm.ring_b(sb), tm_b, sm.b_full(sb), head, row);
    }
    __syncwarp();
    ++nb;
  }
  for (int st = 0; st < C::kNA && st < na; ++st)
    drain_bar(sm.a_full(st), ring_parity<C::kNA>(st + ((na - 1 - st) / C::kNA) * C::kNA));
  for (int st = 0; st < C::kNB && st < nb; ++st)
    drain_bar(sm.b_full(st), ring_parity<C::kNB>(st + ((nb - 1 - st) / C::kNB) * C::kNB));
}

// ------------------------------------------------------------------ dK, dV
template <int D, bool kBiasKey, bool kBiasPair>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dkdv_sm100(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const unsigned FULL = 0xffffffffu;
  const int kb = blockIdx.x, kvh = blockIdx.y, seq = blockIdx.z;
  const int q0 = p.cu_q[seq], k0 = p.cu_k[seq];
  const int Lq = p.cu_q[seq + 1] - q0, Lk = p.cu_k[seq + 1] - k0;
  if (*p.valid == 0 || kb * BN >= Lk) return;  // uniform over the CTA, before any barrier
  const int off = Lk - Lq;    // bottom-right causal offset
  int qb0 = 0;
  if (p.causal) {
    const int qmin = kb * BN - off;  // first query row that sees key kb*BN
    qb0 = qmin > 0 ? qmin / BM : 0;
  }
  const int nqb = ceil_div(Lq, BM);
  const int per_head = nqb > qb0 ? nqb - qb0 : 0;
  const int G = p.group;
  const int n_tiles = per_head * G;

  BwdSmem<D> sm;
  const uint32_t tmem = bwd_setup<D>(sm, smem_raw);
  const Ctl ctl{sm.abort_flag(), p.error, p.wait_limit};
  const int warp = threadIdx.x >> 5;

  if (warp == kBwdLoadWarp) {
    if (ptx::elect_one()) {
      ptx::mbar_arrive_expect_tx(sm.fixed_full(), 2 * BwdCfg<D>::kTile);
      bwd_load_tile<D>(sm.fixed(0), &tm_k, sm.fixed_full(), kvh, k0 + kb * BN);
      bwd_load_tile<D>(sm.fixed(1), &tm_v, sm.fixed_full(), kvh, k0 + kb * BN);
    }
    __syncwarp();
    bwd_stream<D>(sm, &tm_q, &tm_do, n_tiles, ctl, [&](int t, int& head, int& row) {
      head = kvh * G + t / per_head;
      row = q0 + (qb0 + t % per_head) * BM;
    });
    drain_bar(sm.fixed_full(), 0);
  } else if (warp == kBwdMmaWarp) {
    // Order per tile t: S^T(t), dP^T(t) | P(t) ready: dV(t), S^T(t+1) |
    // dS(t) ready: dK(t), dP^T(t+1). The compute warps turn S into P while
    // dP^T(t) runs and dP into dS while dV(t) and S^T(t+1) run. A product
    // that overwrites columns an earlier product reads is issued after it
    // (the tensor pipe runs in order).
    const uint64_t kd = desc_kmajor_sw128(ptx::smem_u32(sm.fixed(0)));
    const uint64_t vd = desc_kmajor_sw128(ptx::smem_u32(sm.fixed(1)));
    using C = BwdCfg<D>;
    // Test hook: o_full's phase 0 completes only through this warp's final
    // commit, so this wait can only run out (and abort the CTA).
    bool ok = !p.test_stall || __all_sync(FULL, wait_bar(sm.o_full(), 0, ctl));
    ok = ok && __all_sync(FULL, wait_bar(sm.fixed_full(), 0, ctl));
    auto a_addr = [&](int t) { return ptx::smem_u32(sm.ring_a(ring_stage<C::kNA>(t))); };
    auto b_addr = [&](int t) { return ptx::smem_u32(sm.ring_b(ring_stage<C::kNB>(t))); };
    auto issue_sT = [&](int t) {  // S^T(t) = K Q(t)^T
      ok = __all_sync(FULL, wait_bar(sm.a_full(ring_stage<C::kNA>(t)), ring_parity<C::kNA>(t), ctl));
      if (!ok) return;
      ptx::tc_fence_after();
      if (ptx::elect_one()) {
        issue_s<D>(tmem + 0, kd, desc_kmajor_sw128(a_addr(t)));
        ptx::tc_commit(sm.s_full());
      }
      __syncwarp();
    };
    auto issue_dpT = [&](int t) {  // dP^T(t) = V dO(t)^T
      ok = __all_sync(FULL, wait_bar(sm.b_full(ring_stage<C::kNB>(t)), ring_parity<C::kNB>(t), ctl));
      if (!ok) return;
      ptx::tc_fence_after();
      if (ptx::elect_one()) {
        issue_s<D>(tmem + 128, vd, desc_kmajor_sw128(b_addr(t)));
        ptx::tc_commit(sm.dp_full());
      }
      __syncwarp();
    };
    if (n_tiles > 0 && ok) {
      issue_sT(0);
      if (ok) issue_dpT(0);
    }
    for (int t = 0; t < n_tiles && ok; ++t) {
      ok = __all_sync(FULL, wait_bar(sm.p_full(), t & 1, ctl));
      if (!ok) break;
      ptx::tc_fence_after();
      if (ptx::elect_one()) {  // dV += P^T dO; then dO(t)'s stage is free
        const uint64_t dmn = desc_mnmajor_sw128(b_addr(t), BwdCfg<D>::kChunk);
        issue_ts_parts<D>(tmem + 256, tmem + 0, dmn, t > 0);
        ptx::tc_commit(sm.b_empty(ring_stage<C::kNB>(t)));
      }
      __syncwarp();
      if (t + 1 < n_tiles) {
        issue_sT(t + 1);
        if (!ok) break;
      }
      ok = __all_sync(FULL, wait_bar(sm.ds_full(), t & 1, ctl));
      if (!ok) break;
      ptx::tc_fence_after();
      if (ptx::elect_one()) {  // dK += dS^T Q; then Q(t)'s stage is free
        const uint64_t qmn = desc_mnmajor_sw128(a_addr(t), BwdCfg<D>::kChunk);
        issue_ts_parts<D>(tmem + 256 + D, tmem + 128, qmn, t > 0);
        ptx::tc_commit(sm.a_empty(ring_stage<C::kNA>(t)));
      }
      __syncwarp();
      if (t + 1 < n_tiles) issue_dpT(t + 1);
    }
    if (ptx::elect_one()) ptx::tc_commit(sm.o_full());
    __syncwarp();
    drain_bar(sm.o_full(), 0);
  } else {
    // compute warps: thread (c, part) owns key kb*BN + c (tensor-memory lane
    // c) and the query rows [32 part, 32 part + 32) of every tile
    const int lane = threadIdx.x & 31;
    const int c = (warp & 3) * 32 + lane, part = warp >> 2, r0 = part * 32;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + lane_base + r0, t_dp = tmem + lane_base + 128 + r0;
    const int kc = kb * BN + c;
    const bool key_ok = kc < Lk;
    float dbk = 0.f, bkey = 0.f;
    bool ok = true;
    for (int t = 0; t < n_tiles && ok; ++t) {
      const int g = t / per_head, qb = qb0 + t % per_head;
      const int h = kvh * G + g;
      if (t % per_head == 0) {
        dbk = 0.f;
        if constexpr (kBiasKey) bkey = key_ok ? p.bias_key[(long long)(k0 + kc) * p.n_heads + h] : 0.f;
      }
      // this tile's row constants: LSE * log2(e) and delta (written by part
      // 0, read by all)
      {
        const int b = t & 1;
        if (part == 0) {
          const int rl = qb * BM + c;
          const long long gi = (long long)h * p.total_q + q0 + rl;
          sm.rows(b, 0)[c] = rl < Lq ? p.lse[gi] * kLog2e : 0.f;
          sm.rows(b, 1)[c] = rl < Lq ? p.delta[gi] : 0.f;
        }
        // Buffer b is written again at tile t + 2, after every thread has
        // arrived for tile t + 1, i.e. finished reading it for tile t.
        ptx::mbar_arrive(sm.rows_full(b));
        ok = __all_sync(FULL, wait_bar(sm.rows_full(b), (t >> 1) & 1, ctl));
        if (!ok) break;
      }
      const float* lse2 = sm.rows(t & 1, 0);
      const float* dl = sm.rows(t & 1, 1);
      // every row of this thread's part sees the key (no per-element mask)
      const bool full = key_ok && qb * BM + r0 + 32 <= Lq && (!p.causal || kc <= qb * BM + r0 + off);
      const float* grow = nullptr;
      if constexpr (kBiasPair)
        grow = p.bias_pair + (long long)seq * p.sb + (long long)(h / p.bias_head_div) * p.sh +
               (long long)kc * p.sc;
      auto visible = [&](int r) {
        const int ql = qb * BM + r;
        return key_ok && ql < Lq && (!p.causal || kc <= ql + off);
      };
      // pass 1: S^T -> P^T, bf16 (to tensor memory for dV, over this part's
      // own S^T columns, and kept packed in registers for dS)
      ok = __all_sync(FULL, wait_bar(sm.s_full(), t & 1, ctl));
      if (!ok) break;
      ptx::tc_fence_after();
      uint32_t pk[16];
      auto pass1 = [&](auto masked) {
        uint32_t sv[32];
        ptx::tmem_ld32(t_s, sv);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float pv[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int r = r0 + e + u;
            float x = __uint_as_float(sv[e + u]) * p.scale;
            if constexpr (kBiasKey) x += bkey;
            const bool vis = decltype(masked)::value ? visible(r) : true;
            if constexpr (kBiasPair) {
              if (vis) x += __ldg(grow + (long long)(qb * BM + r) * p.sr);
            }
            pv[u] = vis ? ptx::ex2(fmaf(x, kLog2e, -lse2[r])) : 0.f;
          }
          pk[e / 2] = ptx::pack_bf16x2(pv[0], pv[1]);
        }
        // columns [r0, r0 + 16): this part's, already read
        ptx::tmem_st16(t_s, pk);
      };
      // (warp-uniform choice: the loop holds warp-collective tensor-memory
      // loads and stores)
      if (__all_sync(FULL, full)) pass1(std::false_type{});
      else pass1(std::true_type{});
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(sm.p_full());
      // pass 2: dP^T -> dS^T
      ok = __all_sync(FULL, wait_bar(sm.dp_full(), t & 1, ctl));
      if (!ok) break;
      ptx::tc_fence_after();
      float* dgrow = p.dbias_pair == nullptr
                         ? nullptr
                         : p.dbias_pair + (long long)seq * p.dsb + (long long)h * p.dsh + kc;
      auto pass2 = [&](auto store_grid) {
        uint32_t dp[32];
        ptx::tmem_ld32(t_dp, dp);
        ptx::tmem_wait_ld();
        uint32_t dk16[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const uint32_t w = pk[e / 2];
          const float pv[2] = {__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u)};
          float dsv[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int r = r0 + e + u;
            const float ds = pv[u] * (__uint_as_float(dp[e + u]) - dl[r]);
            dbk += ds;
            if constexpr (decltype(store_grid)::value) {
              const int ql = qb * BM + r;
              if (key_ok && ql < Lq) dgrow[(long long)ql * p.dsr] = ds;
            }
            dsv[u] = ds;
          }
          dk16[e / 2] = ptx::pack_bf16x2(dsv[0], dsv[1]);
        }
        ptx::tmem_st16(t_dp, dk16);
      };
      if (dgrow != nullptr) pass2(std::true_type{});
      else pass2(std::false_type{});
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(sm.ds_full());
      // the parts add into the zeroed output; the order of the adds is not
      // fixed, so the per-key bias gradient can differ in the last bits
      // between runs (dQ, dK, dV do not)
      if (p.dbias_key != nullptr && key_ok && t % per_head == per_head - 1)
        atomicAdd(p.dbias_key + (long long)(k0 + kc) * p.n_heads + h, dbk);
    }
    const bool have = n_tiles > 0;
    if (have) {
      ok = ok && __all_sync(FULL, wait_bar(sm.o_full(), 0, ctl));
      ptx::tc_fence_after();
    }
    if (ok) {
      // 2D/32 output chunks of 32 columns (dV's, then dK's) over the parts
      const long long o = ((long long)(k0 + kc) * p.n_kv_heads + kvh) * D;
      constexpr int kCh = D / 32;
      for (int q = part; q < 2 * kCh; q += kBwdParts) {
        const bool is_k = q >= kCh;
        const int ch = is_k ? q - kCh : q;
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(is_k ? p.dk : p.dv) + o;
        bwd_store_row<0, 1>(tmem + lane_base + 256 + (is_k ? D : 0) + ch * 32, have,
                            is_k ? p.scale : 1.f, dst + ch * 32, key_ok);
      }
    }
  }
  bwd_teardown<D>(sm, tmem);
}

// ------------------------------------------------------------------ dQ
template <int D, bool kBiasKey, bool kBiasPair>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dq_sm100(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const unsigned FULL = 0xffffffffu;
  // Causal rows see more keys the later they are: the last query blocks go
  // first, so that the longest CTAs do not form the tail of the launch.
  const int qb = gridDim.x - 1 - blockIdx.x, h = blockIdx.y, seq = blockIdx.z;
  const int q0 = p.cu_q[seq], k0 = p.cu_k[seq];
  const int Lq = p.cu_q[seq + 1] - q0, Lk = p.cu_k[seq + 1] - k0;
  if (*p.valid == 0 || qb * BM >= Lq) return;  // uniform over the CTA, before any barrier
  const int off = Lk - Lq;
  const int rows = min(BM, Lq - qb * BM);
  const int n_k = slot_tiles(qb * BM, rows, Lq, Lk, p.causal);
  const int kvh = h / p.group;

  BwdSmem<D> sm;
  const uint32_t tmem = bwd_setup<D>(sm, smem_raw);
  const Ctl ctl{sm.abort_flag(), p.error, p.wait_limit};
  const int warp = threadIdx.x >> 5;

  if (warp == kBwdLoadWarp) {
    if (n_k > 0 && ptx::elect_one()) {
      ptx::mbar_arrive_expect_tx(sm.fixed_full(), 2 * BwdCfg<D>::kTile);
      bwd_load_tile<D>(sm.fixed(0), &tm_q, sm.fixed_full(), h, q0 + qb * BM);
      bwd_load_tile<D>(sm.fixed(1), &tm_do, sm.fixed_full(), h, q0 + qb * BM);
    }
    __syncwarp();
    bwd_stream<D>(sm, &tm_k, &tm_v, n_k, ctl, [&](int j, int& head, int& row) {
      head = kvh;
      row = k0 + j * BN;
    });
    if (n_k > 0) drain_bar(sm.fixed_full(), 0);
  } else if (warp == kBwdMmaWarp) {
    // Order per key tile j: S(j), dP(j) | S(j) read: S(j+1) | dS(j) ready:
    // dP(j+1), dQ(j). The compute warps turn S into P while dP(j) runs and
    // dP into dS while S(j+1) runs. dS(j) goes to tensor-memory columns
    // [384 + 64(j % 2), +64) (free in this kernel), so dP(j+1) need not wait
    // for dQ(j) to have read it; dS(j+2) is written after dp_full(j+2),
    // which dQ(j) precedes.
    const uint64_t qd = desc_kmajor_sw128(ptx::smem_u32(sm.fixed(0)));
    const uint64_t dod = desc_kmajor_sw128(ptx::smem_u32(sm.fixed(1)));
    using C = BwdCfg<D>;
    // Test hook: o_full's phase 0 completes only through this warp's final
    // commit, so this wait can only run out (and abort the CTA).
    bool ok = !p.test_stall || __all_sync(FULL, wait_bar(sm.o_full(), 0, ctl));
    ok = ok && (n_k == 0 || __all_sync(FULL, wait_bar(sm.fixed_full(), 0, ctl)));
    auto a_addr = [&](int j) { return ptx::smem_u32(sm.ring_a(ring_stage<C::kNA>(j))); };
    auto b_addr = [&](int j) { return ptx::smem_u32(sm.ring_b(ring_stage<C::kNB>(j))); };
    auto issue_s_j = [&](int j) {  // S(j) = Q K(j)^T
      ok = __all_sync(FULL, wait_bar(sm.a_full(ring_stage<C::kNA>(j)), ring_parity<C::kNA>(j), ctl));
      if (!ok) return;
      ptx::tc_fence_after();
      if (ptx::elect_one()) {
        issue_s<D>(tmem + 0, qd, desc_kmajor_sw128(a_addr(j)));
        ptx::tc_commit(sm.s_full());
      }
      __syncwarp();
    };
    auto issue_dp_j = [&](int j) {  // dP(j) = dO V(j)^T; then V(j)'s stage is free
      ok = __all_sync(FULL, wait_bar(sm.b_full(ring_stage<C::kNB>(j)), ring_parity<C::kNB>(j), ctl));
      if (!ok) return;
      ptx::tc_fence_after();
      if (ptx::elect_one()) {
        issue_s<D>(tmem + 128, dod, desc_kmajor_sw128(b_addr(j)));
        ptx::tc_commit(sm.dp_full());
        ptx::tc_commit(sm.b_empty(ring_stage<C::kNB>(j)));
      }
      __syncwarp();
    };
    if (n_k > 0 && ok) {
      issue_s_j(0);
      if (ok) issue_dp_j(0);
    }
    for (int j = 0; j < n_k && ok; ++j) {
      ok = __all_sync(FULL, wait_bar(sm.p_full(), j & 1, ctl));  // S(j) has been read
      if (!ok) break;
      if (j + 1 < n_k) {
        issue_s_j(j + 1);
        if (!ok) break;
      }
      ok = __all_sync(FULL, wait_bar(sm.ds_full(), j & 1, ctl));
      if (!ok) break;
      ptx::tc_fence_after();
      if (j + 1 < n_k) {
        issue_dp_j(j + 1);
        if (!ok) break;
      }
      if (ptx::elect_one()) {  // dQ += dS K; then K(j)'s stage is free
        const uint64_t kmn = desc_mnmajor_sw128(a_addr(j), BwdCfg<D>::kChunk);
        const uint32_t ds_col = tmem + 384 + 64 * (j & 1);
        issue_pv_half<D>(tmem + 256, ds_col, kmn, 0, j > 0);
        issue_pv_half<D>(tmem + 256, ds_col, kmn, 1, true);
        ptx::tc_commit(sm.a_empty(ring_stage<C::kNA>(j)));
      }
      __syncwarp();
    }
    if (ptx::elect_one()) ptx::tc_commit(sm.o_full());
    __syncwarp();
    drain_bar(sm.o_full(), 0);
  } else {
    // compute warps: thread (r, part) owns query row qb*BM + r and the keys
    // [32 part, 32 part + 32) of every tile
    const int lane = threadIdx.x & 31;
    const int r = (warp & 3) * 32 + lane, part = warp >> 2, c0 = part * 32;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + lane_base + c0, t_dp = tmem + lane_base + 128 + c0;
    const int ql = qb * BM + r;
    const bool row_ok = ql < Lq;
    const long long gi = (long long)h * p.total_q + q0 + ql;
    const float lse2 = row_ok ? p.lse[gi] * kLog2e : 0.f;
    const float dl = row_ok ? p.delta[gi] : 0.f;
    const float* grow = nullptr;
    if constexpr (kBiasPair)
      grow = p.bias_pair + (long long)seq * p.sb + (long long)(h / p.bias_head_div) * p.sh +
             (long long)ql * p.sr;
    bool ok = true;
    for (int j = 0; j < n_k && ok; ++j) {
      const int kt = j * BN + c0;  // this part's first key
      // every key of this part is visible to the row (no per-element mask)
      const bool full = row_ok && kt + 32 <= Lk && (!p.causal || kt + 31 <= ql + off);
      ok = __all_sync(FULL, wait_bar(sm.s_full(), j & 1, ctl));
      if (!ok) break;
      ptx::tc_fence_after();
      float pr[32];
      auto pass1 = [&](auto masked) {
        uint32_t sv[32];
        ptx::tmem_ld32(t_s, sv);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int kc = kt + e;
          const bool vis = decltype(masked)::value
                               ? row_ok && kc < Lk && (!p.causal || kc <= ql + off)
                               : true;
          float x = __uint_as_float(sv[e]) * p.scale;
          if constexpr (kBiasKey) {
            if (vis) x += __ldg(p.bias_key + (long long)(k0 + kc) * p.n_heads + h);
          }
          if constexpr (kBiasPair) {
            if (vis) x += __ldg(grow + (long long)kc * p.sc);
          }
          pr[e] = vis ? ptx::ex2(fmaf(x, kLog2e, -lse2)) : 0.f;
        }
      };
      // (warp-uniform choice: the loop holds warp-collective loads)
      if (__all_sync(FULL, full)) pass1(std::false_type{});
      else pass1(std::true_type{});
      ptx::tc_fence_before();
      ptx::mbar_arrive(sm.p_full());  // S(j) read: the next S may overwrite it
      ok = __all_sync(FULL, wait_bar(sm.dp_full(), j & 1, ctl));
      if (!ok) break;
      ptx::tc_fence_after();
      {
        uint32_t dp[32];
        ptx::tmem_ld32(t_dp, dp);
        ptx::tmem_wait_ld();
        uint32_t dk16[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2)
          dk16[e / 2] = ptx::pack_bf16x2(pr[e] * (__uint_as_float(dp[e]) - dl),
                                         pr[e + 1] * (__uint_as_float(dp[e + 1]) - dl));
        // dS(j) buffer j % 2: this part's 32 keys in columns [16 part, +16)
        ptx::tmem_st16(tmem + lane_base + 384 + 64 * (j & 1) + 16 * part, dk16);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(sm.ds_full());
    }
    const bool have = n_k > 0;
    if (have) {
      ok = ok && __all_sync(FULL, wait_bar(sm.o_full(), 0, ctl));
      ptx::tc_fence_after();
    }
    if (ok) {  // D/32 output chunks of 32 columns over the parts
      __nv_bfloat16* dst =
          reinterpret_cast<__nv_bfloat16*>(p.dq) + ((long long)(q0 + ql) * p.n_heads + h) * D;
      for (int ch = part; ch < D / 32; ch += kBwdParts)
        bwd_store_row<0, 1>(tmem + lane_base + 256 + ch * 32, have, p.scale, dst + ch * 32, row_ok);
    }
  }
  bwd_teardown<D>(sm, tmem);
}

}  // namespace va
