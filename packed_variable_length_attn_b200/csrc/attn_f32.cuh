// Packed variable-length attention forward with fp32 inputs and fp32
// arithmetic on the CUDA cores (no tensor cores: TF32 would round q, k and v
// to 10 mantissa bits, too coarse for fp32 parity).
//
// One CTA per (sequence, 64-row q-block, head): grid.x = batch * qblocks_max,
// grid.y = n_heads; CTAs past a sequence's last q-block exit at once. 256
// threads: thread (row = tid / 4, quad = tid % 4) scores keys quad + 4t of
// each 64-key tile and accumulates output dims quad + 4t of its row, with an
// exact-exponent online softmax.
#pragma once
#include "common.cuh"

namespace va {

constexpr int kF32Rows = 64;
constexpr int kF32Keys = 64;
constexpr int kF32Threads = 256;

struct F32Params {
  const float* q;
  const float* k;
  const float* v;
  const int* cu_q;
  const int* cu_k;
  int qblocks_max;
  int total_q;
  int n_heads, group;
  float scale;
  int causal;
  const float* bias_key;
  const float* bias_pair;
  long long sb, sh, sr, sc;
  int bias_head_div;  // grid head index = head / bias_head_div
  float* out;
  float* lse;
  const int* valid;  // work count written by the validation pass (0 = invalid input)
};

template <int D>
struct F32Cfg {
  static constexpr int kQStride = D + 4;
  static constexpr int kKStride = D + 1;
  static constexpr int kPStride = kF32Keys + 1;
  static constexpr int kSmemFloats =
      kF32Rows * kQStride + kF32Keys * kKStride + kF32Keys * D + kF32Rows * kPStride;
  static constexpr int kSmemBytes = kSmemFloats * 4;
};

template <int D>
__global__ void __launch_bounds__(kF32Threads) attn_fwd_f32(const F32Params p) {
  using C = F32Cfg<D>;
  if (*p.valid == 0) return;
  const int i = blockIdx.x / p.qblocks_max;
  const int qb = blockIdx.x % p.qblocks_max;
  const int h = blockIdx.y;
  const int q0 = p.cu_q[i], Lq = p.cu_q[i + 1] - q0;
  if (qb * kF32Rows >= Lq) return;
  const int k0 = p.cu_k[i], Lk = p.cu_k[i + 1] - k0;
  const int kvh = h / p.group;
  const int Hkv = p.n_heads / p.group;

  extern __shared__ float fsm[];
  float* Qs = fsm;
  float* Ks = Qs + kF32Rows * C::kQStride;
  float* Vs = Ks + kF32Keys * C::kKStride;
  float* Ps = Vs + kF32Keys * D;

  const int tid = threadIdx.x;
  const int row = tid >> 2, quad = tid & 3;
  const int q_loc = qb * kF32Rows + row;
  const bool row_ok = q_loc < Lq;

  for (int e = tid; e < kF32Rows * D; e += kF32Threads) {
    const int rr = e / D, d = e % D;
    const int ql = qb * kF32Rows + rr;
    Qs[rr * C::kQStride + d] = ql < Lq ? p.q[((long long)(q0 + ql) * p.n_heads + h) * D + d] : 0.f;
  }

  const int limit = p.causal ? min(Lk, q_loc + (Lk - Lq) + 1) : Lk;
  const int last_row = min(qb * kF32Rows + kF32Rows, Lq) - 1;
  int key_end = p.causal ? min(Lk, last_row + (Lk - Lq) + 1) : Lk;
  key_end = max(key_end, 0);
  const int ntiles = (key_end + kF32Keys - 1) / kF32Keys;

  constexpr float kLog2e = 1.4426950408889634f;
  float m = -INFINITY, l = 0.f;
  float acc[D / 4];
#pragma unroll
  for (int t = 0; t < D / 4; ++t) acc[t] = 0.f;
  const float* brow = nullptr;
  if (p.bias_pair != nullptr && row_ok)
    brow = p.bias_pair + (long long)i * p.sb + (long long)(h / p.bias_head_div) * p.sh +
           (long long)q_loc * p.sr;

  for (int kt = 0; kt < ntiles; ++kt) {
    const int kb = kt * kF32Keys;
    __syncthreads();
    for (int e = tid; e < kF32Keys * D; e += kF32Threads) {
      const int c = e / D, d = e % D;
      const bool in = kb + c < Lk;
      const long long off = ((long long)(k0 + kb + c) * Hkv + kvh) * D + d;
      Ks[c * C::kKStride + d] = in ? p.k[off] : 0.f;
      Vs[c * D + d] = in ? p.v[off] : 0.f;
    }
    __syncthreads();
    float s[kF32Keys / 4];
    float tmax = -INFINITY;
#pragma unroll
    for (int t = 0; t < kF32Keys / 4; ++t) {
      const int c = quad + 4 * t;
      float dot = 0.f;
#pragma unroll 8
      for (int d = 0; d < D; ++d) dot = fmaf(Qs[row * C::kQStride + d], Ks[c * C::kKStride + d], dot);
      float x = dot * p.scale;
      const int key = kb + c;
      if (key < Lk) {
        if (p.bias_key != nullptr) x += p.bias_key[(long long)(k0 + key) * p.n_heads + h];
        if (brow != nullptr) x += brow[(long long)key * p.sc];
      }
      x = key < limit ? x * kLog2e : -INFINITY;
      s[t] = x;
      tmax = fmaxf(tmax, x);
    }
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    const float m_new = fmaxf(m, tmax);
    const float base = m_new == -INFINITY ? 0.f : m_new;
    const float alpha = exp2f(m - base);  // 0 while m is -inf
    float rs = 0.f;
#pragma unroll
    for (int t = 0; t < kF32Keys / 4; ++t) {
      const float pv = exp2f(s[t] - base);
      rs += pv;
      Ps[row * C::kPStride + quad + 4 * t] = pv;
    }
    rs += __shfl_xor_sync(0xffffffffu, rs, 1);
    rs += __shfl_xor_sync(0xffffffffu, rs, 2);
    l = l * alpha + rs;
    m = m_new;
#pragma unroll
    for (int t = 0; t < D / 4; ++t) acc[t] *= alpha;
    __syncwarp();
    for (int c = 0; c < kF32Keys; ++c) {
      const float pv = Ps[row * C::kPStride + c];
#pragma unroll
      for (int t = 0; t < D / 4; ++t) acc[t] = fmaf(pv, Vs[c * D + quad + 4 * t], acc[t]);
    }
    __syncwarp();
  }

  if (!row_ok) return;
  const float inv = l > 0.f ? 1.f / l : 0.f;
  float* orow = p.out + ((long long)(q0 + q_loc) * p.n_heads + h) * D;
#pragma unroll
  for (int t = 0; t < D / 4; ++t) orow[quad + 4 * t] = acc[t] * inv;
  if (quad == 0 && p.lse != nullptr)
    p.lse[(long long)h * p.total_q + q0 + q_loc] =
        l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
}

}  // namespace va
