// Packed variable-length attention forward for sm_100a (B200).
//
// Persistent, warp-specialised kernel; one CTA per SM, 12 warps in three
// warpgroups:
//   warps 0-3   softmax group 0: rows of slot 0 (thread = row = TMEM lane)
//   warps 4-7   softmax group 1: rows of slot 1
//   warp  8     MMA issue (one elected lane) + tensor-memory allocation
//   warp  9     work fetch + TMA loads (one elected lane)
//   warps 10-11 idle
// The CTA launches with kLaunchRegs registers per thread; the third
// warpgroup then gives registers up (setmaxnreg.dec to kWorkerRegs) and the
// two softmax groups take them (setmaxnreg.inc to kSoftmaxRegs). The split
// adds up exactly to the launch total, which the host checks against the
// compiled kernel's register count before every first launch.
//
// A work item holds up to two 128-row query tiles ("slots") that stream the
// same 128-key K/V tiles: two heads of one GQA group at one q-block, or two
// q-blocks of one head. Per K/V tile j the tensor core computes
// S_s = Q_s K_j^T into tensor memory (fp32), the softmax group turns S_s into
// P_s (bf16, written back over S_s), and the tensor core accumulates
// O_s += P_s V_j with P read straight from tensor memory.
//
// A cache-mode instantiation (kCache) serves decode steps: K/V tiles are
// read in place from a per-sequence cache (rows i * cache_len ..), and one
// slot holds the rows of all G query heads of a K/V group, token-major.
//
// Tensor memory (512 columns): S0/P0 [0,128), S1/P1 [128,256),
// O0 [256, 256+D), O1 [256+D, 256+2D). The softmax publishes P in two halves
// (keys 0-63, then 64-127), so the first half of P V runs on the tensor core
// while the second half's exponentials are computed. MMA issue order:
// S0(0) S1(0) | PV0a(j) PV0b(j) S0(j+1) PV1a(j) PV1b(j) S1(j+1) | ... : one
// slot's softmax overlaps the other slot's MMAs.
//
// Shared memory: Q0, Q1 (128 rows x D bf16, 64-column 128-byte-swizzled
// chunks as TMA writes them), the K/V ring (128-row tiles, same layout),
// per-key bias staging, O staging for coalesced output stores, the
// work-item ring, mbarriers.
//
// Every mbarrier wait is bounded; on expiry the kernel records
// kErrTimeout in the device error word, all roles leave their loops, the
// loader waits (bounded) for its copies in flight, the MMA warp drains its
// tensor-core work and frees tensor memory, and the CTA exits.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include "common.cuh"
#include "ptx.cuh"

namespace va {

constexpr int kAttnThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 200;
constexpr int kWorkerRegs = 104;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kWorkerRegs == kAttnThreads * kLaunchRegs,
              "register split must add up to the launch allocation");
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// A row's running max is only moved (and O rescaled) when the tile max
// exceeds it by more than this many powers of two; P stays <= 2^8.
constexpr float kRescaleThreshold = 8.0f;
// Default limit of a bounded wait (the launch parameter wait_limit; a caller
// may shorten it to exercise the abort path) and the fixed limit of the
// drains that follow an abort.
constexpr long long kWaitLimitCycles = 1ll << 33;    // ~4 s at 2 GHz
constexpr long long kDrainLimitCycles = 1ll << 29;   // ~0.3 s

template <int D>
struct KCfg {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static constexpr int kChunks = D / 64;                  // 64-column (128 B) chunks
  static constexpr int kQChunk = BM * 128;                // 128 rows x 128 B
  static constexpr int kKVChunk = BN * 128;               // 128 rows x 128 B
  static constexpr int kQTile = kChunks * kQChunk;
  static constexpr int kKVTile = kChunks * kKVChunk;
  static constexpr int kStages = D == 64 ? 8 : 4;         // K/V ring depth (tiles)
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kQTile;
  static constexpr int kBiasOff = kKVOff + kStages * kKVTile;  // float [2 slot][2 buf][BN]
  static constexpr int kEpiOff = kBiasOff + 2 * 2 * BN * 4;     // O staging: 2 KB per softmax warp
  static constexpr int kEpiWarpBytes = 32 * 32 * 2;             // 32 rows x 32 bf16 columns
  // Pair-grid staging ring per softmax warp: the O staging block plus
  // kPairBufs - 1 more blocks of the same size (head_dim 64 has the room).
  static constexpr int kPairBufs = D == 64 ? 3 : 1;
  static constexpr int kPairOff = kEpiOff + 8 * kEpiWarpBytes;
  static constexpr int kItemOff = kPairOff + 8 * (kPairBufs - 1) * kEpiWarpBytes;
  static constexpr int kBarOff = kItemOff + ((2 * (int)sizeof(Item) + 15) / 16) * 16;
  // barriers: q_full[2] q_empty[2] s_full[2] p_full[2][2 halves] o_full[2]
  //           o_empty[2] item_full[2] item_empty[2] bias_full[2][2] drain
  //           kv_full[S] kv_empty[S]
  static constexpr int kNumBars = 23 + 2 * kStages;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem slot, abort flag
  static constexpr int kSmemBytes = kMiscOff + 16 + 1024;  // + alignment slack
};

struct Ctl {
  volatile int* abort;
  int* error;
  long long limit;  // cycles a wait may take before it raises kErrTimeout
};

__device__ __forceinline__ void raise_abort(const Ctl& c) {
  *c.abort = 1;
  atomicCAS(c.error, 0, kErrTimeout);
}

// Bounded wait for the phase of `bar` with the given parity.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const Ctl& c) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*c.abort) return false;
    if (clock64() - t0 > c.limit) {
      raise_abort(c);
      return false;
    }
  }
}

// Bounded wait that ignores the abort flag (used to drain copies in flight).
__device__ __forceinline__ void drain_bar(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kDrainLimitCycles) return;
  }
}

// UMMA shared-memory descriptors (sm_100 format, version 1).
// K-major, 128-byte swizzle: rows 128 B apart, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;                 // leading byte offset (unused for this layout)
  d |= (uint64_t)(1024 >> 4) << 32;       // stride byte offset: next 8-row group
  d |= (uint64_t)1 << 46;                 // descriptor version
  d |= (uint64_t)2 << 61;                 // 128-byte swizzle
  return d;
}
// MN-major, 128-byte swizzle: 64 MN-elements contiguous per 128-B row, K rows
// 128 B apart, 8-row K groups 1024 B apart, 64-element MN chunks `lbo` apart.
__device__ __forceinline__ uint64_t desc_mnmajor_sw128(uint32_t saddr, uint32_t lbo) {
  uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;  // leading byte offset: next 64-wide MN chunk
  d |= (uint64_t)(1024 >> 4) << 32;             // stride byte offset: next 8-row K group
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(int n, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// Tensor-memory columns.
__device__ __forceinline__ uint32_t s_col(int s) { return (uint32_t)(s * 128); }
template <int D>
__device__ __forceinline__ uint32_t o_col(int s) { return (uint32_t)(256 + s * D); }

template <int D>
struct Smem {
  uint8_t* base;
  __device__ uint8_t* q(int s) const { return base + KCfg<D>::kQOff + s * KCfg<D>::kQTile; }
  __device__ uint8_t* kv(int st) const { return base + KCfg<D>::kKVOff + st * KCfg<D>::kKVTile; }
  __device__ float* bias(int s, int b) const {
    return reinterpret_cast<float*>(base + KCfg<D>::kBiasOff) + (s * 2 + b) * BN;
  }
  __device__ uint8_t* epi(int warp) const { return base + KCfg<D>::kEpiOff + warp * KCfg<D>::kEpiWarpBytes; }
  // pair-grid staging block b of a softmax warp (block 0 is its O staging)
  __device__ uint8_t* pair_buf(int warp, int b) const {
    return b == 0 ? epi(warp)
                  : base + KCfg<D>::kPairOff + (warp * (KCfg<D>::kPairBufs - 1) + b - 1) * KCfg<D>::kEpiWarpBytes;
  }
  __device__ Item* items() const { return reinterpret_cast<Item*>(base + KCfg<D>::kItemOff); }
  __device__ uint64_t* bars() const { return reinterpret_cast<uint64_t*>(base + KCfg<D>::kBarOff); }
  __device__ uint64_t* q_full(int s) const { return bars() + 0 + s; }
  __device__ uint64_t* q_empty(int s) const { return bars() + 2 + s; }
  __device__ uint64_t* s_full(int s) const { return bars() + 4 + s; }
  __device__ uint64_t* p_full(int s, int h) const { return bars() + 6 + 2 * s + h; }
  __device__ uint64_t* o_full(int s) const { return bars() + 10 + s; }
  __device__ uint64_t* o_empty(int s) const { return bars() + 12 + s; }
  __device__ uint64_t* item_full(int k) const { return bars() + 14 + k; }
  __device__ uint64_t* item_empty(int k) const { return bars() + 16 + k; }
  __device__ uint64_t* bias_full(int s, int b) const { return bars() + 18 + 2 * s + b; }
  __device__ uint64_t* drain() const { return bars() + 22; }
  __device__ uint64_t* kv_full(int st) const { return bars() + 23 + st; }
  __device__ uint64_t* kv_empty(int st) const { return bars() + 23 + KCfg<D>::kStages + st; }
  __device__ uint32_t* tmem_slot() const { return reinterpret_cast<uint32_t*>(base + KCfg<D>::kMiscOff); }
  __device__ int* abort_flag() const { return reinterpret_cast<int*>(base + KCfg<D>::kMiscOff + 4); }
};

template <bool kCache>
__device__ __forceinline__ Item decode_item(int w, const AttnParams& p) {
  Item it;
  const int2 pr = p.ws.list[w / p.n_hg];
  const int hg = w % p.n_hg;
  // with key ranges a list entry is sequence * ranges + range
  const int ranges = kCache && p.cache_ranges > 1 ? p.cache_ranges : 1;
  const int i = pr.x / ranges, rg = pr.x - i * ranges, g = pr.y;
  it.valid = 1;
  it.seq = pr.x;
  const int q0 = p.cu_q[i];
  it.Lq = p.cu_q[i + 1] - q0;
  int k0, koff = 0;
  if constexpr (kCache) {  // K/V in place in the cache, packed-GQA rows
    const int lk = p.cache_seqlens[i] + (p.cache_extra ? it.Lq : 0);
    const int ks = rg * p.range_keys;  // first key of the range
    k0 = i * p.cache_len + ks;
    it.Lk = ranges > 1 ? max(0, min(lk - ks, p.range_keys)) : lk;
    koff = lk - ks - it.Lk;  // keys of the sequence after the range
    it.kvh = hg;
  } else {
    k0 = p.cu_k[i];
    it.Lk = p.cu_k[i + 1] - k0;
    it.kvh = p.pairing == kPairHeads ? hg : hg / p.group;
  }
  it.kv_row0 = k0;
  fill_slots(it, g, hg, p.pairing, p.group, p.causal);
  if (kCache && koff > 0) {
    // A range with keys after it: query token t sees range key c when
    // c <= t + (Lk + koff - Lq), so the causal mask (and the tiles visited)
    // take Lq - koff in place of Lq.
    it.Lq -= koff;
    it.ntile[0] = slot_tiles(it.q_loc0[0], it.rows[0] / p.group, it.Lq, it.Lk, p.causal);
  }
  it.q_row0[0] = q0 + it.q_loc0[0];
  it.q_row0[1] = q0 + it.q_loc0[1];
  return it;
}

// ------------------------------------------------------------------ loader
// Runs on all 32 lanes of the load warp (uniform control flow); one elected
// lane fetches work and issues the copies. Per item: Q of each active slot,
// then K0, V0, K1, V1, ... (the MMA warp's consumption order).
template <int D, bool kCache>
__device__ void load_role(const Smem<D>& sm, const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                          const CUtensorMap* tm_v, const AttnParams& p, const Ctl& ctl) {
  using C = KCfg<D>;
  const unsigned FULL = 0xffffffffu;
  uint32_t kv_t = 0, q_uses[2] = {0, 0};
  // the work list is written by the schedule kernel launched just before
  // (this kernel may start before it ends: programmatic dependent launch)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int count = *reinterpret_cast<volatile int*>(p.ws.count);
  bool ok = true;
  auto load_kv = [&](const CUtensorMap* tm, int kvh, int row) {
    const int st = kv_t % C::kStages;
    if (!__all_sync(FULL, wait_bar(sm.kv_empty(st), ((kv_t / C::kStages) & 1) ^ 1, ctl))) {
      ok = false;
      return;
    }
    ++kv_t;
    if (ptx::elect_one()) {
      ptx::mbar_arrive_expect_tx(sm.kv_full(st), C::kKVTile);
      for (int c = 0; c < C::kChunks; ++c)
        ptx::tma_load_3d(sm.kv(st) + c * C::kKVChunk, tm, sm.kv_full(st), c * 64, kvh, row);
    }
    __syncwarp();
  };
  for (int it = 0; ok; ++it) {
    const int k = it & 1;
    if (!__all_sync(FULL, wait_bar(sm.item_empty(k), ((it >> 1) & 1) ^ 1, ctl))) break;
    if (ptx::elect_one()) {
      const int w = atomicAdd(p.ws.counter, 1);
      Item item;
      if (w < count) {
        item = decode_item<kCache>(w, p);
      } else {
        item.valid = 0;
      }
      sm.items()[k] = item;
      ptx::mbar_arrive(sm.item_full(k));
    }
    __syncwarp();
    const Item item = sm.items()[k];
    if (!item.valid) break;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (ok && item.ntile[s] > 0) {
        ok = __all_sync(FULL, wait_bar(sm.q_empty(s), (q_uses[s] & 1) ^ 1, ctl));
        ++q_uses[s];
        if (ok && ptx::elect_one()) {
          // (a packed-GQA box may write fewer than 128 rows)
          ptx::mbar_arrive_expect_tx(sm.q_full(s), kCache ? C::kChunks * p.q_box_rows * 128 : C::kQTile);
          for (int c = 0; c < C::kChunks; ++c)
            ptx::tma_load_3d(sm.q(s) + c * C::kQChunk, tm_q, sm.q_full(s), c * 64, item.head[s],
                             item.q_row0[s]);
        }
        __syncwarp();
      }
    }
    const int n = max(item.ntile[0], item.ntile[1]);
    for (int j = 0; j < n && ok; ++j) {
      load_kv(tm_k, item.kvh, item.kv_row0 + j * BN);
      if (ok) load_kv(tm_v, item.kvh, item.kv_row0 + j * BN);
    }
  }
  // Wait for every copy this warp started (immediate on the normal path).
  for (int st = 0; st < C::kStages; ++st) {
    if (kv_t > (uint32_t)st) {
      const uint32_t uses = (kv_t - 1 - st) / C::kStages + 1;
      drain_bar(sm.kv_full(st), (uses - 1) & 1);
    }
  }
#pragma unroll
  for (int s = 0; s < 2; ++s)
    if (q_uses[s] > 0) drain_bar(sm.q_full(s), (q_uses[s] - 1) & 1);
}

// ------------------------------------------------------------------ MMA issue
// The MMA warp issues 32 tensor-core instructions per pair of slot tiles, so
// their operands are prepared once: a descriptor's start-address field holds
// the shared-memory byte address / 16 (14 bits, and every address of the CTA
// is below 2^18), so a descriptor of base + off is the base's descriptor +
// off / 16. The loops below add compile-time offsets only.
struct MmaDescs {
  uint64_t q[2];   // Q of slot s, chunk 0, K-major
  uint64_t k0;     // K ring stage 0, chunk 0, K-major
  uint64_t v0;     // V ring stage 0, MN-major
};

template <int D>
__device__ __forceinline__ uint64_t stage_desc(uint64_t d0, int st) {
  return d0 + (uint64_t)(st * (KCfg<D>::kKVTile >> 4));
}

// S_s = Q_s K^T: M = 128, N = 128 keys, K = D in steps of 16.
template <int D>
__device__ __forceinline__ void issue_s(uint32_t d_tmem, uint64_t qd, uint64_t kd) {
  using C = KCfg<D>;
  static_assert(C::kQChunk == C::kKVChunk, "Q and K chunks share the offsets");
  constexpr uint32_t idesc = idesc_bf16(BN, false);
#pragma unroll
  for (int k16 = 0; k16 < D / 16; ++k16) {
    const uint64_t off = (uint64_t)((((k16 >> 2) * C::kQChunk) + (k16 & 3) * 32) >> 4);
    ptx::mma_ss(d_tmem, qd + off, kd + off, idesc, k16 > 0 ? 1u : 0u);
  }
}

// O_s += P_s[keys 64h .. 64h+63] V[same keys]: M = 128, N = D, K = 64 in
// steps of 16; P from tensor memory (2 keys per 32-bit column).
template <int D>
__device__ __forceinline__ void issue_pv_half(uint32_t o_tmem, uint32_t p_tmem, uint64_t vd, int h,
                                              bool acc) {
  constexpr uint32_t idesc = idesc_bf16(D, true);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int k16 = 4 * h + k;
    ptx::mma_ts(o_tmem, p_tmem + k16 * 8, vd + (uint64_t)((k16 * 16 * 128) >> 4), idesc,
                (acc || k16 > 0) ? 1u : 0u);
  }
}

// Runs on all 32 lanes of the MMA warp (uniform control flow); one elected
// lane issues the tensor-core instructions and their commits. The slot loops
// are unrolled so that every per-slot counter stays in a register.
// kCache (K/V cache mode): the rows of a sequence's last V tile past its
// length are zeroed in shared memory before P V reads the tile. Their
// probabilities are exactly 0, but the cache may hold anything there
// (unwritten slots, NaN), and 0 * NaN would reach the output.
template <int D, bool kCache>
__device__ void mma_role(const Smem<D>& sm, uint32_t tmem, const Ctl& ctl, int test_stall) {
  using C = KCfg<D>;
  const unsigned FULL = 0xffffffffu;
  uint32_t kv_t = 0, q_uses[2] = {0, 0}, o_uses[2] = {0, 0};
  uint32_t tc[2] = {0, 0};  // tiles issued per slot (phase of the P barriers)
  MmaDescs dsc;
  dsc.q[0] = desc_kmajor_sw128(ptx::smem_u32(sm.q(0)));
  dsc.q[1] = desc_kmajor_sw128(ptx::smem_u32(sm.q(1)));
  dsc.k0 = desc_kmajor_sw128(ptx::smem_u32(sm.kv(0)));
  dsc.v0 = desc_mnmajor_sw128(ptx::smem_u32(sm.kv(0)), C::kKVChunk);
  auto wait = [&](uint64_t* bar, uint32_t parity) {
    return __all_sync(FULL, wait_bar(bar, parity, ctl));
  };
  auto next_kv = [&](int& st) {
    st = kv_t % C::kStages;
    const bool r = wait(sm.kv_full(st), (kv_t / C::kStages) & 1);
    ++kv_t;
    return r;
  };
  // Test hook: drain's phase 0 completes only through this warp's final
  // commit, so this wait can only run out (and abort the CTA).
  bool ok = !test_stall || wait(sm.drain(), 0);
  for (int it = 0; ok; ++it) {
    const int k = it & 1;
    if (!wait(sm.item_full(k), (it >> 1) & 1)) break;
    const Item& itm = sm.items()[k];
    const int valid = itm.valid;
    const int nt[2] = {itm.ntile[0], itm.ntile[1]};
    const int item_lk = itm.Lk;
    __syncwarp();
    if (ptx::elect_one()) ptx::mbar_arrive(sm.item_empty(k));
    if (!valid) break;
    const int n = max(nt[0], nt[1]);
    if (n == 0) continue;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (ok && nt[s] > 0) {
        ok = wait(sm.q_full(s), q_uses[s] & 1);
        ++q_uses[s];
      }
    }
    if (!ok) break;
    // K0 and the first scores
    {
      int kst;
      if (!next_kv(kst)) break;
      ptx::tc_fence_after();
      if (ptx::elect_one()) {
        const uint64_t kd = stage_desc<D>(dsc.k0, kst);
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          if (nt[s] > 0) {
            issue_s<D>(tmem + s_col(s), dsc.q[s], kd);
            ptx::tc_commit(sm.s_full(s));
            if (nt[s] == 1) ptx::tc_commit(sm.q_empty(s));
          }
        }
        ptx::tc_commit(sm.kv_empty(kst));
      }
      __syncwarp();
    }
    for (int j = 0; j < n && ok; ++j) {
      int vst;
      if (!next_kv(vst)) { ok = false; break; }
      if (kCache && j == n - 1 && item_lk - j * BN < BN) {
        const int lane = threadIdx.x & 31;
        const int keep = item_lk - j * BN;  // rows of the tile inside the sequence
        uint8_t* vt = sm.kv(vst);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c)
          for (int e = lane; e < (BN - keep) * 8; e += 32)  // 16-byte units of 128-byte rows
            *reinterpret_cast<uint4*>(vt + c * C::kKVChunk + (keep + e / 8) * 128 + (e % 8) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
        ptx::fence_proxy_async_smem();
        __syncwarp();
      }
      const uint64_t vd = stage_desc<D>(dsc.v0, vst);
      int kst = -1;
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        if (ok && j < nt[s]) {
          const uint32_t ph = (tc[s] + j) & 1;
          if (j == 0) {
            ok = wait(sm.o_empty(s), (o_uses[s] & 1) ^ 1);
            ++o_uses[s];
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (ok) ok = wait(sm.p_full(s, h), ph);
            if (ok) {
              ptx::tc_fence_after();
              if (ptx::elect_one()) {
                issue_pv_half<D>(tmem + o_col<D>(s), tmem + s_col(s), vd, h, j > 0);
                if (h == 1 && j == nt[s] - 1) ptx::tc_commit(sm.o_full(s));
              }
              __syncwarp();
            }
          }
        }
        if (ok && j + 1 < nt[s]) {
          if (kst < 0) {
            ok = next_kv(kst);
            ptx::tc_fence_after();
          }
          if (ok) {
            if (ptx::elect_one()) {
              issue_s<D>(tmem + s_col(s), dsc.q[s], stage_desc<D>(dsc.k0, kst));
              ptx::tc_commit(sm.s_full(s));
              if (j + 2 == nt[s]) ptx::tc_commit(sm.q_empty(s));
            }
            __syncwarp();
          }
        }
      }
      if (!ok) break;
      if (ptx::elect_one()) {
        ptx::tc_commit(sm.kv_empty(vst));
        if (kst >= 0) ptx::tc_commit(sm.kv_empty(kst));
      }
      __syncwarp();
    }
    tc[0] += nt[0];
    tc[1] += nt[1];
  }
  // Everything issued so far has completed once `drain` flips.
  if (ptx::elect_one()) ptx::tc_commit(sm.drain());
  __syncwarp();
  drain_bar(sm.drain(), 0);
}

// Multiply this thread's O row (D fp32 columns of tensor memory) by fac.
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t t_o, float fac) {
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[32];
    ptx::tmem_ld32(t_o + c * 32, o);
    ptx::tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * fac);
    ptx::tmem_st32(t_o + c * 32, o);
  }
  ptx::tmem_wait_st();
}

// ------------------------------------------------------------------ softmax

template <int D, bool kBiasKey, bool kBiasPair, bool kCache>
__device__ void softmax_role(const Smem<D>& sm, uint32_t tmem, const AttnParams& p,
                             const Ctl& ctl) {
  using C = KCfg<D>;
  const int warp = threadIdx.x >> 5;
  const int wg = warp >> 2;                    // slot
  const int r = threadIdx.x & 127;             // tile row = TMEM lane
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t t_s = tmem + lane_base + s_col(wg);
  const uint32_t t_o = tmem + lane_base + o_col<D>(wg);
  const unsigned FULL = 0xffffffffu;
  uint32_t tc = 0, o_uses = 0;  // tiles processed (barrier phases), items with output
  bool ok = true;

  for (int it = 0; ok; ++it) {
    const int k = it & 1;
    ok = __all_sync(FULL, wait_bar(sm.item_full(k), (it >> 1) & 1, ctl));
    if (!ok) break;
    // This slot's fields, read from shared memory (a local copy of the item
    // indexed by the warp-dependent slot would live in local memory).
    const Item& itm = sm.items()[k];
    const int valid = itm.valid;
    const int rows = itm.rows[wg];
    const int n = itm.ntile[wg];
    const int head = itm.head[wg];
    const int q_loc0 = itm.q_loc0[wg];
    const int q_row0 = itm.q_row0[wg];
    const int seq = itm.seq;
    const int Lq = itm.Lq;
    const int Lk = itm.Lk;
    const int kv_row0 = itm.kv_row0;
    __syncwarp();
    if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(sm.item_empty(k));
    if (!valid) break;
    if (rows == 0) continue;
    // packed GQA: tile row r is token r / G of query head head + r % G
    constexpr bool pack = kCache;
    const int r_tok = pack ? r / p.group : r;
    const int r_head = pack ? head + r % p.group : head;
    const int q_loc = q_loc0 + r_tok;
    const bool row_ok = r < rows;
    const int limit = p.causal ? min(Lk, q_loc + (Lk - Lq) + 1) : Lk;
    float m_used = -INFINITY, l = 0.f;

    for (int j = 0; j < n; ++j) {
      const int kb = j * BN;
      const uint32_t g = tc + j;
      const int b = g & 1;                   // bias staging buffer
      const uint32_t ph = g & 1;             // phase of s_full / p_full for this tile
      float* bk = nullptr;
      if constexpr (kBiasKey) {
        // this thread's key's bias into the group's staging row, asynchronously
        // (the barrier completes when all 128 copies have landed), ahead of
        // the pair-grid copies so that the two latencies overlap
        bk = sm.bias(wg, b);
        const int key = kb + r;
        const bool in = key < Lk;
        ptx::cp_async4_zfill(ptx::smem_u32(bk + r),
                             in ? p.bias_key + (long long)(kv_row0 + key) * p.n_heads + head
                                : p.bias_key,
                             in ? 4u : 0u);
        ptx::cp_async_mbar_arrive_noinc(sm.bias_full(wg, b));
        ptx::cp_async_commit_group();
      }
      // Pair grid, 16-byte rows: the warp's 32 rows x 128 keys arrive in
      // chunks of 16 keys (2 KB) through a ring of kPairBufs staging blocks,
      // copied straight to shared memory (cp.async, coalesced: 4 lanes per
      // 64-byte row piece, 8 rows per instruction). The first chunks are in
      // flight while the scores are computed.
      const int lane = threadIdx.x & 31;
      const float* prow = nullptr;  // lane's row piece at key kb + 4 * (lane % 4)
      auto pair_dst = [&](int b, int x, int cu) {
        return ptx::smem_u32(sm.pair_buf(warp, b)) + (uint32_t)(4 * x + (cu ^ ((x >> 1) & 3))) * 16u;
      };
      auto pair_issue = [&](int ch) {
        if (ch < BN / 16) {
          const int key0 = kb + ch * 16 + 4 * (lane & 3);
          const int kleft = Lk - key0;
          const uint32_t nb = kleft >= 4 ? 16u : kleft > 0 ? 4u * (uint32_t)kleft : 0u;
#pragma unroll
          for (int k8 = 0; k8 < 4; ++k8) {
            const int x = 8 * k8 + (lane >> 2);
            const bool in = (warp & 3) * 32 + x < rows && nb > 0;
            const float* src = in ? prow + (long long)(8 * k8) * p.sr + ch * 16 : p.bias_pair;
            ptx::cp_async16_zfill(pair_dst(ch % C::kPairBufs, x, lane & 3), src, in ? nb : 0u);
          }
        }
        ptx::cp_async_commit_group();
      };
      if constexpr (kBiasPair) {
        if (p.pair_vec) {
          prow = p.bias_pair + (long long)seq * p.sb + (long long)(head / p.bias_head_div) * p.sh +
                 (long long)(q_loc0 + (warp & 3) * 32 + (lane >> 2)) * p.sr + kb + 4 * (lane & 3);
          __syncwarp();  // earlier reads of the staging blocks are done
#pragma unroll
          for (int ch = 0; ch < C::kPairBufs; ++ch) pair_issue(ch);
        }
      }
      ok = __all_sync(FULL, wait_bar(sm.s_full(wg), ph, ctl));
      if (!ok) break;
      if constexpr (kBiasKey) {
        ok = __all_sync(FULL, wait_bar(sm.bias_full(wg, b), (g >> 1) & 1, ctl));
        if (!ok) break;
      }
      ptx::tc_fence_after();
      // One 128-register row buffer: raw scores -> (log2-domain scores) -> P.
      // Without a bias and with a positive scale the scores stay raw: the
      // scale commutes with the row max and is folded into the exponent FMA.
      uint32_t u[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c)
        ptx::tmem_ld32(t_s + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&u[c * 32]));
      ptx::tmem_wait_ld();
      // With a bias the row holds natural-unit scores s * scale + bias (one
      // packed FMA per pair of keys) and log2(e) goes into the exponent's
      // FMA; without one, the raw scores stay and scale * log2(e) goes there
      // (the scale commutes with the row max when it is positive).
      constexpr bool kBiased = kBiasKey || kBiasPair;
      const bool prescaled = !kBiased && !(p.scale_log2 > 0.f);
      const uint64_t scale2 = ptx::f2(p.scale, p.scale);
      if (prescaled) {
#pragma unroll
        for (int c = 0; c < BN; ++c) u[c] = __float_as_uint(__uint_as_float(u[c]) * p.scale_log2);
      }
      if constexpr (kBiasKey) {
#pragma unroll
        for (int c = 0; c < BN; c += 2) {
          const float2 b2 = *reinterpret_cast<const float2*>(bk + c);
          const uint64_t x2 = ptx::ffma2(ptx::f2(__uint_as_float(u[c]), __uint_as_float(u[c + 1])),
                                         scale2, ptx::f2(b2.x, b2.y));
          float lo, hi;
          ptx::f2_split(x2, lo, hi);
          u[c] = __float_as_uint(lo);
          u[c + 1] = __float_as_uint(hi);
        }
      }
      // Adds a pair of grid entries to a pair of scores: onto s * scale + key
      // bias when there is a per-key bias, else onto the raw scores with the
      // scale applied in the same packed FMA.
      auto pair_add2 = [&](uint32_t& u0, uint32_t& u1, uint32_t b0, uint32_t b1, uint64_t sc2) {
        const uint64_t s2 = ptx::f2(__uint_as_float(u0), __uint_as_float(u1));
        const uint64_t g2 = ptx::f2(__uint_as_float(b0), __uint_as_float(b1));
        const uint64_t x2 = kBiasKey ? ptx::fadd2(s2, g2) : ptx::ffma2(s2, sc2, g2);
        float lo, hi;
        ptx::f2_split(x2, lo, hi);
        u0 = __float_as_uint(lo);
        u1 = __float_as_uint(hi);
      };
      if constexpr (kBiasPair) {
        if (p.pair_vec) {
#pragma unroll
          for (int ch = 0; ch < BN / 16; ++ch) {
            ptx::cp_async_wait_group<C::kPairBufs - 1>();  // chunk ch has landed
            __syncwarp();
#pragma unroll
            for (int cu = 0; cu < 4; ++cu) {
              const uint4 b = ptx::ld_shared_v4(pair_dst(ch % C::kPairBufs, lane, cu));
              const int c = ch * 16 + 4 * cu;
              pair_add2(u[c], u[c + 1], b.x, b.y, scale2);
              pair_add2(u[c + 2], u[c + 3], b.z, b.w, scale2);
            }
            __syncwarp();  // block (ch % kPairBufs) is free again
            pair_issue(ch + C::kPairBufs);
          }
        } else if (row_ok) {
          const float* brow = p.bias_pair + (long long)seq * p.sb +
                              (long long)(head / p.bias_head_div) * p.sh + (long long)q_loc * p.sr;
#pragma unroll
          for (int c = 0; c < BN; c += 4) {
            const int key = kb + c;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (key + e < Lk) {
                const float b = __ldg(brow + (long long)(key + e) * p.sc);
                const float x = __uint_as_float(u[c + e]);
                u[c + e] = __float_as_uint(kBiasKey ? x + b : fmaf(x, p.scale, b));
              }
          }
        }
      }
      if (__any_sync(FULL, kb + BN > limit)) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (kb + c >= limit) u[c] = __float_as_uint(-INFINITY);
      }
      // row max: a shallow tree of 3-input maxes (42 independent leaves)
      float mx[43];
#pragma unroll
      for (int i = 0; i < 42; ++i)
        mx[i] = ptx::fmax3(__uint_as_float(u[3 * i]), __uint_as_float(u[3 * i + 1]),
                           __uint_as_float(u[3 * i + 2]));
      mx[42] = fmaxf(__uint_as_float(u[126]), __uint_as_float(u[127]));
#pragma unroll
      for (int i = 0; i < 14; ++i) mx[i] = ptx::fmax3(mx[3 * i], mx[3 * i + 1], mx[3 * i + 2]);
      mx[14] = mx[42];
#pragma unroll
      for (int i = 0; i < 5; ++i) mx[i] = ptx::fmax3(mx[3 * i], mx[3 * i + 1], mx[3 * i + 2]);
      const float sfac = kBiased ? kLog2e : prescaled ? 1.f : p.scale_log2;
      const float m_tile = ptx::fmax3(ptx::fmax3(mx[0], mx[1], mx[2]), mx[3], mx[4]) * sfac;
      const float m_new = fmaxf(m_used, m_tile);
      const bool need = m_new > m_used + kRescaleThreshold;
      float fac = 1.f;
      if (need) {
        fac = ptx::ex2(m_used - m_new);  // 0 when m_used is -inf
        l *= fac;
        m_used = m_new;
      }
      // O_s already holds PV_s(j-1): S_s(j) was issued after it.
      if (j > 0 && __any_sync(FULL, need)) rescale_o<D>(t_o, fac);
      const float mb = m_used == -INFINITY ? 0.f : m_used;
      // P = 2^(s * sfac - mb): one packed FMA per pair, one XU ex2 per score.
      // (Moving part of the exponentials to an FMA-pipe polynomial balanced
      // the pipes but added about ten instructions per pair; under load the
      // clock is held well below its maximum (sw_power_cap), and all-ex2
      // measured 12-14% faster.) Each half of the keys is stored and
      // published as soon as it is ready.
      const uint64_t sf2 = ptx::f2(sfac, sfac), nm2 = ptx::f2(-mb, -mb);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int cc = 0; cc < BN / 4; ++cc) {
          const int c = h * (BN / 4) + cc;
          const uint64_t x2 = ptx::ffma2(
              ptx::f2(__uint_as_float(u[2 * c]), __uint_as_float(u[2 * c + 1])), sf2, nm2);
          float x0, x1;
          ptx::f2_split(x2, x0, x1);
          const uint64_t p2 = ptx::f2(ptx::ex2(x0), ptx::ex2(x1));
          acc[c & 3] = ptx::fadd2(acc[c & 3], p2);
          float p0, p1;
          ptx::f2_split(p2, p0, p1);
          u[c] = ptx::pack_bf16x2(p0, p1);  // u[c] is dead once u[2c], u[2c+1] are read
        }
        ptx::tmem_st16(t_s + h * 32, &u[h * 32]);
        ptx::tmem_st16(t_s + h * 32 + 16, &u[h * 32 + 16]);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(sm.p_full(wg, h));
      }
      {
        const uint64_t s01 = ptx::fadd2(ptx::fadd2(acc[0], acc[1]), ptx::fadd2(acc[2], acc[3]));
        float r0, r1;
        ptx::f2_split(s01, r0, r1);
        l += r0 + r1;
      }
    }
    if (!ok) break;
    tc += n;

    // epilogue: O / l -> bf16, LSE
    if (n > 0) {
      ok = __all_sync(FULL, wait_bar(sm.o_full(wg), o_uses & 1, ctl));
      if (!ok) break;
      ++o_uses;
      ptx::tc_fence_after();
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    // O / l -> bf16, 32 columns at a time, through a 2 KB per-warp staging
    // block so that the global stores are coalesced: each thread writes its
    // row's 64 bytes into the block, then every store instruction of the warp
    // writes 8 rows x 64 contiguous bytes (4 lanes per row) instead of 32
    // scattered 16-byte pieces. The block holds 32 rows x 4 16-byte units;
    // unit c of row x sits at 4x + (c ^ ((x >> 1) & 3)), which keeps both the
    // row-wise writes and the 8-row reads free of bank conflicts.
    const int lane = threadIdx.x & 31;
    const uint32_t stg = ptx::smem_u32(sm.epi(warp));
    auto unit_addr = [&](int x, int c) { return stg + (uint32_t)(4 * x + (c ^ ((x >> 1) & 3))) * 16u; };
    const int wrow0 = (warp & 3) * 32;  // first tile row of this warp
    // all of this row's O columns from tensor memory, then one wait
    uint32_t o[D];
    if (n > 0) {
#pragma unroll
      for (int c = 0; c < D / 32; ++c)
        ptx::tmem_ld32(t_o + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&o[c * 32]));
      ptx::tmem_wait_ld();
    } else {
#pragma unroll
      for (int e = 0; e < D; ++e) o[e] = 0u;
    }
    // a key range of a decode step: its fp32 output, normalised by its own
    // sum, to the partial buffer (one row per thread; the rows are few)
    const bool part = kCache && p.part_o != nullptr;
    const int rg = part ? seq % p.cache_ranges : 0;
    if (part && row_ok) {
      float* dst = p.part_o + (((long long)rg * p.total_q + q_row0 + r_tok) * p.n_heads + r_head) * D;
#pragma unroll
      for (int c = 0; c < D; c += 4)
        *reinterpret_cast<float4*>(dst + c) =
            make_float4(__uint_as_float(o[c]) * inv, __uint_as_float(o[c + 1]) * inv,
                        __uint_as_float(o[c + 2]) * inv, __uint_as_float(o[c + 3]) * inv);
    }
    if (!part) {
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t vw[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          vw[e] = ptx::pack_bf16x2(__uint_as_float(o[c * 32 + 2 * e]) * inv,
                                   __uint_as_float(o[c * 32 + 2 * e + 1]) * inv);
        __syncwarp();  // the previous block's reads are done
#pragma unroll
        for (int u4 = 0; u4 < 4; ++u4)
          ptx::st_shared_v4(unit_addr(lane, u4), vw[4 * u4], vw[4 * u4 + 1], vw[4 * u4 + 2], vw[4 * u4 + 3]);
        __syncwarp();
#pragma unroll
        for (int k8 = 0; k8 < 4; ++k8) {
          const int x = 8 * k8 + (lane >> 2), cu = lane & 3;
          const uint4 val = ptx::ld_shared_v4(unit_addr(x, cu));
          if (wrow0 + x < rows) {
            const int xr = wrow0 + x;
            const int tok = pack ? xr / p.group : xr, hh = pack ? head + xr % p.group : head;
            __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) +
                                 ((long long)(q_row0 + tok) * p.n_heads + hh) * D + c * 32 + cu * 8;
            *reinterpret_cast<uint4*>(dst) = val;
          }
        }
      }
    }
    if (n > 0) {
      ptx::tc_fence_before();
      ptx::mbar_arrive(sm.o_empty(wg));
    }
    float* lse_out = part ? p.part_lse + (long long)rg * p.n_heads * p.total_q : p.lse;
    if (row_ok && lse_out != nullptr) {
      const float lse = l > 0.f ? (m_used + __log2f(l)) * kLn2 : -INFINITY;
      lse_out[(long long)r_head * p.total_q + q_row0 + r_tok] = lse;
    }
  }
  if constexpr (kBiasKey || kBiasPair) ptx::cp_async_wait_group<0>();  // copies left by an abort
}

// ------------------------------------------------------------------ kernel
template <int D, bool kBiasKey, bool kBiasPair, bool kCache = false>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem<D> sm;
  {
    const uint32_t a = ptx::smem_u32(smem_raw);
    sm.base = smem_raw + ((1024 - (a & 1023)) & 1023);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(sm.q_full(s), 1);
      ptx::mbar_init(sm.q_empty(s), 1);
      ptx::mbar_init(sm.s_full(s), 1);
      for (int b = 0; b < 2; ++b) {
        ptx::mbar_init(sm.p_full(s, b), 128);
        ptx::mbar_init(sm.bias_full(s, b), 128);
      }
      ptx::mbar_init(sm.o_full(s), 1);
      ptx::mbar_init(sm.o_empty(s), 128);
      ptx::mbar_init(sm.item_full(s), 1);
      ptx::mbar_init(sm.item_empty(s), 1 + 8);  // MMA warp, eight softmax warps
    }
    ptx::mbar_init(sm.drain(), 1);
    for (int st = 0; st < KCfg<D>::kStages; ++st) {
      ptx::mbar_init(sm.kv_full(st), 1);
      ptx::mbar_init(sm.kv_empty(st), 1);
    }
    *sm.abort_flag() = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(sm.tmem_slot(), 512);
    ptx::tmem_relinquish();
  }
  if (warp == kLoadWarp && lane == 0) {
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot();
  const Ctl ctl{sm.abort_flag(), p.error, p.wait_limit};

  if (warp < 8) {
    ptx::setmaxnreg_inc<kSoftmaxRegs>();
    softmax_role<D, kBiasKey, kBiasPair, kCache>(sm, tmem, p, ctl);
  } else {
    ptx::setmaxnreg_dec<kWorkerRegs>();
    if (warp == kMmaWarp) {
      mma_role<D, kCache>(sm, tmem, ctl, p.test_stall);
    } else if (warp == kLoadWarp) {
      load_role<D, kCache>(sm, &tm_q, &tm_k, &tm_v, p, ctl);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

}  // namespace va
