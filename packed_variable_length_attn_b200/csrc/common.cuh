// Shared definitions of the packed varlen attention kernels: tile sizes,
// launch parameters, the work item and its decoding from the work list.
#pragma once
#include <cstdint>

namespace va {

constexpr int BM = 128;  // query rows per slot tile (= TMEM lanes)
constexpr int BN = 128;  // keys per K/V tile

// Status codes (mirror varlen_attn_status in include/varlen_attn.h).
constexpr int kErrBadSeqlens = 9;
constexpr int kErrTimeout = 10;

// How the two 128-row slots of a CTA work item are filled.
//  kPairHeads:   GQA (G >= 2). The G x (q-blocks) units (q-block, query head)
//                of one sequence and K/V head, taken q-block by q-block, are
//                paired consecutively: with G even, two heads at the same
//                q-block; with G odd, a q-block's last head shares an item
//                with the next q-block's first one. Both slots read the same
//                K/V tiles.
//  kPairQBlocks: two consecutive q-blocks of one head (no GQA sharing).
//  kPackGQA:     decode-sized queries (Lq * G <= 128 rows): one item per
//                (sequence, K/V head) whose single slot holds the rows of all
//                G query heads of the group, row rho = token (rho / G) of
//                head (rho % G); slot 1 is unused.
constexpr int kPairHeads = 0;
constexpr int kPairQBlocks = 1;
constexpr int kPackGQA = 3;

// Work list in the library workspace (device memory).
struct Workspace {
  int* counter;  // next work index (reset by the schedule kernel)
  int* count;    // number of work items (0 = nothing to do / invalid input)
  int2* list;    // sorted (sequence, group) pairs, `capacity` entries
  int2* tmp;     // unsorted pairs, `capacity` entries
  int capacity;
};

struct SchedParams {
  const int* cu_q;
  const int* cu_k;
  int batch, total_q, total_k, max_q, max_k;
  int causal;
  int pairing;      // kPairHeads / kPairQBlocks / kPackGQA; -1 = validate only
  int group;        // G = Hq / Hkv
  int n_hg;         // work items per (sequence, group) pair
  // K/V read in place from a per-sequence cache (cache_seqlens != null):
  // sequence i's keys are rows i*cache_len .. of the cache, Lk_i =
  // cache_seqlens[i] (+ Lq_i when its new rows were appended); cu_k unused.
  const int* cache_seqlens;
  int cache_len, cache_extra;
  // Key ranges (cache mode, cache_ranges > 1): the list is built over
  // batch * cache_ranges virtual sequences, j = i * cache_ranges + r holding
  // keys [r * range_keys, (r + 1) * range_keys) of sequence i (range_lk).
  int cache_ranges, range_keys;
  Workspace ws;
  int* error;       // device error word
};

// Key count of sequence i: from cu_seqlens_k, or from the cache lengths.
template <typename P>
__device__ __forceinline__ int seq_lk(const P& p, int i) {
  if (p.cache_seqlens != nullptr)
    return p.cache_seqlens[i] + (p.cache_extra ? p.cu_q[i + 1] - p.cu_q[i] : 0);
  return p.cu_k[i + 1] - p.cu_k[i];
}

// Key count of virtual sequence j when the cache's keys are cut into ranges
// (sequence j / cache_ranges, range j % cache_ranges); seq_lk without ranges.
template <typename P>
__device__ __forceinline__ int range_lk(const P& p, int j) {
  if (p.cache_ranges <= 1) return seq_lk(p, j);
  const int i = j / p.cache_ranges;
  const int left = seq_lk(p, i) - (j - i * p.cache_ranges) * p.range_keys;
  return left < 0 ? 0 : left < p.range_keys ? left : p.range_keys;
}

// Query rows of virtual sequence j (those of sequence j / cache_ranges).
template <typename P>
__device__ __forceinline__ int range_lq(const P& p, int j) {
  const int i = p.cache_ranges > 1 ? j / p.cache_ranges : j;
  return p.cu_q[i + 1] - p.cu_q[i];
}

struct AttnParams {
  const int* cu_q;
  const int* cu_k;
  int total_q;
  int n_heads, n_kv_heads, group;  // Hq, Hkv, G = Hq / Hkv
  int pairing, n_hg;
  int causal;
  float scale_log2;                // softmax_scale * log2(e)
  float scale;                     // softmax_scale
  const float* bias_key;           // [Tk, Hq] or null
  const float* bias_pair;          // strided grid or null
  long long sb, sh, sr, sc;
  int bias_head_div;               // grid head index = head / bias_head_div (1: query
                                   // heads; G: K/V heads)
  int pair_vec;                    // 1: 16-byte vector loads of the grid are legal
  void* out;                       // bf16 [Tq, Hq, D]
  float* lse;                      // [Hq, Tq] or null
  Workspace ws;
  int* error;
  long long wait_limit;            // cycles a bounded wait may take
  int test_stall;                  // test hook: the MMA warp first waits on a barrier
                                   // phase nothing completes (its wait runs out)
  // K/V cache mode (see SchedParams) and the packed-GQA rows of kPackGQA
  const int* cache_seqlens;
  int cache_len, cache_extra;
  int q_box_rows;                  // rows one Q tile load writes (128, or G * (128 / G))
  // Key ranges (see SchedParams): each range's output, normalised by its own
  // sum, goes to part_o [ranges, Tq, Hq, D] fp32 and its LSE to part_lse
  // [ranges, Hq, Tq]; a split-combine kernel merges them.
  int cache_ranges, range_keys;
  float* part_o;
  float* part_lse;
};

// One CTA work item: up to two 128-row query tiles (slots) that stream the
// same K/V tiles of one K/V head.
struct Item {
  int valid;
  int seq;
  int kvh;
  int kv_row0;   // cu_k[seq]
  int Lq, Lk;
  int q_row0[2]; // global first row of each slot
  int q_loc0[2]; // first row of each slot, local to the sequence
  int head[2];
  int rows[2];   // valid rows in the slot (0 = slot unused)
  int ntile[2];  // K/V tiles the slot needs (0 = no visible key)
};

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// K/V tiles a slot with local rows [q_loc0, q_loc0 + rows) must visit. With
// the bottom-right causal mask the last row sees keys c < last + Lk - Lq + 1,
// and fully masked tiles past that are skipped.
__host__ __device__ __forceinline__ int slot_tiles(int q_loc0, int rows, int Lq, int Lk,
                                                   int causal) {
  if (rows <= 0 || Lk <= 0) return 0;
  const int nk = ceil_div(Lk, BN);
  if (!causal) return nk;
  const int lim = q_loc0 + rows - 1 + (Lk - Lq) + 1;
  if (lim <= 0) return 0;
  const int n = ceil_div(lim, BN);
  return n < nk ? n : nk;
}

// Number of (sequence, group) pairs sequence i contributes: unit pairs of
// its (q-block, head) units per K/V head, or q-block pairs.
__host__ __device__ __forceinline__ int seq_groups(int Lq, int pairing, int group) {
  const int nqb = ceil_div(Lq, BM);
  if (pairing == kPackGQA) return 1;
  return pairing == kPairHeads ? ceil_div(group * nqb, 2) : ceil_div(nqb, 2);
}

// First local query row of slot s of pair g, and the slot's query head
// (local to the K/V group for kPairHeads).
__host__ __device__ __forceinline__ void slot_unit(int g, int s, int pairing, int group,
                                                   int& q_loc0, int& hl) {
  if (pairing == kPackGQA) {
    q_loc0 = s == 0 ? 0 : (1 << 29);
    hl = 0;
  } else if (pairing == kPairHeads) {
    const int unit = 2 * g + s;
    q_loc0 = (unit / group) * BM;
    hl = unit % group;
  } else {
    q_loc0 = (2 * g + s) * BM;
    hl = 0;
  }
}

__device__ __forceinline__ void fill_slots(Item& it, int g, int hg, int pairing, int group,
                                           int causal) {
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    int active, head, q_loc0;
    if (pairing == kPairHeads || pairing == kPackGQA) {
      int hl;
      slot_unit(g, s, pairing, group, q_loc0, hl);
      active = q_loc0 < it.Lq;
      head = it.kvh * group + hl;  // kPackGQA: the group's first head
    } else {
      head = hg;
      q_loc0 = (2 * g + s) * BM;
      active = q_loc0 < it.Lq;
    }
    int rows = it.Lq - q_loc0;
    rows = rows < BM ? rows : BM;
    if (!active || rows < 0) rows = 0;
    it.head[s] = head;
    it.q_loc0[s] = q_loc0;
    it.rows[s] = rows;
    it.ntile[s] = slot_tiles(q_loc0, rows, it.Lq, it.Lk, causal);
    if (pairing == kPackGQA) it.rows[s] = rows * group;  // tile rows: tokens x heads
  }
}

}  // namespace va
