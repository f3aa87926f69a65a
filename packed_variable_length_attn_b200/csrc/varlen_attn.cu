// Host side of the C ABI declared in include/varlen_attn.h: argument
// validation, TMA descriptor encoding, the per-(device, stream) workspace,
// and the launches of the schedule kernel and the attention kernel.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstdio>
#include <cstring>
#include <map>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <utility>

#include "../../include/varlen_attn.h"
#include "attn_f32.cuh"
#include "attn_sm100.cuh"
#include "sched.cuh"
#include "layout.cuh"
#include "decode.cuh"
#include "bwd_sm100.cuh"

// ---------------------------------------------------------------------------
// Fixed scratch for varlen_attn_fwd_noalloc.
//
// Some callers cannot let a library allocate device memory behind their
// back: runtimes that reserve the whole device pool up front and fail any
// outside cudaMalloc, serving loops that must not stall (cudaMalloc and
// cudaFree can synchronise the device and take unbounded time), and hosts
// that give a plug-in a fixed memory budget. For them the work list lives in
// this array instead of the grow-only workspace. It is part of the library's
// module: every GPU that loads the library holds it until the process exits.
// All calls on one device share it, so calls that can run at the same time
// on that device race on it.
constexpr int kNoAllocMaxPairs = 16384;
constexpr size_t kNoAllocScratchBytes = 256 + 2 * (size_t)kNoAllocMaxPairs * sizeof(int2);
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

using namespace va;

__device__ int g_device_error = 0;

constexpr int kVersion = 100;  // 0.1.0

// Key ranges of the tensor-core decode path (used when the (sequence, K/V
// head) pairs are fewer than the SMs): about this many work items per SM were
// every sequence full, ranges of at least this many keys, at most this many.
constexpr int kRangeItemsPerSm = 8;
constexpr int kMinRangeKeys = 512;
constexpr int kMaxRanges = 64;

struct DeviceInfo {
  bool init = false;
  int sm_count = 0;
  int cc_major = 0, cc_minor = 0;
  int* error_word = nullptr;
};

std::mutex g_mu;
std::map<int, DeviceInfo> g_dev;
struct WsBuf {
  void* ptr = nullptr;
  size_t bytes = 0;
};
std::map<std::pair<int, void*>, WsBuf> g_ws;

thread_local char t_detail[256] = "";

// Records which step failed and CUDA's message; returns VARLEN_ATTN_ERR_CUDA.
int cuda_fail(const char* step, cudaError_t e) {
  snprintf(t_detail, sizeof t_detail, "%s: %s (%d)", step, cudaGetErrorString(e), (int)e);
  return VARLEN_ATTN_ERR_CUDA;
}

// Limit of the kernels' bounded waits, in SM clock cycles (0 = default).
std::atomic<long long> g_wait_limit{0};
// Test hook of the abort path (varlen_attn_set_test_stall).
std::atomic<int> g_test_stall{0};
long long wait_limit() {
  const long long v = g_wait_limit.load(std::memory_order_relaxed);
  return v > 0 ? v : kWaitLimitCycles;
}

thread_local cudaEvent_t t_ev_start = nullptr;
thread_local cudaEvent_t t_ev_stop = nullptr;

int device_info(DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.init) {
    if ((e = cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&di.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&di.cc_minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return cuda_fail("cudaDeviceGetAttribute", e);
    if ((e = cudaGetSymbolAddress(reinterpret_cast<void**>(&di.error_word), g_device_error)) != cudaSuccess)
      return cuda_fail("cudaGetSymbolAddress(error word)", e);
    di.init = true;
  }
  if (di.cc_major != 10 || di.cc_minor != 0) return VARLEN_ATTN_ERR_DEVICE;
  *out = &di;
  return VARLEN_ATTN_OK;
}

// Grow-only workspace of `bytes` for (current device, stream).
int workspace(void* stream, size_t bytes, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
  std::lock_guard<std::mutex> lk(g_mu);
  WsBuf& b = g_ws[std::make_pair(dev, stream)];
  if (b.bytes < bytes) {
    if (b.ptr != nullptr) {
      // Earlier launches on this stream may still read the old buffer.
      if ((e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream))) != cudaSuccess)
        return cuda_fail("cudaStreamSynchronize(workspace growth)", e);
      cudaFree(b.ptr);
      b.ptr = nullptr;
      b.bytes = 0;
    }
    size_t want = bytes < (1u << 16) ? (1u << 16) : bytes;
    if ((e = cudaMalloc(&b.ptr, want)) != cudaSuccess) return cuda_fail("cudaMalloc(workspace)", e);
    b.bytes = want;
  }
  *out = b.ptr;
  return VARLEN_ATTN_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static cudaError_t err = cudaSuccess;
  static int qres = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    err = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q);
    qres = (int)q;
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  if (fn == nullptr)
    snprintf(t_detail, sizeof t_detail, "cudaGetDriverEntryPointByVersion(cuTensorMapEncodeTiled): %s, query %d",
             cudaGetErrorString(err), qres);
  return fn;
}

// [rows, heads, D] bf16, box = 64 columns x 1 head x box_rows rows, 128-byte swizzle.
bool make_tmap(CUtensorMap* m, const void* base, int D, int heads, int rows, int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) snprintf(t_detail, sizeof t_detail, "cuTensorMapEncodeTiled: CUresult %d", (int)r);
  return r == CUDA_SUCCESS;
}

// Tensor map with a box of box_heads heads x box_rows rows (64 columns).
bool make_tmap_box(CUtensorMap* m, const void* base, int D, int heads, int rows, int box_heads,
                   int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) snprintf(t_detail, sizeof t_detail, "cuTensorMapEncodeTiled: CUresult %d", (int)r);
  return r == CUDA_SUCCESS;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Base of a K or V tensor map. With no keys at all (total_k == 0, k and v
// possibly NULL) no K/V tile is ever loaded, but a tensor map still needs a
// valid aligned address: q's stands in.
const void* kv_base(const void* kv, const void* q, int total_k) {
  return total_k > 0 ? kv : q;
}

struct Common {
  int batch, total_q, total_k, max_q, max_k, Hq, Hkv, D, causal;
  const int32_t *cu_q, *cu_k;
  const float *bias_key, *bias_pair;
  int64_t sb, sh, sr, sc;
};

int validate_common(const Common& a, const void* q, const void* k, const void* v, const void* out,
                    const float* lse) {
  if (!q || !out || !a.cu_q || !a.cu_k) return VARLEN_ATTN_ERR_NULL_POINTER;
  // k and v may be NULL only when there are no keys at all (never read then)
  if (a.total_k > 0 && (!k || !v)) return VARLEN_ATTN_ERR_NULL_POINTER;
  if (a.batch <= 0 || a.Hq <= 0 || a.Hkv <= 0 || a.D <= 0 || a.total_q < 0 || a.total_k < 0 ||
      a.max_q < 0 || a.max_k < 0)
    return VARLEN_ATTN_ERR_BAD_SHAPE;
  if (a.Hq % a.Hkv != 0) return VARLEN_ATTN_ERR_GQA_MISMATCH;
  if (a.D != 64 && a.D != 128) return VARLEN_ATTN_ERR_HEAD_DIM;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
    return VARLEN_ATTN_ERR_MISALIGNED;
  if ((lse && !aligned(lse, 4)) || (a.bias_key && !aligned(a.bias_key, 4)) ||
      (a.bias_pair && !aligned(a.bias_pair, 4)) || !aligned(a.cu_q, 4) || !aligned(a.cu_k, 4))
    return VARLEN_ATTN_ERR_MISALIGNED;
  if (a.bias_pair && (a.sb < 0 || a.sh < 0 || a.sr < 0 || a.sc < 0)) return VARLEN_ATTN_ERR_BAD_BIAS;
  // 32-bit indexing limits of the kernels.
  if ((int64_t)a.total_q * a.Hq > INT32_MAX || (int64_t)a.total_k * a.Hkv > INT32_MAX ||
      (int64_t)a.batch + 1 > INT32_MAX / 2)
    return VARLEN_ATTN_ERR_TOO_LARGE;
  return VARLEN_ATTN_OK;
}

template <typename K>
int set_smem(K kernel, int bytes) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  return e == cudaSuccess ? VARLEN_ATTN_OK : cuda_fail("cudaFuncSetAttribute(smem)", e);
}

int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? VARLEN_ATTN_OK : cuda_fail(what, e);
}

template <int D, bool BK, bool BP, bool CACHE = false>
int launch_attn(int grid, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                const AttnParams& prm, cudaStream_t st) {
  auto kern = attn_fwd_sm100<D, BK, BP, CACHE>;
  static thread_local int configured_for = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_for != dev) {
    // The in-kernel register split assumes exactly kLaunchRegs per thread at
    // launch; with fewer, setmaxnreg.inc could never be satisfied.
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return cuda_fail("cudaFuncGetAttributes", e);
    if (fa.numRegs != kLaunchRegs) {
      snprintf(t_detail, sizeof t_detail, "attn_fwd_sm100 compiled with %d registers, expected %d",
               fa.numRegs, kLaunchRegs);
      return VARLEN_ATTN_ERR_CUDA;
    }
    if (int rc = set_smem(kern, KCfg<D>::kSmemBytes)) return rc;
    configured_for = dev;
  }
  // Programmatic dependent launch: the kernel may start while the schedule
  // kernel before it on the stream still runs (its barrier set-up, tensor
  // memory allocation and descriptor prefetch overlap it); the load warp
  // waits for the schedule kernel's results (griddepcontrol.wait) before it
  // reads the work list, and no other role reads what the schedule writes.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kAttnThreads);
  cfg.dynamicSmemBytes = KCfg<D>::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, prm);
  if (e != cudaSuccess) return cuda_fail("launch attn_fwd_sm100", e);
  return check_launch("launch attn_fwd_sm100");
}

int launch_schedule(const SchedParams& sp, cudaStream_t st) {
  static thread_local int configured_for = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  const int smem = kSchedSmemBytes;
  if (configured_for != dev) {
    if (int rc = set_smem(schedule_kernel, smem)) return rc;
    configured_for = dev;
  }
  schedule_kernel<<<1, kSchedThreads, smem, st>>>(sp);
  return check_launch("launch schedule_kernel");
}

Workspace carve(void* base, int capacity) {
  Workspace ws;
  char* b = static_cast<char*>(base);
  ws.counter = reinterpret_cast<int*>(b);
  ws.count = reinterpret_cast<int*>(b + 4);
  ws.list = reinterpret_cast<int2*>(b + 256);
  ws.tmp = ws.list + capacity;
  ws.capacity = capacity;
  return ws;
}

// Device address of g_noalloc_scratch on the current device. In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
constexpr int kMaxDevices = 64;
void* g_noalloc_addr[kMaxDevices] = {};

int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
  if (dev < 0 || dev >= kMaxDevices) {
    snprintf(t_detail, sizeof t_detail, "device ordinal %d beyond %d", dev, kMaxDevices);
    return VARLEN_ATTN_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail("cudaGetSymbolAddress(no-alloc scratch)", e);
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return VARLEN_ATTN_OK;
}

int fwd_bf16(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
             const int32_t* cu_seqlens_k, int batch, int total_q, int total_k, int max_seqlen_q,
             int max_seqlen_k, int n_heads, int n_kv_heads, int head_dim, float softmax_scale,
             int causal, const float* bias_per_key, const float* bias_pair, int64_t bias_stride_b,
             int64_t bias_stride_h, int64_t bias_stride_q, int64_t bias_stride_k, unsigned flags,
             void* out, float* lse, void* stream, bool fixed_scratch) {
  if (flags & ~(unsigned)VARLEN_ATTN_BIAS_PAIR_KV_HEADS) return VARLEN_ATTN_ERR_BAD_BIAS;
  Common a{batch, total_q, total_k, max_seqlen_q, max_seqlen_k, n_heads, n_kv_heads, head_dim,
           causal ? 1 : 0, cu_seqlens_q, cu_seqlens_k, bias_per_key, bias_pair, bias_stride_b,
           bias_stride_h, bias_stride_q, bias_stride_k};
  int rc = validate_common(a, q, k, v, out, lse);
  if (rc) return rc;
  DeviceInfo* di = nullptr;
  if ((rc = device_info(&di))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (total_q == 0 || max_seqlen_q == 0) return VARLEN_ATTN_OK;  // no query rows

  const int G = n_heads / n_kv_heads;
  const int pairing = G >= 2 ? kPairHeads : kPairQBlocks;
  const int n_hg = pairing == kPairHeads ? n_kv_heads : n_heads;
  if ((int64_t)G * ceil_div(max_seqlen_q, BM) > INT32_MAX / 2) return VARLEN_ATTN_ERR_TOO_LARGE;
  const int64_t groups_per_seq = seq_groups(max_seqlen_q, pairing, G);
  const int64_t capacity = (int64_t)batch * groups_per_seq;
  if (capacity * n_hg > INT32_MAX || capacity > (INT32_MAX / 16)) return VARLEN_ATTN_ERR_TOO_LARGE;

  // The work list lives in the grow-only workspace, or, for the no-allocation
  // entry point, in the fixed module array (never allocated, never cleared:
  // the schedule kernel rewrites the counter, the count and every list entry
  // it publishes before the attention kernel reads them).
  void* wsp = nullptr;
  if (fixed_scratch) {
    if (capacity > kNoAllocMaxPairs) {
      snprintf(t_detail, sizeof t_detail,
               "work list of %lld (sequence, q-block group) pairs exceeds the fixed scratch of %d",
               (long long)capacity, kNoAllocMaxPairs);
      return VARLEN_ATTN_ERR_SCRATCH_LIMIT;
    }
    if ((rc = noalloc_scratch(&wsp))) return rc;
  } else if ((rc = workspace(stream, 256 + 2 * (size_t)capacity * sizeof(int2), &wsp))) {
    return rc;
  }
  Workspace ws = carve(wsp, (int)capacity);

  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, q, head_dim, n_heads, total_q, BM) ||
      !make_tmap(&tk, kv_base(k, q, total_k), head_dim, n_kv_heads, total_k, BN) ||
      !make_tmap(&tv, kv_base(v, q, total_k), head_dim, n_kv_heads, total_k, BN))
    return VARLEN_ATTN_ERR_CUDA;

  SchedParams sp;
  std::memset(&sp, 0, sizeof sp);  // no K/V cache
  sp.cu_q = cu_seqlens_q;
  sp.cu_k = cu_seqlens_k;
  sp.batch = batch;
  sp.total_q = total_q;
  sp.total_k = total_k;
  sp.max_q = max_seqlen_q;
  sp.max_k = max_seqlen_k;
  sp.causal = a.causal;
  sp.pairing = pairing;
  sp.group = G;
  sp.n_hg = n_hg;
  sp.ws = ws;
  sp.error = di->error_word;
  if ((rc = launch_schedule(sp, st))) return rc;

  AttnParams prm;
  std::memset(&prm, 0, sizeof prm);  // no K/V cache
  prm.q_box_rows = BM;
  prm.cu_q = cu_seqlens_q;
  prm.cu_k = cu_seqlens_k;
  prm.total_q = total_q;
  prm.n_heads = n_heads;
  prm.n_kv_heads = n_kv_heads;
  prm.group = G;
  prm.pairing = pairing;
  prm.n_hg = n_hg;
  prm.causal = a.causal;
  prm.scale_log2 = softmax_scale * 1.4426950408889634f;
  prm.scale = softmax_scale;
  prm.bias_key = bias_per_key;
  prm.bias_pair = bias_pair;
  prm.sb = bias_stride_b;
  prm.sh = bias_stride_h;
  prm.bias_head_div = (flags & VARLEN_ATTN_BIAS_PAIR_KV_HEADS) ? G : 1;
  prm.sr = bias_stride_q;
  prm.sc = bias_stride_k;
  prm.pair_vec = bias_pair && bias_stride_k == 1 && aligned(bias_pair, 16) &&
                 bias_stride_b % 4 == 0 && bias_stride_h % 4 == 0 && bias_stride_q % 4 == 0;
  prm.out = out;
  prm.lse = lse;
  prm.ws = ws;
  prm.error = di->error_word;
  prm.wait_limit = wait_limit();
  prm.test_stall = g_test_stall.load(std::memory_order_relaxed);

  int64_t items = capacity * n_hg;
  const int grid = (int)(items < di->sm_count ? items : di->sm_count);
  if (t_ev_start && t_ev_stop) {
    cudaError_t e = cudaEventRecord(t_ev_start, st);
    if (e != cudaSuccess) return cuda_fail("cudaEventRecord(start)", e);
  }
  const bool bk = bias_per_key != nullptr, bp = bias_pair != nullptr;
  if (head_dim == 64) {
    if (bk && bp) rc = launch_attn<64, true, true>(grid, tq, tk, tv, prm, st);
    else if (bk) rc = launch_attn<64, true, false>(grid, tq, tk, tv, prm, st);
    else if (bp) rc = launch_attn<64, false, true>(grid, tq, tk, tv, prm, st);
    else rc = launch_attn<64, false, false>(grid, tq, tk, tv, prm, st);
  } else {
    if (bk && bp) rc = launch_attn<128, true, true>(grid, tq, tk, tv, prm, st);
    else if (bk) rc = launch_attn<128, true, false>(grid, tq, tk, tv, prm, st);
    else if (bp) rc = launch_attn<128, false, true>(grid, tq, tk, tv, prm, st);
    else rc = launch_attn<128, false, false>(grid, tq, tk, tv, prm, st);
  }
  if (rc) return rc;
  if (t_ev_start && t_ev_stop) {
    cudaError_t e = cudaEventRecord(t_ev_stop, st);
    if (e != cudaSuccess) return cuda_fail("cudaEventRecord(stop)", e);
  }
  return VARLEN_ATTN_OK;
}

int layout_grid(const DeviceInfo* di, int64_t units) {
  const int64_t want = (units + kLayoutThreads - 1) / kLayoutThreads;
  const int64_t cap = (int64_t)di->sm_count * 8;
  return (int)std::max<int64_t>(1, std::min(want, cap));
}

int rows_args_ok(const void* src, int64_t src_rows, int64_t row_bytes, const int32_t* indices,
                 const int32_t* cu, int batch, const void* dst, int64_t dst_rows) {
  if (!src || !dst || !indices || !cu) return VARLEN_ATTN_ERR_NULL_POINTER;
  if (batch <= 0 || src_rows < 0 || dst_rows < 0 || row_bytes <= 0 || row_bytes % 16 != 0)
    return VARLEN_ATTN_ERR_BAD_SHAPE;
  if (!aligned(src, 16) || !aligned(dst, 16) || !aligned(indices, 4) || !aligned(cu, 4))
    return VARLEN_ATTN_ERR_MISALIGNED;
  return VARLEN_ATTN_OK;
}

template <int D, int RT>
int launch_decode_tma(dim3 grid, const CUtensorMap& tk, const CUtensorMap& tv,
                      const DecodeParams& dp, cudaStream_t st) {
  auto kern = decode_tma_kernel<D, RT>;
  if (int rc = set_smem(kern, Dec2Cfg<D, RT>::kBytes)) return rc;
  kern<<<grid, kDec2Threads, Dec2Cfg<D, RT>::kBytes, st>>>(tk, tv, dp, wait_limit());
  return check_launch("launch decode_tma_kernel");
}

template <int D, int RT>
int launch_decode(dim3 grid, const DecodeParams& dp, cudaStream_t st) {
  auto kern = decode_kernel<D, RT>;
  if (int rc = set_smem(kern, DecSmem<D, RT>::kBytes)) return rc;
  kern<<<grid, kDecThreads, DecSmem<D, RT>::kBytes, st>>>(dp);
  return check_launch("launch decode_kernel");
}

}  // namespace

template <int D, bool BK, bool BP>
int launch_bwd(dim3 grid_a, dim3 grid_q, const CUtensorMap& tq, const CUtensorMap& tk,
               const CUtensorMap& tv, const CUtensorMap& tdo, const BwdParams& bp,
               cudaStream_t st) {
  auto ka = attn_bwd_dkdv_sm100<D, BK, BP>;
  auto kq = attn_bwd_dq_sm100<D, BK, BP>;
  static thread_local int configured_for = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_for != dev) {
    int rc;
    if ((rc = set_smem(ka, BwdCfg<D>::kSmemBytes)) || (rc = set_smem(kq, BwdCfg<D>::kSmemBytes)))
      return rc;
    configured_for = dev;
  }
  ka<<<grid_a, kBwdThreads, BwdCfg<D>::kSmemBytes, st>>>(tq, tk, tv, tdo, bp);
  if (int rc = check_launch("attn_bwd_dkdv_sm100")) return rc;
  kq<<<grid_q, kBwdThreads, BwdCfg<D>::kSmemBytes, st>>>(tq, tk, tv, tdo, bp);
  return check_launch("attn_bwd_dq_sm100");
}

extern "C" {

int varlen_attn_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                    const int32_t* cu_seqlens_k, int batch, int total_q, int total_k,
                    int max_seqlen_q, int max_seqlen_k, int n_heads, int n_kv_heads, int head_dim,
                    float softmax_scale, int causal, const float* bias_per_key,
                    const float* bias_pair, int64_t bias_stride_b, int64_t bias_stride_h,
                    int64_t bias_stride_q, int64_t bias_stride_k, void* out, float* lse,
                    void* stream) {
  return fwd_bf16(q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q,
                  max_seqlen_k, n_heads, n_kv_heads, head_dim, softmax_scale, causal, bias_per_key,
                  bias_pair, bias_stride_b, bias_stride_h, bias_stride_q, bias_stride_k, 0u, out,
                  lse, stream, /*fixed_scratch=*/false);
}

int varlen_attn_fwd_ex(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                       const int32_t* cu_seqlens_k, int batch, int total_q, int total_k,
                       int max_seqlen_q, int max_seqlen_k, int n_heads, int n_kv_heads,
                       int head_dim, float softmax_scale, int causal, const float* bias_per_key,
                       const float* bias_pair, int64_t bias_stride_b, int64_t bias_stride_h,
                       int64_t bias_stride_q, int64_t bias_stride_k, unsigned flags, void* out,
                       float* lse, void* stream) {
  return fwd_bf16(q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q,
                  max_seqlen_k, n_heads, n_kv_heads, head_dim, softmax_scale, causal, bias_per_key,
                  bias_pair, bias_stride_b, bias_stride_h, bias_stride_q, bias_stride_k, flags, out,
                  lse, stream, /*fixed_scratch=*/false);
}

int varlen_attn_fwd_f32(const float* q, const float* k, const float* v,
                        const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                        int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                        int n_heads, int n_kv_heads, int head_dim, float softmax_scale,
                        int causal, const float* bias_per_key, const float* bias_pair,
                        int64_t bias_stride_b, int64_t bias_stride_h, int64_t bias_stride_q,
                        int64_t bias_stride_k, float* out, float* lse, void* stream) {
  Common a{batch, total_q, total_k, max_seqlen_q, max_seqlen_k, n_heads, n_kv_heads, head_dim,
           causal ? 1 : 0, cu_seqlens_q, cu_seqlens_k, bias_per_key, bias_pair, bias_stride_b,
           bias_stride_h, bias_stride_q, bias_stride_k};
  int rc = validate_common(a, q, k, v, out, lse);
  if (rc) return rc;
  DeviceInfo* di = nullptr;
  if ((rc = device_info(&di))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (total_q == 0 || max_seqlen_q == 0) return VARLEN_ATTN_OK;
  const int64_t qblocks = ((int64_t)max_seqlen_q + kF32Rows - 1) / kF32Rows;
  if ((int64_t)batch * qblocks > INT32_MAX || n_heads > 65535) return VARLEN_ATTN_ERR_TOO_LARGE;

  void* wsp = nullptr;
  if ((rc = workspace(stream, 256, &wsp))) return rc;
  Workspace ws = carve(wsp, 0);
  SchedParams sp;
  std::memset(&sp, 0, sizeof sp);
  sp.cu_q = cu_seqlens_q;
  sp.cu_k = cu_seqlens_k;
  sp.batch = batch;
  sp.total_q = total_q;
  sp.total_k = total_k;
  sp.max_q = max_seqlen_q;
  sp.max_k = max_seqlen_k;
  sp.causal = a.causal;
  sp.pairing = -1;  // validate only
  sp.ws = ws;
  sp.error = di->error_word;
  if ((rc = launch_schedule(sp, st))) return rc;

  F32Params prm;
  prm.q = q;
  prm.k = k;
  prm.v = v;
  prm.cu_q = cu_seqlens_q;
  prm.cu_k = cu_seqlens_k;
  prm.qblocks_max = (int)qblocks;
  prm.total_q = total_q;
  prm.n_heads = n_heads;
  prm.group = n_heads / n_kv_heads;
  prm.scale = softmax_scale;
  prm.causal = a.causal;
  prm.bias_key = bias_per_key;
  prm.bias_pair = bias_pair;
  prm.sb = bias_stride_b;
  prm.sh = bias_stride_h;
  prm.bias_head_div = 1;
  prm.sr = bias_stride_q;
  prm.sc = bias_stride_k;
  prm.out = out;
  prm.lse = lse;
  prm.valid = ws.count;
  dim3 grid((unsigned)(batch * qblocks), (unsigned)n_heads);
  if (t_ev_start && t_ev_stop) {
    cudaError_t e = cudaEventRecord(t_ev_start, st);
    if (e != cudaSuccess) return cuda_fail("cudaEventRecord(start)", e);
  }
  if (head_dim == 64) {
    static thread_local int cfg = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (cfg != dev && (rc = set_smem(attn_fwd_f32<64>, F32Cfg<64>::kSmemBytes))) return rc;
    cfg = dev;
    attn_fwd_f32<64><<<grid, kF32Threads, F32Cfg<64>::kSmemBytes, st>>>(prm);
  } else {
    static thread_local int cfg = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (cfg != dev && (rc = set_smem(attn_fwd_f32<128>, F32Cfg<128>::kSmemBytes))) return rc;
    cfg = dev;
    attn_fwd_f32<128><<<grid, kF32Threads, F32Cfg<128>::kSmemBytes, st>>>(prm);
  }
  if ((rc = check_launch("launch attn_fwd_f32"))) return rc;
  if (t_ev_start && t_ev_stop) {
    cudaError_t e = cudaEventRecord(t_ev_stop, st);
    if (e != cudaSuccess) return cuda_fail("cudaEventRecord(stop)", e);
  }
  return VARLEN_ATTN_OK;
}

int varlen_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                            int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                            int n_heads, int n_kv_heads, int head_dim, float softmax_scale,
                            int causal, const float* bias_per_key, const float* bias_pair,
                            int64_t bias_stride_b, int64_t bias_stride_h, int64_t bias_stride_q,
                            int64_t bias_stride_k, void* out, float* lse, void* stream) {
  return fwd_bf16(q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q,
                  max_seqlen_k, n_heads, n_kv_heads, head_dim, softmax_scale, causal, bias_per_key,
                  bias_pair, bias_stride_b, bias_stride_h, bias_stride_q, bias_stride_k, 0u, out,
                  lse, stream, /*fixed_scratch=*/true);
}

const char* varlen_attn_strerror(int status) {
  switch (status) {
    case VARLEN_ATTN_OK: return "ok";
    case VARLEN_ATTN_ERR_NULL_POINTER: return "a required pointer is NULL";
    case VARLEN_ATTN_ERR_BAD_SHAPE: return "batch, heads, totals or max lengths out of range";
    case VARLEN_ATTN_ERR_GQA_MISMATCH: return "n_heads is not a multiple of n_kv_heads";
    case VARLEN_ATTN_ERR_HEAD_DIM: return "head_dim must be 64 or 128";
    case VARLEN_ATTN_ERR_MISALIGNED: return "q/k/v/out must be 16-byte aligned, lse/bias/cu_seqlens 4-byte aligned";
    case VARLEN_ATTN_ERR_BAD_BIAS: return "bias strides must be non-negative";
    case VARLEN_ATTN_ERR_CUDA: return "a CUDA call failed";
    case VARLEN_ATTN_ERR_DEVICE: return "current device is not sm_100 (B200 class)";
    case VARLEN_ATTN_ERR_BAD_SEQLENS: return "cu_seqlens content is invalid (device check)";
    case VARLEN_ATTN_ERR_DEVICE_TIMEOUT: return "a bounded wait in the kernel expired";
    case VARLEN_ATTN_ERR_TOO_LARGE: return "sizes exceed 32-bit indexing";
    case VARLEN_ATTN_ERR_SCRATCH_LIMIT:
      return "work list exceeds the fixed scratch of varlen_attn_fwd_noalloc";
    default: return "unknown status";
  }
}

int varlen_mask_to_seqlens(const uint8_t* mask, int batch, int seqlen, int32_t* cu_seqlens,
                           int32_t* indices, int32_t* max_seqlen, void* stream) {
  if (!mask || !cu_seqlens || !indices || !max_seqlen) return VARLEN_ATTN_ERR_NULL_POINTER;
  if (batch <= 0 || seqlen <= 0) return VARLEN_ATTN_ERR_BAD_SHAPE;
  if ((int64_t)batch * seqlen > INT32_MAX) return VARLEN_ATTN_ERR_TOO_LARGE;
  if (!aligned(cu_seqlens, 4) || !aligned(indices, 4) || !aligned(max_seqlen, 4))
    return VARLEN_ATTN_ERR_MISALIGNED;
  DeviceInfo* di = nullptr;
  if (int rc = device_info(&di)) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  mask_count_kernel<<<batch, kLayoutThreads, 0, st>>>(mask, seqlen, cu_seqlens + 1);
  if (int rc = check_launch("launch mask_count_kernel")) return rc;
  seqlens_scan_kernel<<<1, kLayoutThreads, 0, st>>>(cu_seqlens, batch, max_seqlen);
  if (int rc = check_launch("launch seqlens_scan_kernel")) return rc;
  mask_indices_kernel<<<batch, kLayoutThreads, 0, st>>>(mask, seqlen, cu_seqlens, indices);
  return check_launch("launch mask_indices_kernel");
}


int varlen_gather_rows(const void* src, int64_t src_rows, int64_t row_bytes,
                       const int32_t* indices, const int32_t* cu_seqlens, int batch, void* dst,
                       int64_t dst_rows, void* stream) {
  if (int rc = rows_args_ok(src, src_rows, row_bytes, indices, cu_seqlens, batch, dst, dst_rows))
    return rc;
  DeviceInfo* di = nullptr;
  if (int rc = device_info(&di)) return rc;
  const int64_t units = row_bytes / 16;
  gather_rows_kernel<<<layout_grid(di, dst_rows * units), kLayoutThreads, 0,
                       static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src), src_rows, units, indices, cu_seqlens, batch,
      static_cast<uint4*>(dst), dst_rows, di->error_word);
  return check_launch("launch gather_rows_kernel");
}

int varlen_scatter_rows(const void* src, int64_t src_rows, int64_t row_bytes,
                        const int32_t* indices, const int32_t* cu_seqlens, int batch, void* dst,
                        int64_t dst_rows, void* stream) {
  if (int rc = rows_args_ok(src, src_rows, row_bytes, indices, cu_seqlens, batch, dst, dst_rows))
    return rc;
  DeviceInfo* di = nullptr;
  if (int rc = device_info(&di)) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(dst, 0, (size_t)(dst_rows * row_bytes), st);
  if (e != cudaSuccess) return cuda_fail("cudaMemsetAsync(padded rows)", e);
  const int64_t units = row_bytes / 16;
  scatter_rows_kernel<<<layout_grid(di, src_rows * units), kLayoutThreads, 0, st>>>(
      static_cast<const uint4*>(src), src_rows, units, indices, cu_seqlens, batch,
      static_cast<uint4*>(dst), dst_rows, di->error_word);
  return check_launch("launch scatter_rows_kernel");
}

int varlen_fold_pair_bias_row(const float* bias_pair, int64_t bias_stride_b,
                              int64_t bias_stride_h, int64_t bias_stride_q, int64_t bias_stride_k,
                              int row, int head_div, const int32_t* cu_seqlens_k, int batch,
                              int total_k, int n_heads, const float* bias_in, float* bias_out,
                              void* stream) {
  if (!bias_pair || !cu_seqlens_k || !bias_out) return VARLEN_ATTN_ERR_NULL_POINTER;
  if (batch <= 0 || total_k < 0 || n_heads <= 0 || head_div <= 0 || row < 0)
    return VARLEN_ATTN_ERR_BAD_SHAPE;
  if (bias_stride_b < 0 || bias_stride_h < 0 || bias_stride_q < 0 || bias_stride_k < 0)
    return VARLEN_ATTN_ERR_BAD_BIAS;
  if ((int64_t)total_k * n_heads > INT32_MAX) return VARLEN_ATTN_ERR_TOO_LARGE;
  if (!aligned(bias_pair, 4) || !aligned(bias_out, 4) || (bias_in && !aligned(bias_in, 4)) ||
      !aligned(cu_seqlens_k, 4))
    return VARLEN_ATTN_ERR_MISALIGNED;
  DeviceInfo* di = nullptr;
  if (int rc = device_info(&di)) return rc;
  fold_pair_row_kernel<<<layout_grid(di, (int64_t)total_k * n_heads), kLayoutThreads, 0,
                         static_cast<cudaStream_t>(stream)>>>(
      bias_pair, bias_stride_b, bias_stride_h, bias_stride_q, bias_stride_k, row, head_div,
      cu_seqlens_k, batch, total_k, n_heads, bias_in, bias_out, di->error_word);
  return check_launch("launch fold_pair_row_kernel");
}

int varlen_attn_decode(const void* q, const int32_t* cu_seqlens_q, int batch, int total_q,
                       int max_seqlen_q, void* k_cache, void* v_cache, int cache_len,
                       const int32_t* cache_seqlens, const void* k_new, const void* v_new,
                       int n_heads, int n_kv_heads, int head_dim, float softmax_scale,
                       int causal, int num_splits, void* out, float* lse, void* stream) {
  if (!q || !cu_seqlens_q || !k_cache || !v_cache || !cache_seqlens || !out)
    return VARLEN_ATTN_ERR_NULL_POINTER;
  if ((k_new == nullptr) != (v_new == nullptr)) return VARLEN_ATTN_ERR_NULL_POINTER;
  if (batch <= 0 || batch > 65535 || total_q < 0 || max_seqlen_q < 0 || cache_len <= 0 ||
      n_heads <= 0 || n_kv_heads <= 0 || num_splits < 0 || num_splits > 256)
    return VARLEN_ATTN_ERR_BAD_SHAPE;
  if (n_heads % n_kv_heads != 0) return VARLEN_ATTN_ERR_GQA_MISMATCH;
  if (head_dim != 64 && head_dim != 128) return VARLEN_ATTN_ERR_HEAD_DIM;
  const int G = n_heads / n_kv_heads;
  if ((int64_t)max_seqlen_q * G > kDecMaxRows) return VARLEN_ATTN_ERR_BAD_SHAPE;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      (k_new && (!aligned(k_new, 16) || !aligned(v_new, 16))) || (lse && !aligned(lse, 4)) ||
      !aligned(cu_seqlens_q, 4) || !aligned(cache_seqlens, 4))
    return VARLEN_ATTN_ERR_MISALIGNED;
  if ((int64_t)total_q * n_heads * head_dim > INT32_MAX ||
      (int64_t)batch * cache_len * n_kv_heads * head_dim / 8 > INT32_MAX)
    return VARLEN_ATTN_ERR_TOO_LARGE;
  DeviceInfo* di = nullptr;
  if (int rc = device_info(&di)) return rc;
  if (total_q == 0 || max_seqlen_q == 0) return VARLEN_ATTN_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // splits: fixed ranges of split_blocks key blocks of the cache, so that
  // every CTA streams about the same number of keys whatever its sequence's
  // length (the grid then ends without a tail of long CTAs). Automatic count:
  // splits of at most 1536 keys (smaller ones measured slower: each CTA's
  // set-up, merge and partial output cost more than the shorter tail saves),
  // and about 16 CTAs per SM over the whole grid when that asks for more,
  // each split at least 256 keys.
  int splits = num_splits;
  const int max_blocks = (cache_len + kDecKeys - 1) / kDecKeys;
  if (splits == 0) {
    const int64_t ctas = (int64_t)batch * n_kv_heads;
    const int64_t want = (16 * (int64_t)di->sm_count + ctas - 1) / ctas;
    const int64_t by_size = (max_blocks + 1536 / kDecKeys - 1) / (1536 / kDecKeys);
    const int min_blocks = (256 + kDecKeys - 1) / kDecKeys;
    splits = (int)std::max<int64_t>(
        1, std::min<int64_t>(std::max(want, by_size), std::max(1, max_blocks / min_blocks)));
  }
  splits = std::min(splits, std::max(1, max_blocks));
  const int split_blocks = (max_blocks + splits - 1) / splits;
  splits = (max_blocks + split_blocks - 1) / split_blocks;  // no split starts past the cache
  DecodeParams dp;
  dp.q = static_cast<const __nv_bfloat16*>(q);
  dp.cu_q = cu_seqlens_q;
  dp.k_cache = static_cast<__nv_bfloat16*>(k_cache);
  dp.v_cache = static_cast<__nv_bfloat16*>(v_cache);
  dp.cache_seqlens = cache_seqlens;
  dp.k_new = static_cast<const __nv_bfloat16*>(k_new);
  dp.v_new = static_cast<const __nv_bfloat16*>(v_new);
  dp.batch = batch;
  dp.total_q = total_q;
  dp.cache_len = cache_len;
  dp.n_heads = n_heads;
  dp.n_kv_heads = n_kv_heads;
  dp.group = G;
  dp.causal = causal ? 1 : 0;
  dp.n_splits = splits;
  dp.split_blocks = split_blocks;
  dp.scale_log2 = softmax_scale * 1.4426950408889634f;
  dp.out = static_cast<__nv_bfloat16*>(out);
  dp.lse = lse;
  dp.part_o = nullptr;
  dp.part_lse = nullptr;
  dp.error = di->error_word;
  const dim3 grid(splits, n_kv_heads, batch);
  const int rows = (int)std::min<int64_t>((int64_t)total_q * n_heads / (kDecThreads / 32) + 1,
                                          (int64_t)di->sm_count * 16);
  if (k_new) {
    const int units = n_kv_heads * head_dim / 8;
    if (head_dim == 64)
      decode_append_kernel<64><<<layout_grid(di, (int64_t)total_q * units), kDecThreads, 0, st>>>(dp);
    else
      decode_append_kernel<128><<<layout_grid(di, (int64_t)total_q * units), kDecThreads, 0, st>>>(dp);
    if (int rc = check_launch("launch decode_append_kernel")) return rc;
  }
  const int rows_needed = max_seqlen_q * G;
  if (num_splits == 0) {
    // On the tensor cores, through the packed forward kernel with the K/V
    // read in place from the cache and the rows of all G query heads of a
    // K/V group in one tile (token-major: row = token * G + head in group),
    // longest first. (With several query rows per K/V head the CUDA-core
    // kernels below are bound by their fp32 multiply-adds; with one, both
    // are bound by HBM.) With enough (sequence, K/V head) pairs to fill the
    // GPU, one work item per pair; with fewer, each sequence's keys are cut
    // into fixed ranges of the cache, one work item per (range, pair), whose
    // outputs the split-combine kernel merges by LSE. The ranges are sized
    // for about kRangeItemsPerSm items per SM were every sequence at
    // cache_len (the lengths are on the device), and hold at least
    // kMinRangeKeys keys.
    const int64_t pairs = (int64_t)batch * n_kv_heads;
    int ranges = 1, range_keys = 0;
    if (pairs < di->sm_count) {
      const int64_t want = (kRangeItemsPerSm * (int64_t)di->sm_count + pairs - 1) / pairs;
      const int most = std::max(1, cache_len / kMinRangeKeys);
      ranges = (int)std::min<int64_t>(want, std::min(most, kMaxRanges));
      range_keys = ceil_div(ceil_div(cache_len, ranges), BN) * BN;
      ranges = ceil_div(cache_len, range_keys);  // no range starts past the cache
      if (ranges <= 1) {
        ranges = 1;
        range_keys = 0;
      }
    }
    const int cap = batch * ranges;  // list entries: (sequence, range) pairs
    const size_t list_bytes = (256 + 2 * (size_t)cap * sizeof(int2) + 255) / 256 * 256;
    const size_t po = ranges > 1 ? (size_t)ranges * total_q * n_heads * head_dim * sizeof(float) : 0;
    const size_t pl = ranges > 1 ? (size_t)ranges * n_heads * total_q * sizeof(float) : 0;
    const int box_tok = BM / G;  // tokens of one Q tile load
    CUtensorMap tq, tk, tv;
    if (!make_tmap_box(&tq, q, head_dim, n_heads, total_q, G, box_tok) ||
        !make_tmap(&tk, k_cache, head_dim, n_kv_heads, batch * cache_len, BN) ||
        !make_tmap(&tv, v_cache, head_dim, n_kv_heads, batch * cache_len, BN))
      return VARLEN_ATTN_ERR_CUDA;
    void* wsp = nullptr;
    if (int rc = workspace(stream, list_bytes + po + pl, &wsp)) return rc;
    Workspace ws = carve(wsp, cap);
    float* part_o = ranges > 1 ? reinterpret_cast<float*>(static_cast<char*>(wsp) + list_bytes) : nullptr;
    float* part_lse = ranges > 1 ? reinterpret_cast<float*>(static_cast<char*>(wsp) + list_bytes + po) : nullptr;
    SchedParams sp;
    std::memset(&sp, 0, sizeof sp);
    sp.cu_q = cu_seqlens_q;
    sp.batch = batch;
    sp.total_q = total_q;
    sp.total_k = batch * cache_len;
    sp.max_q = max_seqlen_q;
    sp.max_k = cache_len;
    sp.causal = causal ? 1 : 0;
    sp.pairing = kPackGQA;
    sp.group = G;
    sp.n_hg = n_kv_heads;
    sp.cache_seqlens = cache_seqlens;
    sp.cache_len = cache_len;
    sp.cache_extra = k_new != nullptr;
    sp.cache_ranges = ranges;
    sp.range_keys = range_keys;
    sp.ws = ws;
    sp.error = di->error_word;
    if (int rc = launch_schedule(sp, st)) return rc;
    AttnParams prm;
    std::memset(&prm, 0, sizeof prm);
    prm.cu_q = cu_seqlens_q;
    prm.total_q = total_q;
    prm.n_heads = n_heads;
    prm.n_kv_heads = n_kv_heads;
    prm.group = G;
    prm.pairing = kPackGQA;
    prm.n_hg = n_kv_heads;
    prm.causal = causal ? 1 : 0;
    prm.scale_log2 = softmax_scale * 1.4426950408889634f;
    prm.scale = softmax_scale;
    prm.bias_head_div = 1;
    prm.out = out;
    prm.lse = lse;
    prm.ws = ws;
    prm.error = di->error_word;
    prm.wait_limit = wait_limit();
    prm.test_stall = g_test_stall.load(std::memory_order_relaxed);
    prm.cache_seqlens = cache_seqlens;
    prm.cache_len = cache_len;
    prm.cache_extra = k_new != nullptr;
    prm.q_box_rows = G * box_tok;
    prm.cache_ranges = ranges;
    prm.range_keys = range_keys;
    prm.part_o = part_o;
    prm.part_lse = part_lse;
    const int64_t items = pairs * ranges;
    const int grid = (int)(items < di->sm_count ? items : di->sm_count);
    int rc = head_dim == 64 ? launch_attn<64, false, false, true>(grid, tq, tk, tv, prm, st)
                            : launch_attn<128, false, false, true>(grid, tq, tk, tv, prm, st);
    if (!rc && ranges > 1) {
      dp.n_splits = ranges;
      dp.part_o = part_o;
      dp.part_lse = part_lse;
      if (head_dim == 64) decode_combine_kernel<64><<<rows, kDecThreads, 0, st>>>(dp);
      else decode_combine_kernel<128><<<rows, kDecThreads, 0, st>>>(dp);
      rc = check_launch("launch decode_combine_kernel");
    }
    return rc;
  }
  if (splits > 1) {
    const size_t po = (size_t)splits * total_q * n_heads * head_dim * sizeof(float);
    const size_t pl = (size_t)splits * n_heads * total_q * sizeof(float);
    void* wsp = nullptr;
    if (int rc = workspace(stream, po + pl, &wsp)) return rc;
    dp.part_o = static_cast<float*>(wsp);
    dp.part_lse = reinterpret_cast<float*>(static_cast<char*>(wsp) + po);
  }
  const int RT = rows_needed <= 4 ? 4 : rows_needed <= 8 ? 8 : rows_needed <= 16 ? 16 : 32;
  int rc = VARLEN_ATTN_OK;
  if (RT <= kDec2MaxRows) {
    // up to 16 rows per K/V head: TMA ring, warp-owned key blocks
    CUtensorMap tk, tv;
    const int cache_rows = batch * cache_len;
    if (!make_tmap(&tk, k_cache, head_dim, n_kv_heads, cache_rows, kDecKeys) ||
        !make_tmap(&tv, v_cache, head_dim, n_kv_heads, cache_rows, kDecKeys))
      return VARLEN_ATTN_ERR_CUDA;
    if (head_dim == 64)
      rc = RT == 4 ? launch_decode_tma<64, 4>(grid, tk, tv, dp, st)
           : RT == 8 ? launch_decode_tma<64, 8>(grid, tk, tv, dp, st)
                     : launch_decode_tma<64, 16>(grid, tk, tv, dp, st);
    else
      rc = RT == 4 ? launch_decode_tma<128, 4>(grid, tk, tv, dp, st)
           : RT == 8 ? launch_decode_tma<128, 8>(grid, tk, tv, dp, st)
                     : launch_decode_tma<128, 16>(grid, tk, tv, dp, st);
    if (!rc && splits > 1) {
      if (head_dim == 64) decode_combine_kernel<64><<<rows, kDecThreads, 0, st>>>(dp);
      else decode_combine_kernel<128><<<rows, kDecThreads, 0, st>>>(dp);
    }
  } else if (head_dim == 64) {
    switch (RT) {
      case 4: rc = launch_decode<64, 4>(grid, dp, st); break;
      case 8: rc = launch_decode<64, 8>(grid, dp, st); break;
      case 16: rc = launch_decode<64, 16>(grid, dp, st); break;
      default: rc = launch_decode<64, 32>(grid, dp, st); break;
    }
    if (!rc && splits > 1) decode_combine_kernel<64><<<rows, kDecThreads, 0, st>>>(dp);
  } else {
    switch (RT) {
      case 4: rc = launch_decode<128, 4>(grid, dp, st); break;
      case 8: rc = launch_decode<128, 8>(grid, dp, st); break;
      case 16: rc = launch_decode<128, 16>(grid, dp, st); break;
      default: rc = launch_decode<128, 32>(grid, dp, st); break;
    }
    if (!rc && splits > 1) decode_combine_kernel<128><<<rows, kDecThreads, 0, st>>>(dp);
  }
  if (rc) return rc;
  return check_launch("launch decode_combine_kernel");
}

int varlen_attn_get_device_error(void* stream) {
  DeviceInfo* di = nullptr;
  int rc = device_info(&di);
  if (rc) return rc;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail("cudaStreamSynchronize", e);
  int v = 0;
  if ((e = cudaMemcpy(&v, di->error_word, sizeof v, cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail("cudaMemcpy(error word)", e);
  const int zero = 0;
  if ((e = cudaMemcpy(di->error_word, &zero, sizeof zero, cudaMemcpyHostToDevice)) != cudaSuccess)
    return cuda_fail("cudaMemcpy(error word reset)", e);
  return v;
}

int varlen_attn_set_profile_events(void* start_event, void* stop_event) {
  t_ev_start = static_cast<cudaEvent_t>(start_event);
  t_ev_stop = static_cast<cudaEvent_t>(stop_event);
  return VARLEN_ATTN_OK;
}

int varlen_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                    const float* lse, const void* dout, const int32_t* cu_seqlens_q,
                    const int32_t* cu_seqlens_k, int batch, int total_q, int total_k,
                    int max_seqlen_q, int max_seqlen_k, int n_heads, int n_kv_heads,
                    int head_dim, float softmax_scale, int causal, const float* bias_per_key,
                    const float* bias_pair, int64_t bias_stride_b, int64_t bias_stride_h,
                    int64_t bias_stride_q, int64_t bias_stride_k, unsigned flags, void* dq,
                    void* dk, void* dv, float* dbias_per_key, float* dbias_pair,
                    int64_t dbias_stride_b, int64_t dbias_stride_h, int64_t dbias_stride_q,
                    void* stream) {
  if (flags & ~(unsigned)VARLEN_ATTN_BIAS_PAIR_KV_HEADS) return VARLEN_ATTN_ERR_BAD_BIAS;
  Common a{batch, total_q, total_k, max_seqlen_q, max_seqlen_k, n_heads, n_kv_heads, head_dim,
           causal ? 1 : 0, cu_seqlens_q, cu_seqlens_k, bias_per_key, bias_pair, bias_stride_b,
           bias_stride_h, bias_stride_q, bias_stride_k};
  int rc = validate_common(a, q, k, v, out, lse);
  if (rc) return rc;
  if (!lse || !dout || !dq) return VARLEN_ATTN_ERR_NULL_POINTER;
  if (total_k > 0 && (!dk || !dv)) return VARLEN_ATTN_ERR_NULL_POINTER;
  if (!aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
      (dbias_per_key && !aligned(dbias_per_key, 4)) || (dbias_pair && !aligned(dbias_pair, 4)))
    return VARLEN_ATTN_ERR_MISALIGNED;
  if (dbias_pair && (dbias_stride_b < 0 || dbias_stride_h < 0 || dbias_stride_q < 0))
    return VARLEN_ATTN_ERR_BAD_BIAS;
  if (batch > 65535 || n_heads > 65535) return VARLEN_ATTN_ERR_TOO_LARGE;
  DeviceInfo* di = nullptr;
  if ((rc = device_info(&di))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (total_q == 0 && total_k == 0) return VARLEN_ATTN_OK;

  // workspace: schedule header (validation result) + delta [Hq, Tq]
  void* wsp = nullptr;
  const size_t delta_bytes = (size_t)n_heads * (size_t)(total_q > 0 ? total_q : 1) * 4;
  if ((rc = workspace(stream, 256 + 2 * sizeof(int2) + delta_bytes, &wsp))) return rc;
  Workspace ws = carve(wsp, 1);
  float* delta = reinterpret_cast<float*>(static_cast<char*>(wsp) + 256 + 2 * sizeof(int2));

  SchedParams sp;
  std::memset(&sp, 0, sizeof sp);  // no K/V cache
  sp.cu_q = cu_seqlens_q;
  sp.cu_k = cu_seqlens_k;
  sp.batch = batch;
  sp.total_q = total_q;
  sp.total_k = total_k;
  sp.max_q = max_seqlen_q;
  sp.max_k = max_seqlen_k;
  sp.causal = a.causal;
  sp.pairing = -1;  // validate only: count = 1 when the boundaries are sound, else 0
  sp.n_hg = 1;
  sp.ws = ws;
  sp.error = di->error_word;
  if ((rc = launch_schedule(sp, st))) return rc;

  if (total_q > 0) {
    const long long n = (long long)total_q * n_heads;
    const int blocks = (int)std::min<long long>((n + 255) / 256, (long long)di->sm_count * 8);
    if (head_dim == 64)
      bwd_delta_kernel<64><<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(out),
                                                   static_cast<const __nv_bfloat16*>(dout),
                                                   total_q, n_heads, delta);
    else
      bwd_delta_kernel<128><<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(out),
                                                    static_cast<const __nv_bfloat16*>(dout),
                                                    total_q, n_heads, delta);
    if ((rc = check_launch("bwd_delta_kernel"))) return rc;
  }

  CUtensorMap tq, tk, tv, tdo;
  if (!make_tmap(&tq, q, head_dim, n_heads, total_q, BM) ||
      !make_tmap(&tdo, dout, head_dim, n_heads, total_q, BM) ||
      !make_tmap(&tk, kv_base(k, q, total_k), head_dim, n_kv_heads, total_k, BN) ||
      !make_tmap(&tv, kv_base(v, q, total_k), head_dim, n_kv_heads, total_k, BN))
    return VARLEN_ATTN_ERR_CUDA;

  if (dbias_per_key) {  // the dK/dV kernel adds two half sums per (key, head)
    cudaError_t e = cudaMemsetAsync(dbias_per_key, 0, (size_t)total_k * n_heads * 4, st);
    if (e != cudaSuccess) return cuda_fail("cudaMemsetAsync(dbias_per_key)", e);
  }
  BwdParams bp;
  bp.cu_q = cu_seqlens_q;
  bp.cu_k = cu_seqlens_k;
  bp.valid = ws.count;
  bp.total_q = total_q;
  bp.total_k = total_k;
  bp.n_heads = n_heads;
  bp.n_kv_heads = n_kv_heads;
  bp.group = n_heads / n_kv_heads;
  bp.causal = a.causal;
  bp.scale = softmax_scale;
  bp.lse = lse;
  bp.delta = delta;
  bp.bias_key = bias_per_key;
  bp.bias_pair = bias_pair;
  bp.sb = bias_stride_b;
  bp.sh = bias_stride_h;
  bp.sr = bias_stride_q;
  bp.sc = bias_stride_k;
  bp.bias_head_div = (flags & VARLEN_ATTN_BIAS_PAIR_KV_HEADS) ? bp.group : 1;
  bp.dbias_key = dbias_per_key;
  bp.dbias_pair = dbias_pair;
  bp.dsb = dbias_stride_b;
  bp.dsh = dbias_stride_h;
  bp.dsr = dbias_stride_q;
  bp.dq = dq;
  bp.dk = dk;
  bp.dv = dv;
  bp.error = di->error_word;
  bp.wait_limit = wait_limit();
  bp.test_stall = g_test_stall.load(std::memory_order_relaxed);
  const dim3 grid_a((unsigned)std::max(1, ceil_div(max_seqlen_k, BN)), (unsigned)n_kv_heads,
                    (unsigned)batch);
  const dim3 grid_q((unsigned)std::max(1, ceil_div(max_seqlen_q, BM)), (unsigned)n_heads,
                    (unsigned)batch);
  const bool bk = bias_per_key != nullptr, bpr = bias_pair != nullptr;
  if (head_dim == 64) {
    if (bk && bpr) rc = launch_bwd<64, true, true>(grid_a, grid_q, tq, tk, tv, tdo, bp, st);
    else if (bk) rc = launch_bwd<64, true, false>(grid_a, grid_q, tq, tk, tv, tdo, bp, st);
    else if (bpr) rc = launch_bwd<64, false, true>(grid_a, grid_q, tq, tk, tv, tdo, bp, st);
    else rc = launch_bwd<64, false, false>(grid_a, grid_q, tq, tk, tv, tdo, bp, st);
  } else {
    if (bk && bpr) rc = launch_bwd<128, true, true>(grid_a, grid_q, tq, tk, tv, tdo, bp, st);
    else if (bk) rc = launch_bwd<128, true, false>(grid_a, grid_q, tq, tk, tv, tdo, bp, st);
    else if (bpr) rc = launch_bwd<128, false, true>(grid_a, grid_q, tq, tk, tv, tdo, bp, st);
    else rc = launch_bwd<128, false, false>(grid_a, grid_q, tq, tk, tv, tdo, bp, st);
  }
  return rc;
}

int varlen_attn_set_wait_limit(long long cycles) {
  if (cycles < 0) return VARLEN_ATTN_ERR_BAD_SHAPE;
  g_wait_limit.store(cycles, std::memory_order_relaxed);
  return VARLEN_ATTN_OK;
}

int varlen_attn_set_test_stall(int on) {
  g_test_stall.store(on ? 1 : 0, std::memory_order_relaxed);
  return VARLEN_ATTN_OK;
}

int varlen_attn_launches_per_call(int fp32_path) {
  (void)fp32_path;
  return 2;  // schedule (or validation) kernel + attention kernel
}

int varlen_attn_version(void) { return kVersion; }

const char* varlen_attn_last_error_detail(void) { return t_detail; }

}  // extern "C"
