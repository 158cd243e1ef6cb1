// C-ABI entry points for paged decode attention: argument validation, kernel
// selection, TMA descriptor encoding and launch (see include/pagedkv.h).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <memory>
#include <mutex>
#include <queue>
#include <utility>
#include <vector>

#include "decode_dispatch.h"
#include "decode_kernel.cuh"
#include "pa_internal.h"
#include "prefill_kernel.cuh"
#include "prefix_kernel.cuh"

namespace pagedkv {
namespace {

constexpr size_t kWorkspaceHeader = 256;
constexpr int64_t kDeepContextTokens = 32768;
constexpr int kMaxSplitSeqs = 4096;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elt_bytes(pa_dtype_t dt) { return dt == PA_F32 ? 4 : 2; }

// ---- cuTensorMapEncodeTiled through the runtime's driver entry point ----------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// A pool [num_blocks][num_kv_heads][block_size][head_dim] viewed as a 2-D
// tensor of rows = num_blocks*num_kv_heads*block_size, cols = head_dim; one
// box = 16 rows x 128 bytes, 128-byte swizzle.
struct MapKey {
  const void* base;
  int rows;
  int head_dim;
  int block_size;
  pa_dtype_t dtype;
  bool operator==(const MapKey& o) const {
    return base == o.base && rows == o.rows && head_dim == o.head_dim &&
           block_size == o.block_size && dtype == o.dtype;
  }
};

struct MapCache {
  static constexpr int kSlots = 8;
  MapKey key[kSlots];
  CUtensorMap map[kSlots];
  int used = 0;
  int next = 0;
};

pa_status_t pool_tensor_map(const void* base, int rows, int head_dim, int block_size,
                            pa_dtype_t dtype, CUtensorMap* out) {
  thread_local MapCache cache;
  const MapKey k{base, rows, head_dim, block_size, dtype};
  for (int i = 0; i < cache.used; ++i) {
    if (cache.key[i] == k) {
      *out = cache.map[i];
      return PA_OK;
    }
  }
  auto fn = encode_fn();
  if (fn == nullptr) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const int eb = elt_bytes(dtype);
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(head_dim) * eb};
  // One box = one 16-token pipeline unit x 128 bytes (block sizes 16 and 32
  // are both multiples of it).
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / eb), 16u};
  cuuint32_t estr[2] = {1, 1};
  CUtensorMap m;
  std::memset(&m, 0, sizeof(m));
  CUresult r = fn(&m, dtype == PA_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                  2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  const int slot = cache.used < MapCache::kSlots ? cache.used++ : (cache.next++ % MapCache::kSlots);
  cache.key[slot] = k;
  cache.map[slot] = m;
  *out = m;
  return PA_OK;
}

// q [total_q][num_q_heads][head_dim] (bf16) as a 3-D tensor (head_dim,
// heads, tokens); one box = 64 columns x `group` heads x `tokens` tokens,
// 128-byte swizzle: the query rows of one KV head for a run of tokens.
struct QKey {
  const void* q;
  int total_q, heads, head_dim, group, tokens;
};

struct QCache {
  static constexpr int kSlots = 8;
  QKey key[kSlots];
  CUtensorMap map[kSlots];
  int used = 0, next = 0;
};

pa_status_t q_tensor_map(const void* q, int total_q, int num_q_heads, int head_dim, int group,
                         int tokens, CUtensorMap* out) {
  thread_local QCache cache;
  for (int i = 0; i < cache.used; ++i) {
    const QKey& k = cache.key[i];
    if (k.q == q && k.total_q == total_q && k.heads == num_q_heads && k.head_dim == head_dim &&
        k.group == group && k.tokens == tokens) {
      *out = cache.map[i];
      return PA_OK;
    }
  }
  auto fn = encode_fn();
  if (fn == nullptr) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_q_heads),
                        static_cast<cuuint64_t>(total_q)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                           static_cast<cuuint64_t>(num_q_heads) * head_dim * 2};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(tokens)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUtensorMap m;
  std::memset(&m, 0, sizeof(m));
  CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled (q) failed (%d)", static_cast<int>(r));
  const int slot = cache.used < QCache::kSlots ? cache.used++ : (cache.next++ % QCache::kSlots);
  cache.key[slot] = QKey{q, total_q, num_q_heads, head_dim, group, tokens};
  cache.map[slot] = m;
  *out = m;
  return PA_OK;
}

struct DecodeReq {
  const void* q;
  const void* k_pool;
  const void* v_pool;
  const int32_t* block_tables;
  const int32_t* context_lens;
  int num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq;
  float scale;
  pa_dtype_t dtype;
  void* out;
  uint32_t* dev_err;
  cudaStream_t stream;
};

pa_status_t validate_and_pick(const DecodeReq& r, DecodeInstance* inst) {
  if (r.num_seqs < 0) return fail(PA_ERR_INVALID_ARG, "num_seqs < 0");
  if (r.q == nullptr || r.k_pool == nullptr || r.v_pool == nullptr || r.block_tables == nullptr ||
      r.context_lens == nullptr || r.out == nullptr)
    return fail(PA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (r.num_q_heads <= 0 || r.num_kv_heads <= 0 || r.num_q_heads % r.num_kv_heads != 0)
    return fail(PA_ERR_INVALID_ARG, "num_q_heads (%d) must be a positive multiple of num_kv_heads (%d)",
                r.num_q_heads, r.num_kv_heads);
  if (r.num_blocks <= 0 || r.max_blocks_per_seq <= 0)
    return fail(PA_ERR_INVALID_ARG, "num_blocks and max_blocks_per_seq must be positive");
  if (r.dtype != PA_F32 && r.dtype != PA_BF16) return fail(PA_ERR_INVALID_ARG, "unknown dtype");
  if (!std::isfinite(r.scale)) return fail(PA_ERR_INVALID_ARG, "scale is not finite");
  if (!aligned16(r.q) || !aligned16(r.k_pool) || !aligned16(r.v_pool) || !aligned16(r.out))
    return fail(PA_ERR_INVALID_ARG, "q, pools and out must be 16-byte aligned");
  const int64_t rows = static_cast<int64_t>(r.num_blocks) * r.num_kv_heads * r.block_size;
  if (rows >= (int64_t(1) << 31))
    return fail(PA_ERR_INVALID_ARG, "num_blocks * num_kv_heads * block_size must be < 2^31");
  if (static_cast<int64_t>(r.max_blocks_per_seq) * r.block_size >= (int64_t(1) << 31))
    return fail(PA_ERR_INVALID_ARG, "max_blocks_per_seq * block_size must be < 2^31");
  const int group = r.num_q_heads / r.num_kv_heads;
  bool found = false;
  // bf16 runs on tensor cores for every group size, MHA included: measured on
  // B200 (MHA batch 64) the mma path streams 6.0 TB/s where the CUDA-core
  // path reaches 4.5 TB/s, whose per-block shuffle chains leave the warps
  // latency-bound. fp32 stays on CUDA cores (exact fp32 products).
  if (r.dtype == PA_F32) {
    found = find_decode_f32(r.head_dim, r.block_size, group, inst);
  } else if (group <= 16) {
    // Tables that can hold 32k tokens or more mark long-context batches: the
    // deeper, narrower CTA shape streams them faster.
    const bool deep = static_cast<int64_t>(r.max_blocks_per_seq) * r.block_size >= kDeepContextTokens;
    found = find_decode_bf16_mma(r.head_dim, r.block_size, deep, inst);
  }
  if (!found)
    return fail(PA_ERR_UNSUPPORTED,
                "no kernel for dtype=%s head_dim=%d block_size=%d group=%d",
                r.dtype == PA_F32 ? "f32" : "bf16", r.head_dim, r.block_size, group);
  return PA_OK;
}

// Optional host-side check of the device tables (PAGEDKV_VALIDATE=1): copies
// block tables and context lengths to the host and checks every entry the
// kernels will read. Synchronous; meant for tests and debugging.
pa_status_t host_validate(const DecodeReq& r) {
  static const bool enabled = [] {
    const char* e = std::getenv("PAGEDKV_VALIDATE");
    return e != nullptr && e[0] == '1';
  }();
  if (!enabled || r.num_seqs == 0) return PA_OK;
  std::vector<int32_t> ctx(r.num_seqs);
  std::vector<int32_t> bt(static_cast<size_t>(r.num_seqs) * r.max_blocks_per_seq);
  if (cudaMemcpyAsync(ctx.data(), r.context_lens, ctx.size() * 4, cudaMemcpyDeviceToHost, r.stream) != cudaSuccess ||
      cudaMemcpyAsync(bt.data(), r.block_tables, bt.size() * 4, cudaMemcpyDeviceToHost, r.stream) != cudaSuccess ||
      cudaStreamSynchronize(r.stream) != cudaSuccess)
    return fail(PA_ERR_CUDA, "PAGEDKV_VALIDATE copy failed: %s", cudaGetErrorString(cudaGetLastError()));
  for (int s = 0; s < r.num_seqs; ++s) {
    if (ctx[s] < 0 || static_cast<int64_t>(ctx[s]) > static_cast<int64_t>(r.max_blocks_per_seq) * r.block_size)
      return fail(PA_ERR_INVALID_ARG, "context_lens[%d] = %d out of range", s, ctx[s]);
    const int nb = (ctx[s] + r.block_size - 1) / r.block_size;
    for (int i = 0; i < nb; ++i) {
      const int32_t b = bt[static_cast<size_t>(s) * r.max_blocks_per_seq + i];
      if (b < 0 || b >= r.num_blocks)
        return fail(PA_ERR_INVALID_ARG, "block_tables[%d][%d] = %d out of range", s, i, b);
    }
  }
  return PA_OK;
}

int l2_hint_default() {
  static const int hint = [] {
    const char* e = std::getenv("PAGEDKV_L2_HINT");
    if (e == nullptr) return 1;
    const int v = std::atoi(e);
    return (v >= 0 && v <= 2) ? v : 1;
  }();
  return hint;
}

struct DeviceInfo {
  int sms = 0;
};

pa_status_t device_info(DeviceInfo* info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(PA_ERR_CUDA, "cudaGetDevice failed");
  static std::mutex mu;
  static std::vector<int> sms;
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(sms.size()) <= dev) sms.resize(dev + 1, 0);
  if (sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return fail(PA_ERR_CUDA, "cudaDeviceGetAttribute failed");
    sms[dev] = n;
  }
  info->sms = sms[dev];
  return PA_OK;
}

// Resident CTAs per SM of `kernel` at `threads` x `smem`, queried once per
// (device, kernel, threads, smem): the query costs microseconds of host time
// per call otherwise.
pa_status_t occupancy(const void* kernel, int threads, int smem, int* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(PA_ERR_CUDA, "cudaGetDevice failed");
  struct Entry {
    int dev;
    const void* k;
    int threads, smem, occ;
  };
  static std::mutex mu;
  static std::vector<Entry> cache;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry& e : cache) {
    if (e.dev == dev && e.k == kernel && e.threads == threads && e.smem == smem) {
      *out = e.occ;
      return PA_OK;
    }
  }
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, smem) != cudaSuccess || occ <= 0)
    return fail(PA_ERR_CUDA, "occupancy query failed (smem %d)", smem);
  cache.push_back(Entry{dev, kernel, threads, smem, occ});
  *out = occ;
  return PA_OK;
}

// Raises the kernel's dynamic shared memory limit when needed (per device).
pa_status_t prepare_kernel(const void* kernel, int smem) {
  static std::mutex mu;
  struct Entry {
    int dev;
    const void* k;
    int smem;
  };
  static std::vector<Entry> done;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  for (auto& e : done) {
    if (e.dev == dev && e.k == kernel && e.smem >= smem) return PA_OK;
  }
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess)
    return fail(PA_ERR_CUDA, "cudaFuncSetAttribute(smem=%d): %s", smem, cudaGetErrorString(err));
  done.push_back({dev, kernel, smem});
  return PA_OK;
}

pa_status_t launch_error(const char* what) {
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(err));
  return ok();
}

// Workspace of the split decode:
//   [0, 256)   control header (zero; kept for the workspace contract)
//   pieces     int32 [num_seqs][num_q_heads] (>= one per (sequence, KV head))
//   m, l       float [num_seqs][num_q_heads][pmax]
//   acc        float [num_seqs][num_q_heads][pmax][head_dim]
// pmax bounds the pieces of one (sequence, KV head): a warp takes at least
// partition_tokens of it, so at most ceil(max_blocks_per_seq / pb) + 1.
struct SplitLayout {
  size_t seg_off, m_off, l_off, acc_off, total;
  size_t zero_bytes;  // bytes that must start at zero (the header)
  int pmax;
};

SplitLayout split_layout(int num_seqs, int num_q_heads, int head_dim, int block_size,
                         int max_blocks_per_seq, int partition_tokens) {
  SplitLayout L{};
  const int pb = partition_tokens / block_size;
  L.pmax = (max_blocks_per_seq + pb - 1) / pb + 1;
  const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads * L.pmax;
  L.seg_off = kWorkspaceHeader;
  L.zero_bytes = kWorkspaceHeader;
  L.m_off = L.seg_off + align256(static_cast<size_t>(num_seqs) * num_q_heads * 4);
  L.l_off = L.m_off + align256(rows * 4);
  L.acc_off = L.l_off + align256(rows * 4);
  L.total = L.acc_off + align256(rows * head_dim * 4);
  return L;
}

// Shared-prefix decode hands the split kernel per-sequence skip/base arrays
// and its own partial-array layout.
struct SplitExtras {
  const int32_t* seq_skip_blocks = nullptr;
  const int32_t* seq_part_base = nullptr;
  size_t seg_off = 0, m_off = 0, l_off = 0, acc_off = 0, total = 0;
  int pmax = 0;
  bool after_prefix_kernel = false;  // launched right after the prefix kernel
  int window = 0;                    // sliding window (0 = none)
};

// Which split-decode kernel runs. Measured on B200 (bf16, head_dim 128):
//  * the balanced kernel (every warp an equal run of units, one pass over
//    each warp's range) streams 131072-token contexts at 0.96-0.99 of the
//    measured HBM copy peak against 0.93-0.94 for partition tickets, and a
//    4096-token window over them at 0.51 against 0.41;
//  * partition tickets (each CTA pulls 512-token items; the warps of a CTA
//    split an item) stream MHA batch 64 / GQA batch 256 at 0.94 / 0.93
//    against 0.91 / 0.90, and the shared-prefix suffix pass 10% faster.
// So tables that can hold 32k tokens or more take the balanced kernel, and
// so does the shared-prefix suffix pass, in a smaller CTA shape that fits
// beside the prefix kernel's CTAs (prefix_cow call 75.7 us against 84.0 on
// tickets). PAGEDKV_SPLIT_KERNEL=stream|ticket overrides the choice (tests
// run both).
bool use_stream_kernel(const DecodeReq& r, bool suffix_pass) {
  const char* e = std::getenv("PAGEDKV_SPLIT_KERNEL");
  if (e != nullptr && std::strcmp(e, "stream") == 0) return true;
  if (e != nullptr && std::strcmp(e, "ticket") == 0) return false;
  return suffix_pass ||
         static_cast<int64_t>(r.max_blocks_per_seq) * r.block_size >= kDeepContextTokens;
}

// clear_header: zero the workspace's control header on r.stream right before
// the launch, after every host-side check has passed (a refused call leaves
// the workspace untouched).
pa_status_t run_decode(const DecodeReq& r, bool split, int partition_tokens, void* workspace,
                       size_t workspace_bytes, const SplitExtras* extras = nullptr,
                       bool clear_header = false) {
  DecodeInstance inst;
  pa_status_t st = validate_and_pick(r, &inst);
  if (st != PA_OK) return st;
  if (r.num_seqs == 0) return ok();
  st = host_validate(r);
  if (st != PA_OK) return st;

  DecodeArgs a{};
  a.q = r.q;
  a.out = r.out;
  a.block_tables = r.block_tables;
  a.context_lens = r.context_lens;
  a.dev_err = r.dev_err;
  a.num_seqs = r.num_seqs;
  a.num_q_heads = r.num_q_heads;
  a.num_kv_heads = r.num_kv_heads;
  a.group = r.num_q_heads / r.num_kv_heads;
  a.num_blocks = r.num_blocks;
  a.max_blocks_per_seq = r.max_blocks_per_seq;
  a.scale_log2 = r.scale * 1.4426950408889634f;
  a.l2_hint = l2_hint_default();

  int smem = inst.fixed_smem;
  const void* kernel = inst.kernel;
  int threads = inst.threads;
  dim3 grid;
  if (split) {
    if (partition_tokens <= 0 || partition_tokens % r.block_size != 0)
      return fail(PA_ERR_INVALID_ARG, "partition_tokens (%d) must be a positive multiple of block_size",
                  partition_tokens);
    if (r.num_seqs > kMaxSplitSeqs)
      return fail(PA_ERR_UNSUPPORTED, "pa_decode_split takes at most %d sequences", kMaxSplitSeqs);
    if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      return fail(PA_ERR_INVALID_ARG, "workspace must be non-NULL and 256-byte aligned");
    SplitLayout L = split_layout(r.num_seqs, r.num_q_heads, r.head_dim, r.block_size,
                                 r.max_blocks_per_seq, partition_tokens);
    if (extras != nullptr && extras->window > 0) {
      a.window = extras->window;
    } else if (extras != nullptr) {
      L.seg_off = extras->seg_off;
      L.m_off = extras->m_off;
      L.l_off = extras->l_off;
      L.acc_off = extras->acc_off;
      L.total = extras->total;
      L.pmax = extras->pmax;
      a.seq_skip_blocks = extras->seq_skip_blocks;
      a.seq_part_base = extras->seq_part_base;
    }
    if (workspace_bytes < L.total)
      return fail(PA_ERR_INVALID_ARG, "workspace_bytes %zu < required %zu", workspace_bytes, L.total);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    a.counters = reinterpret_cast<uint32_t*>(ws);
    a.part_m = reinterpret_cast<float*>(ws + L.m_off);
    a.part_l = reinterpret_cast<float*>(ws + L.l_off);
    a.part_acc = reinterpret_cast<float*>(ws + L.acc_off);
    a.partition_blocks = partition_tokens / r.block_size;
    a.max_partitions = L.pmax;
    a.persistent = 1;
    DeviceInfo dinfo;
    st = device_info(&dinfo);
    if (st != PA_OK) return st;
    int occ = 0;
    const bool suffix_pass = a.seq_skip_blocks != nullptr;
    if (use_stream_kernel(r, suffix_pass)) {
      // Balanced pieces per warp (paged_decode_stream_kernel). At most this
      // many pieces per (sequence, KV head): the slots after the prefix
      // pass's (none outside shared-prefix decode).
      a.seg_pieces = reinterpret_cast<int32_t*>(ws + L.seg_off);
      const int pb = partition_tokens / r.block_size;
      a.max_pieces = (r.max_blocks_per_seq + pb - 1) / pb + 1;
      // Units of one KV head's list, at most: bounds the grid for small batches.
      const int64_t units_max = static_cast<int64_t>(r.num_seqs) *
                                ((static_cast<int64_t>(r.max_blocks_per_seq) * r.block_size + 15) / 16);
      if (units_max >= (int64_t(1) << 31))
        return fail(PA_ERR_UNSUPPORTED, "num_seqs * max context / 16 must be < 2^31");
      const DecodeInstance::Stream& sk = inst.stream[suffix_pass ? 1 : 0];
      kernel = sk.kernel;
      threads = sk.threads;
      smem = sk.fixed_smem + (2 * r.num_seqs + 1) * 4;
      st = prepare_kernel(kernel, smem);
      if (st != PA_OK) return st;
      st = occupancy(kernel, threads, smem, &occ);
      if (st != PA_OK) return st;
      // One warp per KV head and group of units; no more groups than units.
      const int64_t W = sk.warps;
      const int64_t need = (units_max * r.num_kv_heads + W - 1) / W;
      const int64_t at_least = (r.num_kv_heads + W - 1) / W;
      const int64_t ctas = std::max(at_least, std::min<int64_t>(need, static_cast<int64_t>(dinfo.sms) * occ));
      grid = dim3(static_cast<unsigned>(ctas));
    } else {
      // Partition tickets (paged_decode_kernel, persistent mode).
      smem += (r.num_seqs + 1) * 4;
      st = prepare_kernel(inst.kernel, smem);
      if (st != PA_OK) return st;
      st = occupancy(inst.kernel, inst.threads, smem, &occ);
      if (st != PA_OK) return st;
      const int64_t max_items = static_cast<int64_t>(r.num_seqs) * r.num_kv_heads * L.pmax;
      const int64_t ctas = std::min<int64_t>(max_items, static_cast<int64_t>(dinfo.sms) * occ);
      grid = dim3(static_cast<unsigned>(ctas > 0 ? ctas : 1));
    }
  } else {
    a.partition_blocks = r.max_blocks_per_seq;
    a.max_partitions = 1;
    a.persistent = 0;
    st = prepare_kernel(inst.kernel, smem);
    if (st != PA_OK) return st;
    grid = dim3(static_cast<unsigned>(r.num_seqs * r.num_kv_heads));
  }

  const int rows = r.num_blocks * r.num_kv_heads * r.block_size;
  CUtensorMap tmk, tmv;
  st = pool_tensor_map(r.k_pool, rows, r.head_dim, r.block_size, r.dtype, &tmk);
  if (st != PA_OK) return st;
  st = pool_tensor_map(r.v_pool, rows, r.head_dim, r.block_size, r.dtype, &tmv);
  if (st != PA_OK) return st;

  void* args[] = {&tmk, &tmv, &a};
  cudaError_t err;
  if (split && clear_header) {
    err = cudaMemsetAsync(workspace, 0, kWorkspaceHeader, r.stream);
    if (err != cudaSuccess) return fail(PA_ERR_CUDA, "clearing the workspace header: %s", cudaGetErrorString(err));
  }
  if (extras != nullptr && extras->after_prefix_kernel) {
    // Runs alongside the shared-prefix kernel (disjoint partial slots) and
    // waits for it at exit, so the merge that depends on this grid sees both.
    a.wait_prior_at_exit = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = r.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelExC(&cfg, kernel, args);
  } else {
    err = cudaLaunchKernel(kernel, grid, dim3(threads), args, smem, r.stream);
  }
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "decode launch: %s", cudaGetErrorString(err));
  if (split) {
    // The merge grid is a programmatic dependent of the decode grid: it may be
    // scheduled before the decode grid ends and waits on the device
    // (griddepcontrol.wait) until the partials are complete and visible.
    int bs = r.block_size;
    void* margs[] = {&a, &bs};
    cudaLaunchConfig_t cfg{};
    const int64_t merge_rows = static_cast<int64_t>(r.num_seqs) * r.num_q_heads;
    cfg.gridDim = dim3(static_cast<unsigned>((merge_rows + kMergeRowsPerCta - 1) / kMergeRowsPerCta));
    cfg.blockDim = dim3(32 * kMergeRowsPerCta);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = r.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelExC(&cfg, inst.merge, margs);
    if (err != cudaSuccess) return fail(PA_ERR_CUDA, "merge launch: %s", cudaGetErrorString(err));
  }
  return launch_error("decode");
}

// ---- uploads of host-built plans --------------------------------------------------------
// pa_prefill and pa_decode_shared_prefix build small plans on the host (work
// items, schedules, group arrays). Plans of up to 30 KB go up as kernel
// parameters (upload_plan, below). For larger ones: an upload from pageable
// memory may make the host wait for the stream, so each call copies its plan
// into a slot of
// a pool of page-locked buffers (one pool per device) and uploads it from
// there with cudaMemcpyAsync, which returns at once. An event recorded after
// the uploads marks the slot busy until the copies have read it. A call takes
// the next slot whose uploads are done; when every slot is still busy (the
// host has run ahead of the stream) the pool grows by one slot, up to
// kMaxSlots, and only past that does a call wait, for the oldest slot. A slot
// grows (a page-locked allocation) when a plan outgrows it.
struct UploadPiece {
  void* dst;         // device destination
  const void* src;   // host source (the plan)
  size_t bytes;
};

class PlanStaging {
 public:
  static constexpr int kMaxSlots = 64;

  // Pieces whose device ranges lie close together (gaps of at most
  // kMergeGap bytes, the layouts' alignment padding) go up as one copy: each
  // cudaMemcpyAsync is a separate operation on the stream, ahead of the
  // kernels that read the plan. The padding between merged pieces receives
  // whatever the staging slot held there; nothing reads it.
  static constexpr size_t kMergeGap = 4096;
  static constexpr int kMaxPieces = 8;

  pa_status_t upload(const UploadPiece* pieces, int n, cudaStream_t stream) {
    if (n > kMaxPieces) return fail(PA_ERR_INVALID_ARG, "plan upload: %d pieces (at most %d)", n, kMaxPieces);
    UploadPiece p[kMaxPieces];
    int m = 0;
    for (int i = 0; i < n; ++i)
      if (pieces[i].bytes > 0) p[m++] = pieces[i];
    if (m == 0) return PA_OK;
    for (int i = 1; i < m; ++i)  // by destination
      for (int j = i; j > 0 && static_cast<uint8_t*>(p[j].dst) < static_cast<uint8_t*>(p[j - 1].dst); --j)
        std::swap(p[j], p[j - 1]);
    struct Run {
      uint8_t* dst;
      size_t bytes;
      int first, last;  // pieces [first, last)
    };
    Run runs[kMaxPieces];
    int nr = 0;
    for (int i = 0; i < m; ++i) {
      uint8_t* d = static_cast<uint8_t*>(p[i].dst);
      if (nr > 0) {
        Run& r = runs[nr - 1];
        uint8_t* end = r.dst + r.bytes;
        if (d >= end && static_cast<size_t>(d - end) <= kMergeGap) {
          r.bytes = static_cast<size_t>(d + p[i].bytes - r.dst);
          r.last = i + 1;
          continue;
        }
      }
      runs[nr++] = Run{d, p[i].bytes, i, i + 1};
    }
    size_t total = 0;
    for (int k = 0; k < nr; ++k) total += (runs[k].bytes + 15) & ~static_cast<size_t>(15);
    std::lock_guard<std::mutex> lock(mu_);
    Slot* sl = nullptr;
    pa_status_t st = acquire(&sl);
    if (st != PA_OK) return st;
    cudaError_t err;
    if (sl->cap < total) {
      if (sl->host != nullptr) cudaFreeHost(sl->host);
      sl->host = nullptr;
      sl->cap = 0;
      const size_t cap = std::max<size_t>(total, 64 * 1024);
      if ((err = cudaHostAlloc(reinterpret_cast<void**>(&sl->host), cap, cudaHostAllocPortable)) != cudaSuccess)
        return fail(PA_ERR_CUDA, "plan staging buffer: %s", cudaGetErrorString(err));
      sl->cap = cap;
    }
    size_t off = 0;
    for (int k = 0; k < nr; ++k) {
      const Run& r = runs[k];
      for (int i = r.first; i < r.last; ++i)
        std::memcpy(sl->host + off + (static_cast<uint8_t*>(p[i].dst) - r.dst), p[i].src, p[i].bytes);
      if ((err = cudaMemcpyAsync(r.dst, sl->host + off, r.bytes, cudaMemcpyHostToDevice, stream)) != cudaSuccess)
        return fail(PA_ERR_CUDA, "plan upload: %s", cudaGetErrorString(err));
      off += (r.bytes + 15) & ~static_cast<size_t>(15);
    }
    if ((err = cudaEventRecord(sl->done, stream)) != cudaSuccess)
      return fail(PA_ERR_CUDA, "plan staging record: %s", cudaGetErrorString(err));
    return PA_OK;
  }

 private:
  struct Slot {
    uint8_t* host = nullptr;
    size_t cap = 0;
    cudaEvent_t done = nullptr;
  };

  // True when the slot's previous uploads are complete (or it has none). A
  // "not ready" answer is not an error: it is cleared from the runtime's
  // last-error state unless an error was already pending there.
  static bool idle(const Slot& sl) {
    if (sl.done == nullptr) return true;
    const cudaError_t pending = cudaPeekAtLastError();
    const cudaError_t q = cudaEventQuery(sl.done);
    if (q == cudaErrorNotReady && pending == cudaSuccess) (void)cudaGetLastError();
    return q == cudaSuccess;
  }

  pa_status_t acquire(Slot** out) {
    const int n = static_cast<int>(slots_.size());
    for (int t = 0; t < n; ++t) {
      Slot* sl = slots_[(next_ + t) % n].get();
      if (idle(*sl)) {
        next_ = (next_ + t + 1) % n;
        *out = sl;
        return ensure_event(sl);
      }
    }
    if (n < kMaxSlots) {
      slots_.push_back(std::make_unique<Slot>());
      *out = slots_.back().get();
      return ensure_event(*out);
    }
    Slot* sl = slots_[next_].get();  // every slot busy: wait for the oldest
    next_ = (next_ + 1) % n;
    const cudaError_t err = cudaEventSynchronize(sl->done);
    if (err != cudaSuccess) return fail(PA_ERR_CUDA, "plan staging wait: %s", cudaGetErrorString(err));
    *out = sl;
    return PA_OK;
  }

  static pa_status_t ensure_event(Slot* sl) {
    if (sl->done != nullptr) return PA_OK;
    const cudaError_t err = cudaEventCreateWithFlags(&sl->done, cudaEventDisableTiming);
    if (err != cudaSuccess) return fail(PA_ERR_CUDA, "plan staging event: %s", cudaGetErrorString(err));
    return PA_OK;
  }

  std::mutex mu_;
  std::vector<std::unique_ptr<Slot>> slots_;
  int next_ = 0;
};

// Plans of up to kParamPlanBytes travel as the parameters of a small
// scatter kernel instead: the driver copies a launch's parameters when the
// launch is enqueued, so the host buffer is free at once, no copy-engine
// operation sits on the stream ahead of the plan's kernels, and the call can
// be captured into a CUDA graph (a replay scatters the captured plan again).
// Three parameter sizes, so that a small plan does not carry 30 KB.
constexpr int kParamPlanPieces = 8;

template <size_t N>
struct PlanParams {
  uint8_t* dst[kParamPlanPieces];
  uint32_t bytes[kParamPlanPieces];
  uint32_t off[kParamPlanPieces];  // piece i's bytes start at data + off[i] (16-byte aligned)
  int n;
  alignas(16) uint8_t data[N];
};

// One 16-byte chunk of the packed data per thread, 32 threads per CTA: lanes
// reading different parameter addresses are served one address at a time, so
// the chunks are spread over as many CTAs (and SMs) as there are 512-byte
// slices.
template <size_t N>
__global__ void __launch_bounds__(32) plan_scatter_kernel(const __grid_constant__ PlanParams<N> p) {
  const uint32_t c = blockIdx.x * 32 + threadIdx.x;
  for (int i = 0; i < p.n; ++i) {
    const uint32_t c0 = p.off[i] / 16, nb = p.bytes[i];
    if (c < c0 || c >= c0 + (nb + 15) / 16) continue;
    const uint32_t b0 = (c - c0) * 16;
    uint8_t* d = p.dst[i] + b0;
    const uint8_t* src = p.data + p.off[i] + b0;
    if (b0 + 16 <= nb && (reinterpret_cast<uintptr_t>(d) & 15u) == 0) {
      *reinterpret_cast<uint4*>(d) = *reinterpret_cast<const uint4*>(src);
    } else {
      for (uint32_t k = 0; k < 16 && b0 + k < nb; ++k) d[k] = src[k];
    }
    return;
  }
}

template <size_t N>
pa_status_t scatter_plan(const UploadPiece* p, int m, size_t total, cudaStream_t stream) {
  thread_local PlanParams<N> prm;
  size_t off = 0;
  prm.n = m;
  for (int i = 0; i < m; ++i) {
    prm.dst[i] = static_cast<uint8_t*>(p[i].dst);
    prm.bytes[i] = static_cast<uint32_t>(p[i].bytes);
    prm.off[i] = static_cast<uint32_t>(off);
    std::memcpy(prm.data + off, p[i].src, p[i].bytes);
    off += (p[i].bytes + 15) & ~static_cast<size_t>(15);
  }
  const unsigned ctas = static_cast<unsigned>((total / 16 + 31) / 32);
  plan_scatter_kernel<N><<<ctas, 32, 0, stream>>>(prm);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "plan scatter launch: %s", cudaGetErrorString(err));
  return PA_OK;
}

constexpr size_t kParamPlanBytes = 30 * 1024;

// Uploads a host plan on `stream`: as kernel parameters when it fits (set
// PAGEDKV_PLAN_UPLOAD=staging to force the other path, for tests), else
// through the current device's staging ring (rings live until the process
// exits). A staged upload is refused while the stream is being captured.
pa_status_t upload_plan(const UploadPiece* pieces, int n, cudaStream_t stream) {
  UploadPiece p[kParamPlanPieces];
  int m = 0;
  size_t total = 0;
  for (int i = 0; i < n; ++i) {
    if (pieces[i].bytes == 0) continue;
    if (m == kParamPlanPieces) return fail(PA_ERR_INVALID_ARG, "plan upload: more than %d pieces", kParamPlanPieces);
    p[m++] = pieces[i];
    total += (pieces[i].bytes + 15) & ~static_cast<size_t>(15);
  }
  if (m == 0) return PA_OK;
  const char* mode = std::getenv("PAGEDKV_PLAN_UPLOAD");
  const bool force_staging = mode != nullptr && std::strcmp(mode, "staging") == 0;
  if (!force_staging && total <= kParamPlanBytes) {
    if (total <= 2048) return scatter_plan<2048>(p, m, total, stream);
    if (total <= 8192) return scatter_plan<8192>(p, m, total, stream);
    return scatter_plan<kParamPlanBytes>(p, m, total, stream);
  }
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaError_t err = cudaStreamIsCapturing(stream, &cap);
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "cudaStreamIsCapturing: %s", cudaGetErrorString(err));
  if (cap != cudaStreamCaptureStatusNone)
    return fail(PA_ERR_UNSUPPORTED,
                "a host plan of %zu bytes (more than %zu, or staging forced) is uploaded from a "
                "reused staging slot and cannot be captured into a graph", total, kParamPlanBytes);
  int dev = 0;
  err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(err));
  static std::mutex mu;
  static std::vector<PlanStaging*> rings;
  PlanStaging* ring;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (static_cast<int>(rings.size()) <= dev) rings.resize(dev + 1, nullptr);
    if (rings[dev] == nullptr) rings[dev] = new PlanStaging();
    ring = rings[dev];
  }
  return ring->upload(p, m, stream);
}

// ---- shared-prefix decode ------------------------------------------------------------
// Workspace: [0,256) header | skip int32 [B] | part_base int32 [B] |
// members int32 [B] | items PrefixItem [B*Hkv*kMaxPrefixParts] | q tiles |
// packed q | pieces int32 [B][Hq] | m, l float [B][Hq][pmax] |
// acc float [B][Hq][pmax][D], where
// pmax = kMaxPrefixParts + ceil(max_blocks_per_seq / partition blocks) + 1.
constexpr int kMaxPrefixParts = 16;
constexpr int kPrefixRows = 64;  // query rows per prefix CTA (4 warps x 16)

struct PrefixLayout {
  size_t skip_off, base_off, members_off, items_off, qtiles_off, qpack_off;
  SplitExtras ex;
  size_t max_items, max_qtiles;
};

constexpr int kTcPrefixRows = 128;  // query rows per tcgen05 prefix tile

// Q rows of one tcgen05 prefix tile: members [member_begin, + count) of the
// packed member list, heads kvh * group .. + group.
struct QPackTile {
  int32_t member_begin, count, kvh, pad;
};

PrefixLayout prefix_layout(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                           int block_size, int max_blocks_per_seq, int partition_tokens) {
  PrefixLayout L{};
  const int pb = partition_tokens / block_size;
  L.ex.pmax = kMaxPrefixParts + (max_blocks_per_seq + pb - 1) / pb + 1;
  const size_t B = static_cast<size_t>(num_seqs);
  const size_t G = static_cast<size_t>(std::max(1, num_q_heads / std::max(1, num_kv_heads)));
  L.max_items = B * static_cast<size_t>(num_kv_heads) * kMaxPrefixParts;
  // row tiles: each group's members in runs of 128 / G, per KV head
  L.max_qtiles = (B + (B * G + kTcPrefixRows - 1) / kTcPrefixRows) * static_cast<size_t>(num_kv_heads);
  L.skip_off = kWorkspaceHeader;
  L.base_off = L.skip_off + align256(B * 4);
  L.members_off = L.base_off + align256(B * 4);
  L.items_off = L.members_off + align256(B * 4);
  L.qtiles_off = L.items_off + align256(L.max_items * std::max(sizeof(PrefixItem), sizeof(PrefillItem)));
  L.qpack_off = L.qtiles_off + align256(L.max_qtiles * sizeof(QPackTile));
  const size_t qpack_bytes = L.max_qtiles * kTcPrefixRows * static_cast<size_t>(head_dim) * 2;
  const size_t rows = B * num_q_heads * L.ex.pmax;
  L.ex.seg_off = L.qpack_off + align256(qpack_bytes);
  L.ex.m_off = L.ex.seg_off + align256(B * num_q_heads * 4);
  L.ex.l_off = L.ex.m_off + align256(rows * 4);
  L.ex.acc_off = L.ex.l_off + align256(rows * 4);
  L.ex.total = L.ex.acc_off + align256(rows * static_cast<size_t>(head_dim) * 4);
  return L;
}

// Packs the query rows of each tcgen05 prefix tile contiguously ([tile][token
// = member][head][head_dim], rows past the tile's members zero) so that one
// 3-D TMA box loads a tile's Q. One CTA per tile, one thread per row.
__global__ void __launch_bounds__(kTcPrefixRows) q_pack_kernel(const __nv_bfloat16* __restrict__ q,
                                                               const int32_t* __restrict__ members,
                                                               const QPackTile* __restrict__ tiles,
                                                               int group, int num_q_heads, int head_dim,
                                                               int tokens, __nv_bfloat16* __restrict__ qpack) {
  grid_dependents_launch();  // the prefix kernel may start; it waits before reading qpack
  const QPackTile tl = tiles[blockIdx.x];
  const int r = threadIdx.x;
  const int m = r / group, g = r % group;
  if (m >= tokens) return;
  uint4* dst = reinterpret_cast<uint4*>(
      qpack + ((static_cast<int64_t>(blockIdx.x) * tokens + m) * group + g) * head_dim);
  const int n16 = head_dim / 8;
  if (m < tl.count) {
    const int64_t s = members[tl.member_begin + m];
    const uint4* src = reinterpret_cast<const uint4*>(
        q + (s * num_q_heads + static_cast<int64_t>(tl.kvh) * group + g) * head_dim);
    for (int i = 0; i < n16; ++i) dst[i] = src[i];
  } else {
    for (int i = 0; i < n16; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
  }
}

pa_status_t run_shared_prefix(const DecodeReq& r, int partition_tokens, int num_groups,
                              const int32_t* offs, const int32_t* members, const int32_t* blocks,
                              void* workspace, size_t workspace_bytes) {
  DecodeInstance inst;
  pa_status_t st = validate_and_pick(r, &inst);
  if (st != PA_OK) return st;
  if (r.dtype != PA_BF16) return fail(PA_ERR_UNSUPPORTED, "pa_decode_shared_prefix is bf16 only");
  // PAGEDKV_PREFIX_KERNEL=tcgen05 selects the tcgen05 pass (the prefill kernel
  // with one 128-row tile per CTA, Q packed by a small kernel). Its prefix
  // kernel is faster than the 64-row mma.sync pass (37.6 vs 41.3 us on the
  // 8 x 4008-token, 16-branch workload), but the whole call measured slower
  // (70.3 vs 69.0 us): two 100 KB CTAs per SM leave no room for the suffix
  // kernel that runs alongside. The default stays mma.sync.
  const char* kname = std::getenv("PAGEDKV_PREFIX_KERNEL");
  const bool tc = kname != nullptr && std::strcmp(kname, "tcgen05") == 0;
  PrefixInstance pinst;
  if (!(tc ? find_tc_prefix_bf16(r.head_dim, r.block_size, &pinst)
           : find_prefix_bf16(r.head_dim, r.block_size, &pinst)))
    return fail(PA_ERR_UNSUPPORTED, "no shared-prefix kernel for head_dim=%d block_size=%d",
                r.head_dim, r.block_size);
  if (partition_tokens <= 0 || partition_tokens % r.block_size != 0)
    return fail(PA_ERR_INVALID_ARG, "partition_tokens (%d) must be a positive multiple of block_size",
                partition_tokens);
  if (r.num_seqs > kMaxSplitSeqs)
    return fail(PA_ERR_UNSUPPORTED, "at most %d sequences", kMaxSplitSeqs);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(PA_ERR_INVALID_ARG, "workspace must be non-NULL and 256-byte aligned");
  const int G = r.num_q_heads / r.num_kv_heads;
  const int B = r.num_seqs;
  if (num_groups < 0 || (num_groups > 0 && (offs == nullptr || members == nullptr || blocks == nullptr)))
    return fail(PA_ERR_INVALID_ARG, "bad group arrays");
  const PrefixLayout L = prefix_layout(B, r.num_q_heads, r.num_kv_heads, r.head_dim, r.block_size,
                                       r.max_blocks_per_seq, partition_tokens);
  if (workspace_bytes < L.ex.total)
    return fail(PA_ERR_INVALID_ARG, "workspace_bytes %zu < required %zu", workspace_bytes, L.ex.total);
  if (B == 0) return ok();

  const int chunk_rows = tc ? kTcPrefixRows : kPrefixRows;
  thread_local std::vector<int32_t> skip, base, mem;
  thread_local std::vector<PrefixItem> items;
  thread_local std::vector<PrefillItem> tc_items;
  thread_local std::vector<QPackTile> qtiles;
  thread_local std::vector<char> seen;
  skip.assign(B, 0);
  base.assign(B, 0);
  seen.assign(B, 0);
  mem.clear();
  items.clear();
  tc_items.clear();
  qtiles.clear();
  // groups: validate, and find the prefix partition size
  int64_t total_blocks = 0;
  int max_blocks = 0;
  bool many_chunks = false;
  if (num_groups > 0 && offs[0] != 0) return fail(PA_ERR_INVALID_ARG, "group_offsets[0] must be 0");
  for (int g = 0; g < num_groups; ++g) {
    const int b0 = offs[g], b1 = offs[g + 1];
    if (b1 < b0 || b1 > B) return fail(PA_ERR_INVALID_ARG, "group_offsets not increasing within [0, %d]", B);
    if (blocks[g] < 1 || blocks[g] > r.max_blocks_per_seq)
      return fail(PA_ERR_INVALID_ARG, "group_blocks[%d] = %d out of range", g, blocks[g]);
    for (int i = b0; i < b1; ++i) {
      const int m = members[i];
      if (m < 0 || m >= B || seen[m]) return fail(PA_ERR_INVALID_ARG, "group member %d invalid or repeated", m);
      seen[m] = 1;
    }
    const int chunks = ((b1 - b0) * G + chunk_rows - 1) / chunk_rows;
    many_chunks = many_chunks || chunks > 1;
    total_blocks += static_cast<int64_t>(blocks[g]) * chunks * r.num_kv_heads;
    max_blocks = std::max(max_blocks, blocks[g]);
  }
  DeviceInfo dinfo;
  st = device_info(&dinfo);
  if (st != PA_OK) return st;
  // Partition so that the items fill about one wave (the kernel's CTAs per
  // SM x SMs), at most kMaxPrefixParts per group, and at least four blocks
  // each; fewer partitions mean fewer partials for the merge. Rounding up the
  // partitions of each group can overflow the wave, so the size grows until
  // the items fit (a second, nearly empty wave costs a whole item's time).
  int per_sm = tc ? 2 : 3;
  if (!tc) {
    st = prepare_kernel(pinst.kernel, pinst.smem);
    if (st != PA_OK) return st;
    st = occupancy(pinst.kernel, pinst.threads, pinst.smem, &per_sm);
    if (st != PA_OK) return st;
  }
  const int64_t slots = static_cast<int64_t>(per_sm) * dinfo.sms;
  int pbp = static_cast<int>((total_blocks + slots - 1) / slots);
  pbp = std::max(pbp, (max_blocks + kMaxPrefixParts - 1) / kMaxPrefixParts);
  pbp = std::max(pbp, 4);
  auto count_items = [&](int part_blocks) {
    int64_t n = 0;
    for (int g = 0; g < num_groups; ++g) {
      const int members_g = offs[g + 1] - offs[g];
      if (members_g == 0) continue;
      const int chunks = (members_g * G + chunk_rows - 1) / chunk_rows;
      n += static_cast<int64_t>((blocks[g] + part_blocks - 1) / part_blocks) * chunks * r.num_kv_heads;
    }
    return n;
  };
  while (pbp < max_blocks && count_items(pbp) > slots) ++pbp;
  const int per_chunk = std::max(1, chunk_rows / G);
  for (int g = 0; g < num_groups; ++g) {
    const int b0 = offs[g], b1 = offs[g + 1];
    if (b1 - b0 == 0) continue;
    const int nparts = (blocks[g] + pbp - 1) / pbp;
    const int first = static_cast<int>(mem.size());
    for (int i = b0; i < b1; ++i) {
      skip[members[i]] = blocks[g];
      base[members[i]] = nparts;
      mem.push_back(members[i]);
    }
    for (int c = first; c < first + (b1 - b0); c += per_chunk) {
      const int cnt = std::min(per_chunk, first + (b1 - b0) - c);
      for (int h = 0; h < r.num_kv_heads; ++h) {
        // tcgen05: the tile's Q rows are packed at token index tile * per_chunk;
        // no causal limit (every row sees the whole shared span: p0 past it)
        const int tile = static_cast<int>(qtiles.size());
        if (tc) qtiles.push_back(QPackTile{c, cnt, h, 0});
        for (int p = 0; p < nparts; ++p) {
          const int bb = p * pbp, be = std::min(blocks[g], (p + 1) * pbp);
          if (tc)
            tc_items.push_back(PrefillItem{members[b0], tile * per_chunk, cnt, be * r.block_size, bb, be,
                                           be * r.block_size, h, p, 0, 0, c});
          else
            items.push_back(PrefixItem{members[b0], c, cnt, bb, be, h, p, 0});
        }
      }
    }
  }
  if (items.size() > L.max_items || tc_items.size() > L.max_items || qtiles.size() > L.max_qtiles)
    return fail(PA_ERR_INVALID_ARG, "too many prefix items");

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaError_t err;
  const UploadPiece plan[] = {
      {ws + L.skip_off, skip.data(), static_cast<size_t>(B) * 4},
      {ws + L.base_off, base.data(), static_cast<size_t>(B) * 4},
      {ws + L.members_off, mem.data(), mem.size() * 4},
      {ws + L.items_off, items.data(), items.size() * sizeof(PrefixItem)},
      {ws + L.items_off, tc_items.data(), tc_items.size() * sizeof(PrefillItem)},
      {ws + L.qtiles_off, qtiles.data(), qtiles.size() * sizeof(QPackTile)}};
  st = upload_plan(plan, 6, r.stream);
  if (st != PA_OK) return st;

  SplitExtras ex = L.ex;
  ex.seq_skip_blocks = reinterpret_cast<const int32_t*>(ws + L.skip_off);
  ex.seq_part_base = reinterpret_cast<const int32_t*>(ws + L.base_off);

  if (!tc_items.empty()) {
    auto* qpack = reinterpret_cast<__nv_bfloat16*>(ws + L.qpack_off);
    q_pack_kernel<<<static_cast<unsigned>(qtiles.size()), kTcPrefixRows, 0, r.stream>>>(
        static_cast<const __nv_bfloat16*>(r.q), reinterpret_cast<const int32_t*>(ws + L.members_off),
        reinterpret_cast<const QPackTile*>(ws + L.qtiles_off), G, r.num_q_heads, r.head_dim, per_chunk,
        qpack);
    if ((err = cudaGetLastError()) != cudaSuccess) return fail(PA_ERR_CUDA, "q pack launch: %s", cudaGetErrorString(err));
    st = prepare_kernel(pinst.kernel, pinst.smem);
    if (st != PA_OK) return st;
    const int rows = r.num_blocks * r.num_kv_heads * r.block_size;
    CUtensorMap tmk, tmv, tmq;
    st = pool_tensor_map(r.k_pool, rows, r.head_dim, r.block_size, r.dtype, &tmk);
    if (st != PA_OK) return st;
    st = pool_tensor_map(r.v_pool, rows, r.head_dim, r.block_size, r.dtype, &tmv);
    if (st != PA_OK) return st;
    st = q_tensor_map(qpack, static_cast<int>(qtiles.size()) * per_chunk, G, r.head_dim, G, per_chunk, &tmq);
    if (st != PA_OK) return st;
    PrefillArgs pf{};
    DecodeArgs& a = pf.d;
    a.q = r.q;
    a.block_tables = r.block_tables;
    a.context_lens = r.context_lens;
    a.part_m = reinterpret_cast<float*>(ws + ex.m_off);
    a.part_l = reinterpret_cast<float*>(ws + ex.l_off);
    a.part_acc = reinterpret_cast<float*>(ws + ex.acc_off);
    a.dev_err = r.dev_err;
    a.num_seqs = B;
    a.num_q_heads = r.num_q_heads;
    a.num_kv_heads = r.num_kv_heads;
    a.group = G;
    a.num_blocks = r.num_blocks;
    a.max_blocks_per_seq = r.max_blocks_per_seq;
    a.max_partitions = ex.pmax;
    a.scale_log2 = r.scale * 1.4426950408889634f;
    pf.items = reinterpret_cast<const PrefillItem*>(ws + L.items_off);
    pf.out_tokens = reinterpret_cast<const int32_t*>(ws + L.members_off);
    // The output map is unused here (rows are scattered through out_tokens).
    void* args[] = {&tmk, &tmv, &tmq, &tmq, &pf};
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(tc_items.size()));
    cfg.blockDim = dim3(pinst.threads);
    cfg.dynamicSmemBytes = pinst.smem;
    cfg.stream = r.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelExC(&cfg, pinst.kernel, args);
    if (err != cudaSuccess) return fail(PA_ERR_CUDA, "prefix launch: %s", cudaGetErrorString(err));
    ex.after_prefix_kernel = true;
  }
  if (!items.empty()) {
    st = prepare_kernel(pinst.kernel, pinst.smem);
    if (st != PA_OK) return st;
    const int rows = r.num_blocks * r.num_kv_heads * r.block_size;
    CUtensorMap tmk, tmv;
    st = pool_tensor_map(r.k_pool, rows, r.head_dim, r.block_size, r.dtype, &tmk);
    if (st != PA_OK) return st;
    st = pool_tensor_map(r.v_pool, rows, r.head_dim, r.block_size, r.dtype, &tmv);
    if (st != PA_OK) return st;
    PrefixArgs pa{};
    pa.d.q = r.q;
    pa.d.block_tables = r.block_tables;
    pa.d.context_lens = r.context_lens;
    pa.d.part_m = reinterpret_cast<float*>(ws + ex.m_off);
    pa.d.part_l = reinterpret_cast<float*>(ws + ex.l_off);
    pa.d.part_acc = reinterpret_cast<float*>(ws + ex.acc_off);
    pa.d.dev_err = r.dev_err;
    pa.d.num_seqs = B;
    pa.d.num_q_heads = r.num_q_heads;
    pa.d.num_kv_heads = r.num_kv_heads;
    pa.d.group = G;
    pa.d.num_blocks = r.num_blocks;
    pa.d.max_blocks_per_seq = r.max_blocks_per_seq;
    pa.d.max_partitions = ex.pmax;
    pa.d.scale_log2 = r.scale * 1.4426950408889634f;
    // Tiles re-read by several row chunks stay in L2; otherwise read once.
    pa.d.l2_hint = many_chunks ? 2 : 1;
    pa.items = reinterpret_cast<const PrefixItem*>(ws + L.items_off);
    pa.members = reinterpret_cast<const int32_t*>(ws + L.members_off);
    void* args[] = {&tmk, &tmv, &pa};
    err = cudaLaunchKernel(pinst.kernel, dim3(static_cast<unsigned>(items.size())), dim3(pinst.threads),
                           args, pinst.smem, r.stream);
    if (err != cudaSuccess) return fail(PA_ERR_CUDA, "prefix launch: %s", cudaGetErrorString(err));
    ex.after_prefix_kernel = true;
  }
  return run_decode(r, true, partition_tokens, workspace, workspace_bytes, &ex);
}

// ---- paged prefill -------------------------------------------------------------------
// Workspace: [0,256) header | merge_lens int32 [total_q] | items PrefillItem
// [max_items] | schedule offsets int32 [max_items + 1] | m, l float
// [total_q][Hq][pmax] | acc float [...][head_dim],
// pmax = ceil(max_blocks_per_seq / partition blocks).
struct PrefillLayout {
  size_t lens_off, items_off, sched_off, m_off, l_off, acc_off, total, max_items;
  int pmax;
};

PrefillLayout prefill_layout(int num_seqs, int total_q, int num_q_heads, int num_kv_heads,
                             int head_dim, int block_size, int max_blocks_per_seq,
                             int partition_tokens) {
  PrefillLayout L{};
  const int pb = partition_tokens / block_size;
  L.pmax = (max_blocks_per_seq + pb - 1) / pb;
  const int G = std::max(1, num_q_heads / std::max(1, num_kv_heads));
  const int tq = std::max(1, kPrefixRows / G);
  const size_t tiles = static_cast<size_t>(total_q) / tq + num_seqs;
  L.max_items = tiles * num_kv_heads * L.pmax;
  L.lens_off = kWorkspaceHeader;
  L.items_off = L.lens_off + align256(static_cast<size_t>(total_q) * 4);
  const size_t rows = static_cast<size_t>(total_q) * num_q_heads * L.pmax;
  L.sched_off = L.items_off + align256(L.max_items * sizeof(PrefillItem));
  L.m_off = L.sched_off + align256((L.max_items + 1) * 4);
  L.l_off = L.m_off + align256(rows * 4);
  L.acc_off = L.l_off + align256(rows * 4);
  L.total = L.acc_off + align256(rows * static_cast<size_t>(head_dim) * 4);
  return L;
}

// The prefill items: one per (sequence, run of tq query tokens, KV head, KV
// partition of pb blocks), in sequence order with each sequence's query
// tiles last-first (the longest spans first), so that work handed out last
// is short. lens (optional) receives each query token's attended length.
void prefill_items(int B, const int32_t* ctx_host, const int32_t* qlen_host, int num_kv_heads, int G,
                   int block_size, int tq, int pb, std::vector<PrefillItem>& items,
                   std::vector<int32_t>* lens, bool* any_split) {
  items.clear();
  *any_split = false;
  int q_base = 0;
  for (int s = 0; s < B; ++s) {
    const int qlen = qlen_host[s], ctx = ctx_host[s];
    for (int t = qlen > 0 ? (qlen - 1) / tq * tq : -1; t >= 0; t -= tq) {
      const int count = std::min(tq, qlen - t);
      const int p0 = ctx - qlen + t;
      const int kv_end = p0 + count;  // last position + 1
      const int nblk = (kv_end + block_size - 1) / block_size;
      const int nparts = (nblk + pb - 1) / pb;
      *any_split = *any_split || nparts > 1;
      if (lens != nullptr)
        for (int i = 0; i < count; ++i) (*lens)[q_base + t + i] = kv_end;
      for (int h = 0; h < num_kv_heads; ++h)
        for (int p = 0; p < nparts; ++p)
          items.push_back(PrefillItem{s, q_base + t, count, p0, p * pb, std::min(nblk, (p + 1) * pb),
                                      kv_end, h, p, nparts == 1 ? 1 : 0, h * G, -1});
    }
    q_base += qlen;
  }
}

// Persistent schedule over `ctas` CTAs: each item goes, in list order, to
// the CTA with the least estimated work so far (cost ~ KV chunks x active
// tiles, plus a constant per item; ties to the lowest CTA), and each CTA's
// items are stored together, in list order: CTA b runs sched_items
// [sched_offs[b], sched_offs[b + 1]). owner (optional) receives each item's CTA.
void prefill_schedule(const std::vector<PrefillItem>& items, unsigned ctas, int block_size,
                      int tile_tokens, std::vector<PrefillItem>& sched_items,
                      std::vector<int32_t>& sched_offs, std::vector<int32_t>& owner) {
  using Load = std::pair<int64_t, int32_t>;
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
  for (unsigned b = 0; b < ctas; ++b) heap.push(Load{0, static_cast<int32_t>(b)});
  owner.resize(items.size());
  sched_offs.assign(ctas + 1, 0);
  for (size_t i = 0; i < items.size(); ++i) {
    const PrefillItem& it = items[i];
    const int64_t span = std::max(0, std::min(it.block_end * block_size, it.kv_end) -
                                         it.block_begin * block_size);
    const int64_t cost = span * (it.q_count > tile_tokens ? 21 : 15) / 64 + 20;
    const Load ld = heap.top();
    heap.pop();
    owner[i] = ld.second;
    ++sched_offs[ld.second + 1];
    heap.push(Load{ld.first + cost, ld.second});
  }
  for (unsigned b = 0; b < ctas; ++b) sched_offs[b + 1] += sched_offs[b];
  sched_items.resize(items.size());
  thread_local std::vector<int32_t> fill;
  fill.assign(sched_offs.begin(), sched_offs.end() - 1);
  for (size_t i = 0; i < items.size(); ++i) sched_items[fill[owner[i]]++] = items[i];
}

// The plan pa_prefill makes for the tcgen05 kernel, exposed for inspection
// (pa_prefill_plan). Host-only: no CUDA call.
pa_status_t prefill_plan(const int32_t* ctx_host, const int32_t* qlen_host, int B, int num_q_heads,
                         int num_kv_heads, int block_size, int partition_tokens, int max_ctas,
                         int32_t* items_out, int max_items, int* num_items, int* num_ctas) {
  if (num_items == nullptr || num_ctas == nullptr)
    return fail(PA_ERR_INVALID_ARG, "num_items and num_ctas are required");
  if (B < 0 || (B > 0 && (ctx_host == nullptr || qlen_host == nullptr)))
    return fail(PA_ERR_INVALID_ARG, "context_lens and query_lens (host) are required");
  if (num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0)
    return fail(PA_ERR_INVALID_ARG, "num_q_heads (%d) must be a positive multiple of num_kv_heads (%d)",
                num_q_heads, num_kv_heads);
  PrefixInstance pinst;
  if (!find_prefill_bf16(128, block_size, true, &pinst))
    return fail(PA_ERR_UNSUPPORTED, "no tcgen05 prefill kernel for block_size=%d", block_size);
  if (partition_tokens <= 0 || partition_tokens % block_size != 0)
    return fail(PA_ERR_INVALID_ARG, "partition_tokens (%d) must be a positive multiple of block_size",
                partition_tokens);
  for (int s = 0; s < B; ++s)
    if (qlen_host[s] < 0 || ctx_host[s] < qlen_host[s])
      return fail(PA_ERR_INVALID_ARG, "sequence %d: query_len %d, context_len %d out of range", s,
                  qlen_host[s], ctx_host[s]);
  const int G = num_q_heads / num_kv_heads;
  const int tile_tokens = std::max(1, pinst.rows / G);
  thread_local std::vector<PrefillItem> items, sched_items;
  thread_local std::vector<int32_t> sched_offs, owner;
  bool any_split = false;
  prefill_items(B, ctx_host, qlen_host, num_kv_heads, G, block_size, pinst.tiles * tile_tokens,
                partition_tokens / block_size, items, nullptr, &any_split);
  const size_t n = items.size();
  const bool persistent = max_ctas > 0 && n > static_cast<size_t>(max_ctas);
  *num_items = static_cast<int>(n);
  *num_ctas = persistent ? max_ctas : static_cast<int>(n);
  if (items_out == nullptr) return ok();
  if (max_items < 0 || static_cast<size_t>(max_items) < n)
    return fail(PA_ERR_INVALID_ARG, "max_items %d < %zu items", max_items, n);
  const PrefillItem* list = items.data();
  if (persistent) {
    prefill_schedule(items, static_cast<unsigned>(max_ctas), block_size, tile_tokens, sched_items,
                     sched_offs, owner);
    list = sched_items.data();
  }
  int b = 0;
  for (size_t i = 0; i < n; ++i) {
    while (persistent && static_cast<size_t>(sched_offs[b + 1]) <= i) ++b;
    const PrefillItem& it = list[i];
    int32_t* row = items_out + 6 * i;
    row[0] = it.seq;
    row[1] = it.q_begin;
    row[2] = it.q_count;
    row[3] = it.kvh;
    row[4] = it.part;
    row[5] = persistent ? b : static_cast<int32_t>(i);
  }
  return ok();
}

pa_status_t run_prefill(const DecodeReq& r_in, const int32_t* ctx_host, const int32_t* qlen_host,
                        int total_q, int partition_tokens, void* workspace, size_t workspace_bytes) {
  // With no new tokens q and out are never touched and may be NULL; every
  // other argument is still checked.
  DecodeReq r = r_in;
  if (total_q == 0) {
    if (r.q == nullptr) r.q = r.k_pool;
    if (r.out == nullptr) r.out = const_cast<void*>(r.k_pool);  // never written
  }
  DecodeInstance inst;
  pa_status_t st = validate_and_pick(r, &inst);  // shapes, alignment, dtype, group (merge kernel)
  if (st != PA_OK) return st;
  if (r.dtype != PA_BF16) return fail(PA_ERR_UNSUPPORTED, "pa_prefill is bf16 only");
  // PAGEDKV_PREFILL_KERNEL=mma_sync selects the 64-row mma.sync kernel (kept
  // for comparison); the default is the tcgen05 kernel.
  const char* kname = std::getenv("PAGEDKV_PREFILL_KERNEL");
  const bool tcgen05 = kname == nullptr || std::strcmp(kname, "mma_sync") != 0;
  PrefixInstance pinst;
  if (!find_prefill_bf16(r.head_dim, r.block_size, tcgen05, &pinst))
    return fail(PA_ERR_UNSUPPORTED, "no prefill kernel for head_dim=%d block_size=%d", r.head_dim,
                r.block_size);
  if (partition_tokens <= 0 || partition_tokens % r.block_size != 0)
    return fail(PA_ERR_INVALID_ARG, "partition_tokens (%d) must be a positive multiple of block_size",
                partition_tokens);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(PA_ERR_INVALID_ARG, "workspace must be non-NULL and 256-byte aligned");
  if (total_q < 0) return fail(PA_ERR_INVALID_ARG, "total_q < 0");
  const int B = r.num_seqs;
  if (B > 0 && (ctx_host == nullptr || qlen_host == nullptr))
    return fail(PA_ERR_INVALID_ARG, "context_lens and query_lens (host) are required");
  int64_t sum_q = 0;
  for (int s = 0; s < B; ++s) {
    if (qlen_host[s] < 0 || ctx_host[s] < qlen_host[s] ||
        static_cast<int64_t>(ctx_host[s]) > static_cast<int64_t>(r.max_blocks_per_seq) * r.block_size)
      return fail(PA_ERR_INVALID_ARG, "sequence %d: query_len %d, context_len %d out of range", s,
                  qlen_host[s], ctx_host[s]);
    sum_q += qlen_host[s];
  }
  if (sum_q != total_q) return fail(PA_ERR_INVALID_ARG, "sum of query_lens %lld != total_q %d",
                                    (long long)sum_q, total_q);
  const PrefillLayout L = prefill_layout(B, total_q, r.num_q_heads, r.num_kv_heads, r.head_dim,
                                         r.block_size, r.max_blocks_per_seq, partition_tokens);
  if (workspace_bytes < L.total)
    return fail(PA_ERR_INVALID_ARG, "workspace_bytes %zu < required %zu", workspace_bytes, L.total);
  if (total_q == 0) return ok();

  const int G = r.num_q_heads / r.num_kv_heads;
  const int tq = pinst.tiles * std::max(1, pinst.rows / G);  // query tokens per CTA
  const int pb = partition_tokens / r.block_size;
  thread_local std::vector<int32_t> lens;
  thread_local std::vector<PrefillItem> items;
  lens.assign(total_q, 0);
  bool any_split = false;
  prefill_items(B, ctx_host, qlen_host, r.num_kv_heads, G, r.block_size, tq, pb, items, &lens,
                &any_split);
  if (items.size() > L.max_items) return fail(PA_ERR_INVALID_ARG, "too many prefill items");
  st = prepare_kernel(pinst.kernel, pinst.smem);
  if (st != PA_OK) return st;

  // The tcgen05 kernel runs persistently when there are more items than
  // resident CTAs (prefill_schedule); a CTA starts the next item's loads
  // while it finishes the current one.
  thread_local std::vector<PrefillItem> sched_items;
  thread_local std::vector<int32_t> sched_offs, owner;
  unsigned grid = static_cast<unsigned>(items.size());
  const PrefillItem* upload_items = items.data();
  bool persistent = false;
  if (pinst.q_map) {
    DeviceInfo di;
    int occ = 0;
    if ((st = device_info(&di)) != PA_OK) return st;
    if ((st = occupancy(pinst.kernel, pinst.threads, pinst.smem, &occ)) != PA_OK) return st;
    size_t ctas = static_cast<size_t>(di.sms) * occ;
    // PAGEDKV_PREFILL_CTAS=n caps the persistent grid (tests use it to give
    // every CTA many items at small sizes).
    if (const char* cap = std::getenv("PAGEDKV_PREFILL_CTAS")) {
      const long n = std::strtol(cap, nullptr, 10);
      if (n > 0) ctas = std::min(ctas, static_cast<size_t>(n));
    }
    if (items.size() > ctas) {
      persistent = true;
      grid = static_cast<unsigned>(ctas);
      prefill_schedule(items, grid, r.block_size, std::max(1, pinst.rows / G), sched_items,
                       sched_offs, owner);
      upload_items = sched_items.data();
    }
  }

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaError_t err;
  const UploadPiece plan[] = {
      {ws + L.lens_off, lens.data(), lens.size() * 4},
      {ws + L.items_off, upload_items, items.size() * sizeof(PrefillItem)},
      {ws + L.sched_off, sched_offs.data(), persistent ? sched_offs.size() * 4 : 0}};
  st = upload_plan(plan, 3, r.stream);
  if (st != PA_OK) return st;
  const int rows = r.num_blocks * r.num_kv_heads * r.block_size;
  CUtensorMap tmk, tmv;
  st = pool_tensor_map(r.k_pool, rows, r.head_dim, r.block_size, r.dtype, &tmk);
  if (st != PA_OK) return st;
  st = pool_tensor_map(r.v_pool, rows, r.head_dim, r.block_size, r.dtype, &tmv);
  if (st != PA_OK) return st;
  PrefillArgs pf{};
  DecodeArgs& a = pf.d;
  a.q = r.q;
  a.out = r.out;
  a.block_tables = r.block_tables;
  a.context_lens = reinterpret_cast<const int32_t*>(ws + L.lens_off);  // per query token (merge)
  a.part_m = reinterpret_cast<float*>(ws + L.m_off);
  a.part_l = reinterpret_cast<float*>(ws + L.l_off);
  a.part_acc = reinterpret_cast<float*>(ws + L.acc_off);
  a.dev_err = r.dev_err;
  a.num_seqs = total_q;  // the merge walks (query token, head) rows
  a.num_q_heads = r.num_q_heads;
  a.num_kv_heads = r.num_kv_heads;
  a.group = G;
  a.num_blocks = r.num_blocks;
  a.max_blocks_per_seq = r.max_blocks_per_seq;
  a.partition_blocks = pb;
  a.max_partitions = L.pmax;
  a.scale_log2 = r.scale * 1.4426950408889634f;
  pf.items = reinterpret_cast<const PrefillItem*>(ws + L.items_off);
  pf.out_tokens = nullptr;
  pf.sched_off = persistent ? reinterpret_cast<const int32_t*>(ws + L.sched_off) : nullptr;
  CUtensorMap tmq, tmo;
  void* args3[] = {&tmk, &tmv, &pf};
  void* args5[] = {&tmk, &tmv, &tmq, &tmo, &pf};
  if (pinst.q_map) {
    // out has q's layout: the same boxes serve the output tiles' stores.
    const int tile_tokens = std::max(1, pinst.rows / G);
    st = q_tensor_map(r.q, total_q, r.num_q_heads, r.head_dim, G, tile_tokens, &tmq);
    if (st != PA_OK) return st;
    st = q_tensor_map(r.out, total_q, r.num_q_heads, r.head_dim, G, tile_tokens, &tmo);
    if (st != PA_OK) return st;
  }
  err = cudaLaunchKernel(pinst.kernel, dim3(grid), dim3(pinst.threads), pinst.q_map ? args5 : args3,
                         pinst.smem, r.stream);
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "prefill launch: %s", cudaGetErrorString(err));
  if (any_split) {
    int bs = r.block_size;
    void* margs[] = {&a, &bs};
    cudaLaunchConfig_t cfg{};
    const int64_t merge_rows = static_cast<int64_t>(total_q) * r.num_q_heads;
    cfg.gridDim = dim3(static_cast<unsigned>((merge_rows + kMergeRowsPerCta - 1) / kMergeRowsPerCta));
    cfg.blockDim = dim3(32 * kMergeRowsPerCta);
    cfg.stream = r.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelExC(&cfg, inst.merge, margs);
    if (err != cudaSuccess) return fail(PA_ERR_CUDA, "merge launch: %s", cudaGetErrorString(err));
  }
  return launch_error("prefill");
}

// ---- scratch for pa_decode_split_static ------------------------------------------
// Callers that cannot allocate device memory get their split-decode scratch
// (ticket counters + per-partition partials) from this fixed array instead of
// a workspace argument. It is part of the library's device image: every GPU
// that loads the library holds these bytes until the process exits.
constexpr size_t kStaticScratchBytes = PA_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_static_split_scratch[kStaticScratchBytes];

// Device address of the array in the current context. In host code the
// array's name is only a host-side stand-in, so the address is fetched with
// cudaGetSymbolAddress once per context (with that context's device current)
// and cached, keyed by the current driver context: an address belongs to the
// context it was taken in.
CUcontext current_context() {
  using Fn = CUresult (*)(CUcontext*);
  static Fn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<Fn>(p);
    return static_cast<Fn>(nullptr);
  }();
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

pa_status_t static_scratch_address(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(err));
  if (dev < 0 || dev >= kMaxDevices) return fail(PA_ERR_UNSUPPORTED, "device %d >= %d", dev, kMaxDevices);
  struct Entry {
    CUcontext ctx;
    void* addr;
  };
  static std::mutex mu;
  static std::vector<Entry> cache;
  std::lock_guard<std::mutex> lock(mu);
  CUcontext ctx = current_context();
  for (const Entry& e : cache) {
    if (ctx != nullptr && e.ctx == ctx) {
      *out = e.addr;
      return PA_OK;
    }
  }
  // First use in this context (or no context current yet: the runtime call
  // below then sets up and makes current the device's primary context).
  void* p = nullptr;
  err = cudaGetSymbolAddress(&p, g_static_split_scratch);
  if (err != cudaSuccess || p == nullptr)
    return fail(PA_ERR_CUDA, "cudaGetSymbolAddress(static scratch): %s", cudaGetErrorString(err));
  ctx = current_context();
  if (ctx == nullptr) return fail(PA_ERR_CUDA, "no current CUDA context");
  cache.push_back(Entry{ctx, p});
  *out = p;
  return PA_OK;
}

}  // namespace
}  // namespace pagedkv

using namespace pagedkv;

extern "C" {

pa_status_t pa_decode(const void* q, const void* k_pool, const void* v_pool,
                      const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                      int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                      int num_blocks, int max_blocks_per_seq, float scale, pa_dtype_t dtype,
                      void* out, uint32_t* dev_err, void* stream) {
  PA_NVTX_RANGE("pa_decode");
  DecodeReq r{q, k_pool, v_pool, block_tables, context_lens, num_seqs, num_q_heads, num_kv_heads,
              head_dim, block_size, num_blocks, max_blocks_per_seq, scale, dtype, out, dev_err,
              static_cast<cudaStream_t>(stream)};
  return run_decode(r, false, 0, nullptr, 0);
}

size_t pa_decode_split_workspace_size(int num_seqs, int num_q_heads, int head_dim, int block_size,
                                      int max_blocks_per_seq, int partition_tokens) {
  if (num_seqs < 0 || num_q_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      max_blocks_per_seq <= 0 || partition_tokens <= 0 || partition_tokens % block_size != 0)
    return 0;
  return split_layout(num_seqs, num_q_heads, head_dim, block_size, max_blocks_per_seq,
                      partition_tokens)
      .total;
}

pa_status_t pa_decode_split_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  PA_NVTX_RANGE("pa_decode_split_workspace_init");
  if (workspace == nullptr || workspace_bytes < kWorkspaceHeader)
    return fail(PA_ERR_INVALID_ARG, "workspace must hold at least %zu bytes", kWorkspaceHeader);
  cudaError_t err =
      cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "workspace init: %s", cudaGetErrorString(err));
  return ok();
}

pa_status_t pa_decode_split(const void* q, const void* k_pool, const void* v_pool,
                            const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                            int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                            int num_blocks, int max_blocks_per_seq, float scale, pa_dtype_t dtype,
                            int partition_tokens, void* workspace, size_t workspace_bytes,
                            void* out, uint32_t* dev_err, void* stream) {
  PA_NVTX_RANGE("pa_decode_split");
  DecodeReq r{q, k_pool, v_pool, block_tables, context_lens, num_seqs, num_q_heads, num_kv_heads,
              head_dim, block_size, num_blocks, max_blocks_per_seq, scale, dtype, out, dev_err,
              static_cast<cudaStream_t>(stream)};
  return run_decode(r, true, partition_tokens, workspace, workspace_bytes);
}

pa_status_t pa_decode_split_static(const void* q, const void* k_pool, const void* v_pool,
                                   const int32_t* block_tables, const int32_t* context_lens,
                                   int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                   int block_size, int num_blocks, int max_blocks_per_seq,
                                   float scale, pa_dtype_t dtype, int partition_tokens, void* out,
                                   uint32_t* dev_err, void* stream) {
  PA_NVTX_RANGE("pa_decode_split_static");
  DecodeReq r{q, k_pool, v_pool, block_tables, context_lens, num_seqs, num_q_heads, num_kv_heads,
              head_dim, block_size, num_blocks, max_blocks_per_seq, scale, dtype, out, dev_err,
              static_cast<cudaStream_t>(stream)};
  // Everything that can be checked on the host is checked before the device
  // is touched, the scratch size included.
  DecodeInstance inst;
  pa_status_t st = validate_and_pick(r, &inst);
  if (st != PA_OK) return st;
  if (partition_tokens <= 0 || partition_tokens % block_size != 0)
    return fail(PA_ERR_INVALID_ARG, "partition_tokens (%d) must be a positive multiple of block_size",
                partition_tokens);
  if (num_seqs == 0) return ok();
  const SplitLayout layout = split_layout(num_seqs, num_q_heads, head_dim, block_size,
                                         max_blocks_per_seq, partition_tokens);
  const size_t need = layout.total;
  if (need > kStaticScratchBytes)
    return fail(PA_ERR_INVALID_ARG,
                "pa_decode_split_static needs %zu bytes of scratch for these sizes but its static "
                "scratch holds %zu; use pa_decode_split with a caller workspace or a larger "
                "partition_tokens",
                need, kStaticScratchBytes);
  void* scratch = nullptr;
  st = static_scratch_address(&scratch);
  if (st != PA_OK) return st;
  // The array keeps whatever the last call left; the control header must
  // start at zero. run_decode clears it on the stream after its own checks
  // (sequence count, PAGEDKV_VALIDATE), so a refused call writes nothing.
  return run_decode(r, true, partition_tokens, scratch, kStaticScratchBytes, nullptr,
                    /*clear_header=*/true);
}

pa_status_t pa_decode_split_static_fill_header(uint8_t byte, void* stream) {
  void* scratch = nullptr;
  pa_status_t st = static_scratch_address(&scratch);
  if (st != PA_OK) return st;
  const cudaError_t err = cudaMemsetAsync(scratch, byte, kWorkspaceHeader, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "filling the static header: %s", cudaGetErrorString(err));
  return ok();
}

size_t pa_decode_shared_prefix_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads,
                                              int head_dim, int block_size,
                                              int max_blocks_per_seq, int partition_tokens) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      max_blocks_per_seq <= 0 || partition_tokens <= 0 || partition_tokens % block_size != 0)
    return 0;
  return prefix_layout(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                       max_blocks_per_seq, partition_tokens)
      .ex.total;
}

pa_status_t pa_decode_shared_prefix(const void* q, const void* k_pool, const void* v_pool,
                                    const int32_t* block_tables, const int32_t* context_lens,
                                    int num_seqs, int num_q_heads, int num_kv_heads,
                                    int head_dim, int block_size, int num_blocks,
                                    int max_blocks_per_seq, float scale, pa_dtype_t dtype,
                                    int partition_tokens, int num_groups,
                                    const int32_t* group_offsets, const int32_t* group_members,
                                    const int32_t* group_blocks, void* workspace,
                                    size_t workspace_bytes, void* out, uint32_t* dev_err,
                                    void* stream) {
  PA_NVTX_RANGE("pa_decode_shared_prefix");
  DecodeReq r{q, k_pool, v_pool, block_tables, context_lens, num_seqs, num_q_heads, num_kv_heads,
              head_dim, block_size, num_blocks, max_blocks_per_seq, scale, dtype, out, dev_err,
              static_cast<cudaStream_t>(stream)};
  return run_shared_prefix(r, partition_tokens, num_groups, group_offsets, group_members,
                           group_blocks, workspace, workspace_bytes);
}

pa_status_t pa_decode_split_window(const void* q, const void* k_pool, const void* v_pool,
                                   const int32_t* block_tables, const int32_t* context_lens,
                                   int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                   int block_size, int num_blocks, int max_blocks_per_seq,
                                   float scale, pa_dtype_t dtype, int partition_tokens, int window,
                                   void* workspace, size_t workspace_bytes, void* out,
                                   uint32_t* dev_err, void* stream) {
  PA_NVTX_RANGE("pa_decode_split_window");
  if (window < 1) return fail(PA_ERR_INVALID_ARG, "window must be >= 1");
  DecodeReq r{q, k_pool, v_pool, block_tables, context_lens, num_seqs, num_q_heads, num_kv_heads,
              head_dim, block_size, num_blocks, max_blocks_per_seq, scale, dtype, out, dev_err,
              static_cast<cudaStream_t>(stream)};
  SplitExtras ex;
  ex.window = window;
  return run_decode(r, true, partition_tokens, workspace, workspace_bytes, &ex);
}

size_t pa_prefill_workspace_size(int num_seqs, int total_q, int num_q_heads, int num_kv_heads,
                                 int head_dim, int block_size, int max_blocks_per_seq,
                                 int partition_tokens) {
  if (num_seqs < 0 || total_q < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      block_size <= 0 || max_blocks_per_seq <= 0 || partition_tokens <= 0 ||
      partition_tokens % block_size != 0)
    return 0;
  return prefill_layout(num_seqs, total_q, num_q_heads, num_kv_heads, head_dim, block_size,
                        max_blocks_per_seq, partition_tokens)
      .total;
}

pa_status_t pa_prefill(const void* q, const void* k_pool, const void* v_pool,
                       const int32_t* block_tables, const int32_t* context_lens,
                       const int32_t* query_lens, int num_seqs, int total_q, int num_q_heads,
                       int num_kv_heads, int head_dim, int block_size, int num_blocks,
                       int max_blocks_per_seq, float scale, pa_dtype_t dtype,
                       int partition_tokens, void* workspace, size_t workspace_bytes, void* out,
                       uint32_t* dev_err, void* stream) {
  PA_NVTX_RANGE("pa_prefill");
  // validate_and_pick checks the device-side shapes; context_lens here is a
  // host array, so a placeholder non-null device pointer is not needed.
  DecodeReq r{q, k_pool, v_pool, block_tables, context_lens, num_seqs, num_q_heads, num_kv_heads,
              head_dim, block_size, num_blocks, max_blocks_per_seq, scale, dtype, out, dev_err,
              static_cast<cudaStream_t>(stream)};
  return run_prefill(r, context_lens, query_lens, total_q, partition_tokens, workspace,
                     workspace_bytes);
}

pa_status_t pa_prefill_plan(const int32_t* context_lens, const int32_t* query_lens, int num_seqs,
                            int num_q_heads, int num_kv_heads, int block_size, int partition_tokens,
                            int max_ctas, int32_t* items_out, int max_items, int* num_items,
                            int* num_ctas) {
  return prefill_plan(context_lens, query_lens, num_seqs, num_q_heads, num_kv_heads, block_size,
                      partition_tokens, max_ctas, items_out, max_items, num_items, num_ctas);
}

}  // extern "C"
