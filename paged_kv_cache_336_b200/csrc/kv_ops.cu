// KV-append scatter and whole-block copy (copy-on-write data movement), with
// their C-ABI entry points (see include/pagedkv.h).
//
// * Append: decode writes each new token's K and V into its slot in the partly
//   filled tail block ("What is PagedAttention?", How It Works / Map Logical
//   to Physical Blocks; "PagedAttention: Optimizing KV Cache in vLLM",
//   section 4, step 3: the write proceeds on the private block).
// * Copy: the private block receives the shared block's contents (same
//   section, step 3); the whole block is copied.
//
// * Swap: whole blocks to and from page-locked host memory when a sequence is
//   preempted ("What is PagedAttention?", How It Works: allocation failure is
//   met by admission control, preemption, swap or rejection).
//
// All are copies moved as 16-byte vectors; every index is checked on the
// device and an out-of-range one is reported and skipped.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdlib>
#include <unordered_set>
#include <vector>
#include <cstdint>

#include "device_common.cuh"
#include "pa_internal.h"

namespace pagedkv {
namespace {

// One thread per 16-byte unit of (token, kv head, row unit); K and V together.
__global__ void __launch_bounds__(256)
    kv_append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                     const int64_t* __restrict__ slots, int num_tokens, int num_kv_heads,
                     int units_per_row, int block_size, int64_t num_slots, uint4* k_pool,
                     uint4* v_pool, uint32_t* dev_err) {
  const int64_t per_token = static_cast<int64_t>(num_kv_heads) * units_per_row;
  const int64_t total = per_token * num_tokens;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / per_token;
    const int64_t rem = i - t * per_token;
    const int64_t h = rem / units_per_row;
    const int64_t u = rem - h * units_per_row;
    const int64_t slot = slots[t];
    if (slot < 0) continue;  // padding
    if (slot >= num_slots) {
      if (rem == 0) report(dev_err, PA_DEVERR_SLOT);
      continue;
    }
    const int64_t blk = slot / block_size;
    const int64_t off = slot - blk * block_size;
    const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * units_per_row + u;
    k_pool[dst] = k_new[i];
    v_pool[dst] = v_new[i];
  }
}

// grid.y walks pairs, grid.x x blockDim.x walks the 16-byte units of a block.
constexpr int kCopyUnroll = 4;  // 16-byte units of K and of V in flight per thread

__global__ void __launch_bounds__(256)
    copy_blocks_kernel(uint4* k_pool, uint4* v_pool, const int64_t* __restrict__ pairs,
                       int num_pairs, int64_t units_per_block, int num_blocks,
                       uint32_t* dev_err) {
  for (int pr = blockIdx.y; pr < num_pairs; pr += gridDim.y) {
    const int64_t src = pairs[2 * static_cast<int64_t>(pr)];
    const int64_t dst = pairs[2 * static_cast<int64_t>(pr) + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
      if (blockIdx.x == 0 && threadIdx.x == 0) report(dev_err, PA_DEVERR_COPY_PAIR);
      continue;
    }
    if (src == dst) continue;
    const uint4* ks = k_pool + src * units_per_block;
    const uint4* vs = v_pool + src * units_per_block;
    uint4* kd = k_pool + dst * units_per_block;
    uint4* vd = v_pool + dst * units_per_block;
    // Each thread loads kCopyUnroll units of K and of V before storing any:
    // source and destination lie in the same pool, so the compiler would not
    // move a later load above an earlier store, and a plain loop waits out a
    // memory round trip per unit. A pair's source and destination are
    // different blocks, and no destination is another pair's source.
    const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x * kCopyUnroll;
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x * kCopyUnroll + threadIdx.x;
         base < units_per_block; base += step) {
      uint4 kr[kCopyUnroll], vr[kCopyUnroll];
#pragma unroll
      for (int i = 0; i < kCopyUnroll; ++i) {
        const int64_t u = base + static_cast<int64_t>(i) * blockDim.x;
        if (u < units_per_block) {
          kr[i] = ks[u];
          vr[i] = vs[u];
        }
      }
#pragma unroll
      for (int i = 0; i < kCopyUnroll; ++i) {
        const int64_t u = base + static_cast<int64_t>(i) * blockDim.x;
        if (u < units_per_block) {
          kd[u] = kr[i];
          vd[u] = vr[i];
        }
      }
    }
  }
}

// Whole-block copies between two differently indexed block arrays (device
// pool <-> mapped host buffer). grid.y walks pairs; pair p copies block
// pairs[2p] of `src` to block pairs[2p+1] of `dst`, K and V.
__global__ void __launch_bounds__(256)
    swap_blocks_kernel(const uint4* src_k, const uint4* src_v, uint4* dst_k, uint4* dst_v,
                       const int64_t* __restrict__ pairs, int num_pairs, int64_t units_per_block,
                       int src_blocks, int dst_blocks, uint32_t* dev_err) {
  for (int pr = blockIdx.y; pr < num_pairs; pr += gridDim.y) {
    const int64_t src = pairs[2 * static_cast<int64_t>(pr)];
    const int64_t dst = pairs[2 * static_cast<int64_t>(pr) + 1];
    if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
      if (blockIdx.x == 0 && threadIdx.x == 0) report(dev_err, PA_DEVERR_COPY_PAIR);
      continue;
    }
    const uint4* ks = src_k + src * units_per_block;
    const uint4* vs = src_v + src * units_per_block;
    uint4* kd = dst_k + dst * units_per_block;
    uint4* vd = dst_v + dst * units_per_block;
    for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < units_per_block;
         u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
      kd[u] = ks[u];
      vd[u] = vs[u];
    }
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address of a page-locked, mapped host buffer.
pa_status_t mapped(void* host, void** dev) {
  cudaError_t err = cudaHostGetDevicePointer(dev, host, 0);
  if (err != cudaSuccess) {
    cudaGetLastError();
    return fail(PA_ERR_INVALID_ARG, "host buffer is not page-locked and mapped: %s",
                cudaGetErrorString(err));
  }
  return PA_OK;
}

pa_status_t launch_swap(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                        const int64_t* pairs, int num_pairs, size_t block_bytes, int src_blocks,
                        int dst_blocks, uint32_t* dev_err, cudaStream_t stream) {
  if (num_pairs < 0) return fail(PA_ERR_INVALID_ARG, "num_pairs < 0");
  if (num_pairs == 0) return ok();
  if (src_k == nullptr || src_v == nullptr || dst_k == nullptr || dst_v == nullptr || pairs == nullptr)
    return fail(PA_ERR_INVALID_ARG, "NULL pointer");
  if (block_bytes == 0 || block_bytes % 16 != 0 || src_blocks <= 0 || dst_blocks <= 0)
    return fail(PA_ERR_INVALID_ARG, "bad block_bytes or block counts");
  if (!aligned16(src_k) || !aligned16(src_v) || !aligned16(dst_k) || !aligned16(dst_v))
    return fail(PA_ERR_INVALID_ARG, "buffers must be 16-byte aligned");
  const int64_t upb = static_cast<int64_t>(block_bytes / 16);
  const int gx = static_cast<int>(std::min<int64_t>((upb + 1023) / 1024, 64));
  const int gy = std::min(num_pairs, 65535);
  swap_blocks_kernel<<<dim3(gx, gy), 256, 0, stream>>>(
      static_cast<const uint4*>(src_k), static_cast<const uint4*>(src_v), static_cast<uint4*>(dst_k),
      static_cast<uint4*>(dst_v), pairs, num_pairs, upb, src_blocks, dst_blocks, dev_err);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "swap launch: %s", cudaGetErrorString(err));
  return ok();
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

}  // namespace
bool validate_copy_pairs() {
  static const bool enabled = [] {
    const char* e = std::getenv("PAGEDKV_VALIDATE");
    return e != nullptr && e[0] == '1';
  }();
  return enabled;
}

}  // namespace pagedkv

using namespace pagedkv;

extern "C" {

pa_status_t pa_kv_append(const void* k_new, const void* v_new, const int64_t* slot_mapping,
                         int num_tokens, int num_kv_heads, int head_dim, int block_size,
                         int num_blocks, pa_dtype_t dtype, void* k_pool, void* v_pool,
                         uint32_t* dev_err, void* stream) {
  PA_NVTX_RANGE("pa_kv_append");
  if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "num_tokens < 0");
  if (num_tokens == 0) return ok();
  if (k_new == nullptr || v_new == nullptr || slot_mapping == nullptr || k_pool == nullptr ||
      v_pool == nullptr)
    return fail(PA_ERR_INVALID_ARG, "NULL pointer");
  if (dtype != PA_F32 && dtype != PA_BF16) return fail(PA_ERR_INVALID_ARG, "unknown dtype");
  if (num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
    return fail(PA_ERR_INVALID_ARG, "sizes must be positive");
  const int eb = dtype == PA_F32 ? 4 : 2;
  if ((head_dim * eb) % 16 != 0) return fail(PA_ERR_INVALID_ARG, "head_dim * element size must be a multiple of 16");
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) || !aligned16(v_pool))
    return fail(PA_ERR_INVALID_ARG, "k_new, v_new and pools must be 16-byte aligned");
  const int upr = head_dim * eb / 16;
  const int64_t total = static_cast<int64_t>(num_tokens) * num_kv_heads * upr;
  const int64_t want = (total + 255) / 256;
  const int grid = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(sm_count()) * 8));
  kv_append_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), slot_mapping, num_tokens,
      num_kv_heads, upr, block_size, static_cast<int64_t>(num_blocks) * block_size,
      static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), dev_err);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "kv_append launch: %s", cudaGetErrorString(err));
  return ok();
}

pa_status_t pa_copy_blocks(void* k_pool, void* v_pool, const int64_t* src_dst_pairs, int num_pairs,
                           size_t block_bytes, int num_blocks, uint32_t* dev_err, void* stream) {
  PA_NVTX_RANGE("pa_copy_blocks");
  if (num_pairs < 0) return fail(PA_ERR_INVALID_ARG, "num_pairs < 0");
  if (num_pairs == 0) return ok();
  if (k_pool == nullptr || v_pool == nullptr || src_dst_pairs == nullptr)
    return fail(PA_ERR_INVALID_ARG, "NULL pointer");
  if (block_bytes == 0 || block_bytes % 16 != 0)
    return fail(PA_ERR_INVALID_ARG, "block_bytes must be a positive multiple of 16");
  if (num_blocks <= 0) return fail(PA_ERR_INVALID_ARG, "num_blocks must be positive");
  if (!aligned16(k_pool) || !aligned16(v_pool)) return fail(PA_ERR_INVALID_ARG, "pools must be 16-byte aligned");
  if (validate_copy_pairs()) {
    // PAGEDKV_VALIDATE=1: the pairs come to the host (synchronously) and a list
    // whose result would depend on the order of the copies is refused.
    std::vector<int64_t> h(2 * static_cast<size_t>(num_pairs));
    cudaError_t e = cudaMemcpyAsync(h.data(), src_dst_pairs, h.size() * 8, cudaMemcpyDeviceToHost,
                                    static_cast<cudaStream_t>(stream));
    if (e == cudaSuccess) e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "PAGEDKV_VALIDATE copy failed: %s", cudaGetErrorString(e));
    std::unordered_set<int64_t> dst;
    for (int i = 0; i < num_pairs; ++i) {
      const int64_t a = h[2 * i], b = h[2 * i + 1];
      if (a < 0 || a >= num_blocks || b < 0 || b >= num_blocks)
        return fail(PA_ERR_INVALID_ARG, "copy pair %d (%lld, %lld) outside [0, %d)", i, (long long)a,
                    (long long)b, num_blocks);
      if (!dst.insert(b).second)
        return fail(PA_ERR_INVALID_ARG, "copy pairs: destination %lld appears twice", (long long)b);
    }
    for (int i = 0; i < num_pairs; ++i)
      if (dst.count(h[2 * i]))
        return fail(PA_ERR_INVALID_ARG, "copy pairs: block %lld is both a source and a destination",
                    (long long)h[2 * i]);
  }
  const int64_t upb = static_cast<int64_t>(block_bytes / 16);
  const int gx = static_cast<int>(std::min<int64_t>((upb + 256 * kCopyUnroll - 1) / (256 * kCopyUnroll), 64));
  const int gy = std::min(num_pairs, 65535);
  copy_blocks_kernel<<<dim3(gx, gy), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), src_dst_pairs, num_pairs, upb,
      num_blocks, dev_err);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "copy_blocks launch: %s", cudaGetErrorString(err));
  return ok();
}

pa_status_t pa_swap_out(const void* k_pool, const void* v_pool, void* host_k, void* host_v,
                        const int64_t* pairs, int num_pairs, size_t block_bytes, int num_blocks,
                        int num_host_slots, uint32_t* dev_err, void* stream) {
  PA_NVTX_RANGE("pa_swap_out");
  if (num_pairs == 0) return ok();
  if (host_k == nullptr || host_v == nullptr) return fail(PA_ERR_INVALID_ARG, "NULL host buffer");
  void *dk = nullptr, *dv = nullptr;
  pa_status_t st = mapped(host_k, &dk);
  if (st != PA_OK) return st;
  if ((st = mapped(host_v, &dv)) != PA_OK) return st;
  return launch_swap(k_pool, v_pool, dk, dv, pairs, num_pairs, block_bytes, num_blocks,
                     num_host_slots, dev_err, static_cast<cudaStream_t>(stream));
}

pa_status_t pa_swap_in(const void* host_k, const void* host_v, void* k_pool, void* v_pool,
                       const int64_t* pairs, int num_pairs, size_t block_bytes, int num_blocks,
                       int num_host_slots, uint32_t* dev_err, void* stream) {
  PA_NVTX_RANGE("pa_swap_in");
  if (num_pairs == 0) return ok();
  if (host_k == nullptr || host_v == nullptr) return fail(PA_ERR_INVALID_ARG, "NULL host buffer");
  void *dk = nullptr, *dv = nullptr;
  pa_status_t st = mapped(const_cast<void*>(host_k), &dk);
  if (st != PA_OK) return st;
  if ((st = mapped(const_cast<void*>(host_v), &dv)) != PA_OK) return st;
  return launch_swap(dk, dv, k_pool, v_pool, pairs, num_pairs, block_bytes, num_host_slots,
                     num_blocks, dev_err, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
