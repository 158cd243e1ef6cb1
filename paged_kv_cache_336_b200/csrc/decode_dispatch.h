// Registry of compiled decode-kernel instances (filled by decode_inst_*.cu).
#pragma once

#include <cstdint>

#include "pagedkv.h"

namespace pagedkv {

struct DecodeInstance {
  const void* kernel = nullptr;  // paged_decode_kernel<Cfg> (whole-context decode)
  const void* merge = nullptr;   // lse_merge_kernel<T, D>
  int threads = 0;
  int fixed_smem = 0;            // dynamic smem bytes before the prefix array
  int stages = 0;
  const char* name = "";
  // Split decode: paged_decode_stream_kernel<Cfg> (balanced pieces per warp),
  // in two CTA shapes: [0] the long-context one, [1] a smaller one that
  // shares SMs with a concurrent kernel (the shared-prefix pass).
  struct Stream {
    const void* kernel = nullptr;
    int threads = 0;
    int fixed_smem = 0;          // dynamic smem bytes before the per-sequence arrays
    int warps = 0;
  } stream[2];
};

// Each returns false when (head_dim, block_size, group) has no instance.
bool find_decode_f32(int head_dim, int block_size, int group, DecodeInstance* out);
// deep: the CTA shape for long contexts (see decode_inst_bf16.cu).
bool find_decode_bf16_mma(int head_dim, int block_size, bool deep, DecodeInstance* out);

struct PrefixInstance {
  const void* kernel = nullptr;  // prefix_decode_kernel<PrefixCfg<BS, D>> (or a prefill kernel)
  int threads = 0;
  int smem = 0;
  int rows = 64;                 // query rows (tokens x group heads) per tile
  int tiles = 1;                 // tiles per CTA
  bool q_map = false;            // takes a 3-D tensor map of q after the pool maps
};

// Shared-prefix pass kernels (bf16); false when (head_dim, block_size) has none.
bool find_prefix_bf16(int head_dim, int block_size, PrefixInstance* out);
// Paged prefill kernels (bf16); same shapes, same instance record. tcgen05:
// the 128-row tensor-memory kernel; otherwise the 64-row mma.sync kernel.
bool find_prefill_bf16(int head_dim, int block_size, bool tcgen05, PrefixInstance* out);
// tcgen05 shared-prefix pass: the prefill kernel with one 128-row tile per CTA.
bool find_tc_prefix_bf16(int head_dim, int block_size, PrefixInstance* out);

}  // namespace pagedkv
