// bf16 instances of the paged decode kernel (tensor-core path, groups 1..16).
#include "decode_dispatch.h"
#include "decode_kernel.cuh"

namespace pagedkv {

template <int BS, int D, int G>
static DecodeInstance make_bf16(const char* name) {
  using Cfg = DecodeCfg<__nv_bfloat16, BS, D, G>;
  DecodeInstance r;
  r.kernel = reinterpret_cast<const void*>(&paged_decode_kernel<Cfg>);
  r.merge = reinterpret_cast<const void*>(&lse_merge_kernel<__nv_bfloat16, D>);
  r.threads = Cfg::kThreads;
  r.fixed_smem = Cfg::kFixedSmem;
  r.stages = Cfg::NS;
  r.name = name;
  return r;
}

bool find_decode_bf16_mma(int head_dim, int block_size, DecodeInstance* out) {
  if (block_size == 16 && head_dim == 64) { *out = make_bf16<16, 64, 0>("mma_bf16"); return true; }
  if (block_size == 16 && head_dim == 128) { *out = make_bf16<16, 128, 0>("mma_bf16"); return true; }
  if (block_size == 16 && head_dim == 256) { *out = make_bf16<16, 256, 0>("mma_bf16"); return true; }
  if (block_size == 32 && head_dim == 64) { *out = make_bf16<32, 64, 0>("mma_bf16"); return true; }
  if (block_size == 32 && head_dim == 128) { *out = make_bf16<32, 128, 0>("mma_bf16"); return true; }
  if (block_size == 32 && head_dim == 256) { *out = make_bf16<32, 256, 0>("mma_bf16"); return true; }
  return false;
}

}  // namespace pagedkv
