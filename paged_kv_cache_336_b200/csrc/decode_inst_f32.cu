// fp32 instances of the paged decode kernel (CUDA-core path).
#include "decode_dispatch.h"
#include "decode_kernel.cuh"
#include "decode_stream_kernel.cuh"

namespace pagedkv {

template <int BS, int D, int G>
static DecodeInstance make_f32() {
  using Cfg = DecodeCfg<float, BS, D, G>;
  DecodeInstance r;
  r.kernel = reinterpret_cast<const void*>(&paged_decode_kernel<Cfg>);
  r.merge = reinterpret_cast<const void*>(&lse_merge_kernel<float, D>);
  r.threads = Cfg::kThreads;
  r.fixed_smem = Cfg::kFixedSmem;
  r.stages = Cfg::NS;
  r.name = "simt_f32";
  for (DecodeInstance::Stream& st : r.stream) {
    st.kernel = reinterpret_cast<const void*>(&paged_decode_stream_kernel<Cfg>);
    st.threads = Cfg::kThreads;
    st.fixed_smem = StreamCfg<Cfg>::kFixedSmem;
    st.warps = Cfg::W;
  }
  return r;
}

template <int BS, int D>
static bool pick_group(int group, DecodeInstance* out) {
  switch (group) {
    case 1: *out = make_f32<BS, D, 1>(); return true;
    case 2: *out = make_f32<BS, D, 2>(); return true;
    case 4: *out = make_f32<BS, D, 4>(); return true;
    case 8: *out = make_f32<BS, D, 8>(); return true;
    default: return false;
  }
}

bool find_decode_f32(int head_dim, int block_size, int group, DecodeInstance* out) {
  if (block_size == 16 && head_dim == 64) return pick_group<16, 64>(group, out);
  if (block_size == 16 && head_dim == 128) return pick_group<16, 128>(group, out);
  if (block_size == 32 && head_dim == 64) return pick_group<32, 64>(group, out);
  if (block_size == 32 && head_dim == 128) return pick_group<32, 128>(group, out);
  return false;
}

}  // namespace pagedkv
