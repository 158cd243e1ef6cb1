// bf16 instances of the paged decode kernel (tensor-core path, groups 1..16).
//
// Two CTA shapes per (block size, head_dim), chosen by the host:
//  * wide: 4 warps x 2 ring stages (64 KB of ring at head_dim 128; three CTAs
//    and 12 warps per SM). Best measured for contexts up to a few thousand
//    tokens: MHA batch 64 and GQA batch 256 stream at ~96.7% of the measured
//    HBM copy peak against ~92% for 4 x 3.
//  * deep: 2 warps x 3 stages (48 KB; four CTAs per SM). Best measured for
//    131072-token contexts in 512-token partitions (96.9% against 91.7% for
//    wide): each warp walks more units of an item per fill and drain.
#include <cstdlib>
#include <cstring>

#include "decode_dispatch.h"
#include "decode_kernel.cuh"
#include "decode_stream_kernel.cuh"
#include "prefill_kernel.cuh"
#include "prefix_kernel.cuh"
#include "tc_prefill_kernel.cuh"

namespace pagedkv {

template <int BS, int D, int W, int NS>
static DecodeInstance make_bf16(const char* name) {
  using Cfg = DecodeCfg<__nv_bfloat16, BS, D, 0, W, NS>;
  DecodeInstance r;
  r.kernel = reinterpret_cast<const void*>(&paged_decode_kernel<Cfg>);
  r.merge = reinterpret_cast<const void*>(&lse_merge_kernel<__nv_bfloat16, D>);
  r.threads = Cfg::kThreads;
  r.fixed_smem = Cfg::kFixedSmem;
  r.stages = Cfg::NS;
  r.name = name;
  return r;
}

template <int BS, int D, int W, int NS>
static void add_stream(DecodeInstance* r, int which) {
  using Cfg = DecodeCfg<__nv_bfloat16, BS, D, 0, W, NS>;
  DecodeInstance::Stream& st = r->stream[which];
  st.kernel = reinterpret_cast<const void*>(&paged_decode_stream_kernel<Cfg>);
  st.threads = Cfg::kThreads;
  st.fixed_smem = StreamCfg<Cfg>::kFixedSmem;
  st.warps = Cfg::W;
}

// Balanced split-decode CTA shapes (warps x ring stages of 16-token K+V
// units); every shape keeps 192 KB of ring per SM at head_dim 128.
//  [0] long contexts: 8 x 3, one CTA per SM: its 8 warps are the 8 KV heads
//      of one group in the long-context batches, reading the same blocks
//      together; measured on the 131072-token batch at 0.988 of the HBM copy
//      peak against 0.962-0.970 for 4 x 2, 4 x 3 and 2 x 3 at the same clock.
//  [1] the shared-prefix suffix pass, which starts beside the prefix kernel:
//      4 x 2 (64 KB CTAs fit next to its CTAs); the whole prefix_cow call
//      measured 75.7 us against 77.7 for 2 x 3 and 84.0 on partition tickets.
// PAGEDKV_STREAM_SHAPE ("4x3", "4x2", "2x3", "8x3") sets both for measurements.
template <int BS, int D>
static void pick_stream(DecodeInstance* r) {
  const char* e = std::getenv("PAGEDKV_STREAM_SHAPE");
  if constexpr (D == 256) {
    add_stream<BS, D, 4, 2>(r, 0);
    add_stream<BS, D, 4, 2>(r, 1);
  } else {
    if (e != nullptr && std::strcmp(e, "4x2") == 0) {
      add_stream<BS, D, 4, 2>(r, 0);
      add_stream<BS, D, 4, 2>(r, 1);
    } else if (e != nullptr && std::strcmp(e, "2x3") == 0) {
      add_stream<BS, D, 2, 3>(r, 0);
      add_stream<BS, D, 2, 3>(r, 1);
    } else if (e != nullptr && std::strcmp(e, "4x3") == 0) {
      add_stream<BS, D, 4, 3>(r, 0);
      add_stream<BS, D, 4, 3>(r, 1);
    } else if (e != nullptr && std::strcmp(e, "8x3") == 0) {
      add_stream<BS, D, 8, 3>(r, 0);
      add_stream<BS, D, 8, 3>(r, 1);
    } else {
      add_stream<BS, D, 8, 3>(r, 0);
      add_stream<BS, D, 4, 2>(r, 1);
    }
  }
}

template <int BS, int D>
static void pick(bool deep, DecodeInstance* out) {
  if constexpr (D == 256) {
    // 16 KB stages: the default shape (4 warps x 2 stages) for both.
    *out = make_bf16<BS, D, 0, 0>("mma_bf16");
  } else {
    if (deep) *out = make_bf16<BS, D, 2, 3>("mma_bf16_deep");
    else *out = make_bf16<BS, D, 4, 2>("mma_bf16_wide");
  }
  pick_stream<BS, D>(out);
}

bool find_decode_bf16_mma(int head_dim, int block_size, bool deep, DecodeInstance* out) {
  if (block_size == 16 && head_dim == 64) { pick<16, 64>(deep, out); return true; }
  if (block_size == 16 && head_dim == 128) { pick<16, 128>(deep, out); return true; }
  if (block_size == 16 && head_dim == 256) { pick<16, 256>(deep, out); return true; }
  if (block_size == 32 && head_dim == 64) { pick<32, 64>(deep, out); return true; }
  if (block_size == 32 && head_dim == 128) { pick<32, 128>(deep, out); return true; }
  if (block_size == 32 && head_dim == 256) { pick<32, 256>(deep, out); return true; }
  return false;
}

template <int BS, int D, int MINB>
static PrefixInstance make_prefix_minb() {
  using Cfg = PrefixCfg<BS, D, MINB>;
  PrefixInstance r;
  r.kernel = reinterpret_cast<const void*>(&prefix_decode_kernel<Cfg>);
  r.threads = Cfg::kThreads;
  r.smem = Cfg::kSmem;
  return r;
}

// The prefix kernel's registers are sized for two CTAs per SM: 168 per
// thread and no spills at head_dim 128, against 128 and 72 bytes of spills
// for three. Measured on the shared-prefix calls: prefix 92.3 against
// 96.4 us, prefix_cow 74.7 against 76.1. PAGEDKV_PREFIX_MINB=3 selects the
// three-CTA build.
template <int BS, int D>
static PrefixInstance make_prefix() {
  const char* e = std::getenv("PAGEDKV_PREFIX_MINB");
  if (e != nullptr && std::strcmp(e, "3") == 0) return make_prefix_minb<BS, D, 3>();
  return make_prefix_minb<BS, D, 2>();
}

bool find_prefix_bf16(int head_dim, int block_size, PrefixInstance* out) {
  if (block_size == 16 && head_dim == 64) { *out = make_prefix<16, 64>(); return true; }
  if (block_size == 16 && head_dim == 128) { *out = make_prefix<16, 128>(); return true; }
  if (block_size == 32 && head_dim == 64) { *out = make_prefix<32, 64>(); return true; }
  if (block_size == 32 && head_dim == 128) { *out = make_prefix<32, 128>(); return true; }
  return false;
}

template <int BS, int D>
static PrefixInstance make_prefill() {
  using Cfg = PrefixCfg<BS, D>;
  PrefixInstance r;
  r.kernel = reinterpret_cast<const void*>(&prefill_kernel<Cfg>);
  r.threads = Cfg::kThreads;
  r.smem = Cfg::kSmem;
  return r;
}

// tcgen05 prefill: two 128-row tiles per CTA sharing each K/V chunk (measured
// faster than one tile per CTA at two CTAs per SM).
constexpr int kTcPrefillTiles = 2;

template <int BS, int D, int TILES = kTcPrefillTiles, int HALVES = 1>
static PrefixInstance make_tc_prefill() {
  using Cfg = TcCfg<BS, D, TILES, HALVES>;
  PrefixInstance r;
  r.kernel = reinterpret_cast<const void*>(&tc_prefill_kernel<Cfg>);
  r.threads = Cfg::kThreads;
  r.smem = Cfg::kSmem;
  r.rows = Cfg::ROWS;
  r.tiles = Cfg::TILES;
  r.q_map = true;
  return r;
}

// Threads per query row in the tcgen05 softmax: PAGEDKV_PREFILL_HALVES=2
// splits each row's logits between two threads (16 softmax warps).
template <int BS, int D>
static PrefixInstance pick_prefill(bool tcgen05) {
  if (!tcgen05) return make_prefill<BS, D>();
  const char* e = std::getenv("PAGEDKV_PREFILL_HALVES");
  if (e != nullptr && std::strcmp(e, "2") == 0) return make_tc_prefill<BS, D, kTcPrefillTiles, 2>();
  return make_tc_prefill<BS, D>();
}

bool find_prefill_bf16(int head_dim, int block_size, bool tcgen05, PrefixInstance* out) {
  if (block_size == 16 && head_dim == 64) { *out = pick_prefill<16, 64>(tcgen05); return true; }
  if (block_size == 16 && head_dim == 128) { *out = pick_prefill<16, 128>(tcgen05); return true; }
  if (block_size == 32 && head_dim == 64) { *out = pick_prefill<32, 64>(tcgen05); return true; }
  if (block_size == 32 && head_dim == 128) { *out = pick_prefill<32, 128>(tcgen05); return true; }
  return false;
}

bool find_tc_prefix_bf16(int head_dim, int block_size, PrefixInstance* out) {
  if (block_size == 16 && head_dim == 64) { *out = make_tc_prefill<16, 64, 1>(); return true; }
  if (block_size == 16 && head_dim == 128) { *out = make_tc_prefill<16, 128, 1>(); return true; }
  if (block_size == 32 && head_dim == 64) { *out = make_tc_prefill<32, 64, 1>(); return true; }
  if (block_size == 32 && head_dim == 128) { *out = make_tc_prefill<32, 128, 1>(); return true; }
  return false;
}

}  // namespace pagedkv
