// Shared-prefix pass of pa_decode_shared_prefix (sm_100a, bf16).
//
// Sequences forked from one prompt hold the same physical blocks for the
// prompt ("PagedAttention: Optimizing KV Cache in vLLM", section 4, step 1).
// This kernel reads those blocks once per KV head for all of the group's
// query rows instead of once per sequence, and leaves one partial (running
// max, running sum, unnormalised accumulator) per (sequence, query head) per
// prefix partition; the split kernel covers each sequence's own blocks and
// the log-sum-exp merge joins both.
//
// One CTA per item = (group row chunk, KV head, prefix partition): a
// producer warp streams the partition's 16-token units (K and V tiles, 2-D
// TMA, 128-byte swizzle) into a CTA-wide ring of NS stages; four consumer
// warps each own 16 query rows (row r = member r / G, head r % G of the KV
// head's group) and all read every stage, so a tile crosses HBM once for up
// to 64 rows. Full barriers complete on the TMA byte count, empty barriers
// on the four consumer warps' arrivals. All waits are bounded.
#pragma once

#include "decode_kernel.cuh"

namespace pagedkv {

// Host-built description of one CTA's work (32 bytes).
struct PrefixItem {
  int32_t rep_seq;       // batch position whose block table holds the shared blocks
  int32_t member_begin;  // first member of this row chunk, index into members[]
  int32_t member_count;  // members in this chunk (member_count * group <= 64)
  int32_t block_begin;   // shared blocks [block_begin, block_end) of this partition
  int32_t block_end;
  int32_t kvh;
  int32_t part;          // partial slot of this partition
  int32_t pad;
};

struct PrefixArgs {
  DecodeArgs d;             // q, block tables, partial arrays, sizes, scale, dev_err
  const PrefixItem* items;  // [gridDim.x]
  const int32_t* members;   // batch positions, grouped
};

template <int BS_, int D_, int MINB_ = 2>
struct PrefixCfg {
  static constexpr int MINB = MINB_;  // resident CTAs per SM the registers are sized for
  using Mma = DecodeCfg<__nv_bfloat16, BS_, D_, 0, 4, 2>;  // unit geometry + per-warp math
  using Geo = typename Mma::Geo;
  static constexpr int BS = BS_;
  static constexpr int D = D_;
  static constexpr int UR = Mma::UR;
  static constexpr int UPB = Mma::UPB;
  static constexpr int CW = 4;                   // consumer warps (16 query rows each)
  static constexpr int kThreads = 32 * (CW + 1); // + one producer warp
  static constexpr int kStageBytes = 2 * Geo::kTileBytes;
  static constexpr int NS = cmin(8, cmax(2, 65536 / kStageBytes));
  static constexpr int kSmem = 1024 + NS * kStageBytes + 2 * NS * 8;
};

template <class Cfg>
__global__ void __launch_bounds__(Cfg::kThreads, Cfg::MINB)
    prefix_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const PrefixArgs pa) {
  using Geo = typename Cfg::Geo;
  constexpr int NS = Cfg::NS;
  constexpr int CW = Cfg::CW;
  constexpr int BS = Cfg::BS;
  constexpr int UR = Cfg::UR;
  constexpr int UPB = Cfg::UPB;
  constexpr int D = Cfg::D;
  const DecodeArgs& a = pa.d;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + NS * Cfg::kStageBytes);
  uint64_t* empty = full + NS;

  // The suffix kernel that follows is independent of this one: let it start.
  grid_dependents_launch();
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const PrefixItem it = pa.items[blockIdx.x];
  const int G = a.group;
  const int Hkv = a.num_kv_heads;
  const int nunits = (it.block_end - it.block_begin) * UPB;  // shared blocks are full

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], CW);
    }
    fence_barrier_init();
    tma_prefetch_descriptor(&tm_k);
    tma_prefetch_descriptor(&tm_v);
  }
  __syncthreads();

  if (warp == CW) {
    // ---- producer warp -----------------------------------------------------
    const uint64_t policy = l2_policy(a.l2_hint);
    const int32_t* bt = a.block_tables + static_cast<int64_t>(it.rep_seq) * a.max_blocks_per_seq +
                        it.block_begin;
    const int nblk = it.block_end - it.block_begin;
    int ids = (lane < nblk) ? bt[lane] : -1;
    int chunk = 0;
    for (int u = 0; u < nunits; ++u) {
      const int b = u / UPB;
      const int half = u - b * UPB;
      if ((b >> 5) != chunk) {  // next 32 block ids
        chunk = b >> 5;
        ids = (chunk * 32 + lane < nblk) ? bt[chunk * 32 + lane] : -1;
      }
      const int phys = __shfl_sync(0xffffffffu, ids, b & 31);
      const int stage = u % NS;
      const int use = u / NS;
      bool ok = true;
      if (use > 0) ok = mbar_wait_bounded(&empty[stage], (use - 1) & 1, a.dev_err);
      if (!__all_sync(0xffffffffu, ok)) break;  // consumers stopped; they time out too
      if (lane == 0) {
        if (phys >= 0 && phys < a.num_blocks) {
          uint8_t* kdst = ring + stage * Cfg::kStageBytes;
          uint8_t* vdst = kdst + Geo::kTileBytes;
          const int32_t y = (phys * Hkv + it.kvh) * BS + half * UR;
          mbar_arrive_expect_tx(&full[stage], 2 * Geo::kTileBytes);
#pragma unroll
          for (int c = 0; c < Geo::kChunks; ++c) {
            tma_load_2d(kdst + c * Geo::kChunkBytes, &tm_k, &full[stage], c * Geo::kBoxCols, y, policy);
            tma_load_2d(vdst + c * Geo::kChunkBytes, &tm_v, &full[stage], c * Geo::kBoxCols, y, policy);
          }
        } else {
          report(a.dev_err, PA_DEVERR_BLOCK_ID);
          mbar_arrive(&full[stage]);  // consumers read a stale stage; the error is reported
        }
      }
    }
    // Let in-flight copies land before the CTA can exit (bounded).
    if (nunits > 0) {
      const int last = nunits - 1;
      for (int u = max(0, last - NS + 1); u <= last; ++u)
        mbar_wait_bounded(&empty[u % NS], (u / NS) & 1, a.dev_err);
    }
    return;
  }

  // ---- consumer warps: rows 16*warp .. 16*warp+15 -------------------------------
  const int g = lane >> 2;
  const int r0 = warp * 16 + g;
  const int r1 = r0 + 8;
  const bool v0 = r0 < it.member_count * G;
  const bool v1 = r1 < it.member_count * G;
  const int s0 = v0 ? pa.members[it.member_begin + r0 / G] : 0;
  const int s1 = v1 ? pa.members[it.member_begin + r1 / G] : 0;
  const int64_t h0 = static_cast<int64_t>(it.kvh) * G + (r0 % G);
  const int64_t h1 = static_cast<int64_t>(it.kvh) * G + (r1 % G);
  const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(a.q);
  MmaWarp<typename Cfg::Mma> st;
  st.begin_rows(q + (static_cast<int64_t>(s0) * a.num_q_heads + h0) * D,
                q + (static_cast<int64_t>(s1) * a.num_q_heads + h1) * D, v0, v1, a.scale_log2, lane);
  const bool active = __any_sync(0xffffffffu, v0 || v1);
  bool timed_out = false;
  int u = 0;
  // Two units (32 tokens) per softmax step while at least two remain.
  for (; u + 1 < nunits && !timed_out; u += 2) {
    const int st0 = u % NS, st1 = (u + 1) % NS;
    bool ok = mbar_wait_bounded(&full[st0], (u / NS) & 1, a.dev_err);
    ok = ok && mbar_wait_bounded(&full[st1], ((u + 1) / NS) & 1, a.dev_err);
    if (!__all_sync(0xffffffffu, ok)) {
      timed_out = true;
      break;
    }
    if (active) {
      uint8_t* k0 = ring + st0 * Cfg::kStageBytes;
      uint8_t* k1 = ring + st1 * Cfg::kStageBytes;
      const uint8_t* kts[2] = {k0, k1};
      uint8_t* vts[2] = {k0 + Geo::kTileBytes, k1 + Geo::kTileBytes};
      st.template block_units<2>(kts, vts, 0, 2 * UR, lane);
    }
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&empty[st0]);
      mbar_arrive(&empty[st1]);
    }
  }
  for (; u < nunits && !timed_out; ++u) {
    const int stage = u % NS;
    const bool ok = mbar_wait_bounded(&full[stage], (u / NS) & 1, a.dev_err);
    if (!__all_sync(0xffffffffu, ok)) {
      timed_out = true;
      break;
    }
    if (active) {
      uint8_t* kt = ring + stage * Cfg::kStageBytes;
      st.block(kt, kt + Geo::kTileBytes, 0, UR, lane);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
  }
  if (timed_out) return;
  const int64_t pr0 = v0 ? (static_cast<int64_t>(s0) * a.num_q_heads + h0) * a.max_partitions + it.part : -1;
  const int64_t pr1 = v1 ? (static_cast<int64_t>(s1) * a.num_q_heads + h1) * a.max_partitions + it.part : -1;
  st.store_partials(a, pr0, pr1, lane);
}

}  // namespace pagedkv
