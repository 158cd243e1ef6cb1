// Paged prefill (chunked prefill) attention for sm_100a, bf16.
//
// A request's new tokens attend causally to its whole paged context: new
// token i of a sequence with context length ctx and q_len new tokens sits at
// position p = ctx - q_len + i and attends to tokens 0..p, reached through
// the block table like decode ("What is PagedAttention?", How It Works:
// prefill allocates enough blocks for the input; the table maps logical to
// physical blocks). Unlike decode, many queries share every KV tile, so the
// products are a real dense contraction.
//
// One CTA per item = (sequence, tile of 64 / G query tokens x G heads = 64
// query rows, KV head, KV partition). As in the shared-prefix pass, a
// producer warp streams the partition's 16-token K/V units (2-D TMA,
// 128-byte swizzle) into a CTA-wide ring; four consumer warps own 16 rows
// each and read every stage; each row masks tokens past its own position.
// A tile whose KV fits one partition writes its rows' outputs directly;
// otherwise each partition leaves partials that the log-sum-exp merge joins.
#pragma once

#include "prefix_kernel.cuh"

namespace pagedkv {

// Host-built description of one CTA's work (48 bytes).
struct PrefillItem {
  int32_t seq;          // batch position (block table row)
  int32_t q_begin;      // global index of the tile's first query token
  int32_t q_count;      // query tokens in the tile (q_count * group <= 64)
  int32_t p0;           // position of the tile's first query token
  int32_t block_begin;  // KV blocks [block_begin, block_end) of this partition
  int32_t block_end;
  int32_t kv_end;       // tokens past this are never attended by the tile (last position + 1)
  int32_t kvh;
  int32_t part;         // partial slot (KV partition index)
  int32_t final_out;    // 1: the tile has a single partition, write outputs directly
  int32_t q_head0;      // tcgen05 kernel: first head of the Q box (kvh * group; 0 for packed Q)
  int32_t out_begin;    // tcgen05 kernel: >= 0: output row j is out_tokens[out_begin + j]
};

struct PrefillArgs {
  DecodeArgs d;              // q, block tables, partials, out, sizes, scale, dev_err
  const PrefillItem* items;  // [gridDim.x], or [sched_off[gridDim.x]] with a schedule
  const int32_t* out_tokens; // output token (or sequence) of each item row; see out_begin
  // tcgen05 kernel: NULL, one item per CTA (item blockIdx.x); else CTA b runs
  // items [sched_off[b], sched_off[b + 1]) in order (a persistent launch).
  const int32_t* sched_off;
};

template <class Cfg>
__global__ void __launch_bounds__(Cfg::kThreads, 2)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const PrefillArgs pf) {
  using Geo = typename Cfg::Geo;
  constexpr int NS = Cfg::NS;
  constexpr int CW = Cfg::CW;
  constexpr int BS = Cfg::BS;
  constexpr int UR = Cfg::UR;
  constexpr int UPB = Cfg::UPB;
  constexpr int D = Cfg::D;
  const DecodeArgs& a = pf.d;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + NS * Cfg::kStageBytes);
  uint64_t* empty = full + NS;

  grid_dependents_launch();  // the merge grid may be scheduled early; it waits on the device
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const PrefillItem it = pf.items[blockIdx.x];
  const int G = a.group;
  const int Hkv = a.num_kv_heads;
  const int span0 = it.block_begin * BS;                          // first token of the partition
  const int span_end = min(it.block_end * BS, it.kv_end);         // one past its last used token
  const int nunits = span_end > span0 ? (span_end - span0 + UR - 1) / UR : 0;

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
    const uint64_t policy = l2_policy(2);  // every tile of a sequence re-reads its blocks
    const int32_t* bt = a.block_tables + static_cast<int64_t>(it.seq) * a.max_blocks_per_seq +
                        it.block_begin;
    const int nblk = it.block_end - it.block_begin;
    int ids = (lane < nblk) ? bt[lane] : -1;
    int chunk = 0;
    for (int u = 0; u < nunits; ++u) {
      const int b = u / UPB;
      const int half = u - b * UPB;
      if ((b >> 5) != chunk) {
        chunk = b >> 5;
        ids = (chunk * 32 + lane < nblk) ? bt[chunk * 32 + lane] : -1;
      }
      const int phys = __shfl_sync(0xffffffffu, ids, b & 31);
      const int stage = u % NS;
      const int use = u / NS;
      bool ok = true;
      if (use > 0) ok = mbar_wait_bounded(&empty[stage], (use - 1) & 1, a.dev_err);
      if (!__all_sync(0xffffffffu, ok)) break;
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
          mbar_arrive(&full[stage]);
        }
      }
    }
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
  const bool v0 = r0 < it.q_count * G;
  const bool v1 = r1 < it.q_count * G;
  const int j0 = r0 / G, j1 = r1 / G;                     // query token within the tile
  const int64_t t0 = it.q_begin + (v0 ? j0 : 0);          // global query token
  const int64_t t1 = it.q_begin + (v1 ? j1 : 0);
  const int64_t h0 = static_cast<int64_t>(it.kvh) * G + (r0 % G);
  const int64_t h1 = static_cast<int64_t>(it.kvh) * G + (r1 % G);
  const int pos0 = v0 ? it.p0 + j0 : -1;                  // causal limit (inclusive)
  const int pos1 = v1 ? it.p0 + j1 : -1;
  const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(a.q);
  MmaWarp<typename Cfg::Mma> st;
  st.begin_rows(q + (t0 * a.num_q_heads + h0) * D, q + (t1 * a.num_q_heads + h1) * D, v0, v1,
                a.scale_log2, lane);
  bool timed_out = false;
  int u = 0;
  for (; u + 1 < nunits && !timed_out; u += 2) {
    const int st0 = u % NS, st1 = (u + 1) % NS;
    bool ok = mbar_wait_bounded(&full[st0], (u / NS) & 1, a.dev_err);
    ok = ok && mbar_wait_bounded(&full[st1], ((u + 1) / NS) & 1, a.dev_err);
    if (!__all_sync(0xffffffffu, ok)) {
      timed_out = true;
      break;
    }
    const int sp = span0 + u * UR;
    const int lim0 = pos0 - sp, lim1 = pos1 - sp;
    if (__any_sync(0xffffffffu, lim0 >= 0 || lim1 >= 0)) {  // some row of the warp sees the span
      uint8_t* k0 = ring + st0 * Cfg::kStageBytes;
      uint8_t* k1 = ring + st1 * Cfg::kStageBytes;
      const uint8_t* kts[2] = {k0, k1};
      uint8_t* vts[2] = {k0 + Geo::kTileBytes, k1 + Geo::kTileBytes};
      st.template block_units<2, true>(kts, vts, 0, min(2 * UR, span_end - sp), lane, lim0, lim1);
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
    const int sp = span0 + u * UR;
    const int lim0 = pos0 - sp, lim1 = pos1 - sp;
    if (__any_sync(0xffffffffu, lim0 >= 0 || lim1 >= 0)) {
      uint8_t* kt = ring + stage * Cfg::kStageBytes;
      const uint8_t* kts[1] = {kt};
      uint8_t* vts[1] = {kt + Geo::kTileBytes};
      st.template block_units<1, true>(kts, vts, 0, min(UR, span_end - sp), lane, lim0, lim1);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
  }
  if (timed_out) return;
  if (it.final_out) {
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
    st.store_final(out + (t0 * a.num_q_heads + h0) * D, out + (t1 * a.num_q_heads + h1) * D, v0, v1,
                   lane);
  } else {
    const int64_t pr0 = v0 ? (t0 * a.num_q_heads + h0) * a.max_partitions + it.part : -1;
    const int64_t pr1 = v1 ? (t1 * a.num_q_heads + h1) * a.max_partitions + it.part : -1;
    st.store_partials(a, pr0, pr1, lane);
  }
}

}  // namespace pagedkv
