// Balanced split decode for sm_100a: every warp of the grid streams an equal
// share of the batch's K/V units (templates; instantiated in decode_inst_*.cu).
//
// What is computed is the same as paged_decode_kernel: for each sequence s
// and query head h, softmax(scale * K_s q) V_s over the tokens of the KV head
// h reads, reached through the sequence's block table ("What is
// PagedAttention?", How It Works / Map Logical to Physical Blocks), combined
// blockwise with a running max/sum ("PagedAttention: Optimizing KV Cache in
// vLLM", section 3), so that any cut of the context into pieces merged by
// log-sum-exp gives the contiguous result.
//
// How (B200 design, ours):
// * Each KV head's work is one list of 16-token units, sequence after
//   sequence (a sequence's units start at its sliding-window or shared-prefix
//   start; an empty sequence has one unit with nothing to read, so that its
//   zero output is still written). A (sequence, KV head) is a segment. Every
//   CTA builds the per-sequence prefix sum of units in shared memory.
// * The grid is persistent (SMs x occupancy) and static. Global warp w works
//   for KV head h = w % Hkv, in group g = w / Hkv, on units [g*C, (g+1)*C)
//   of h's list, with C = max(ceil(U_h / groups), ceil(U_max / (P - 1))):
//   every warp streams the same bytes (no tickets, no tail of uneven
//   items), and no segment (at most U_max units) is cut into more than P
//   pieces, the partial slots the workspace holds. The Hkv warps of a group
//   read the same blocks' tiles for different KV heads at the same time, so
//   the DRAM pages of a block ([Hkv][block_size][head_dim] contiguous) are
//   read together.
// * Each warp owns an NS-stage ring fed by its lane 0 with 2-D TMA loads of a
//   unit's K and V tiles (128-byte swizzle), completing on mbarriers. The
//   ring runs on across segment boundaries, so the next segment's loads are
//   in flight while the current one is finished, and the next segment's
//   query rows are prefetched into L2 when a segment begins. The lanes hold
//   the TMA row coordinates of the next 32 units (a block-table read each,
//   one window ahead).
// * The math is the per-warp state of the other decode kernel (mma.sync for
//   bf16, any group 1..16; CUDA cores for fp32). When a segment ends inside
//   the warp's range the warp writes it out from registers: as the final
//   output if the warp covered the whole segment, else as a partial
//   (m, l, acc) in slot `base + piece`, piece = g - floor(P_seg / C), where
//   P_seg is the segment's first unit in h's list. The warp that covers a
//   segment's first unit records the number of pieces for the merge kernel,
//   which runs as a programmatic dependent.
#pragma once

#include "decode_kernel.cuh"

namespace pagedkv {

template <class Cfg>
struct StreamCfg {
  static constexpr int kMiscInts = 8;
  // ring + barriers + misc, 1024-byte aligned ring; the two per-sequence
  // arrays (prefix [B + 1], first unit [B]) follow.
  static constexpr int kFixedSmem = 1024 + Cfg::kRingBytes + Cfg::kBarBytes + kMiscInts * 4;
  static_assert(kFixedSmem + (2 * 4096 + 1) * 4 <= 227 * 1024, "shared memory budget exceeded");
};

// First 16-token unit of sequence s the split kernel reads (sliding window
// start, blocks a shared-prefix pass covered), or -1 when there is nothing
// to read.
__device__ __forceinline__ int stream_first_unit(const DecodeArgs& a, int s, int ctx, int bs) {
  const int upb = bs / 16;
  int ub = first_token(a, ctx) / 16;
  if (a.seq_skip_blocks != nullptr) {
    const int full = ctx / bs;
    const int g = a.seq_skip_blocks[s];
    ub = max(ub, (g < 0 ? 0 : (g > full ? full : g)) * upb);
  }
  const int ue = (ctx + 15) / 16;
  return ub < ue ? ub : -1;
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::kThreads)
    paged_decode_stream_kernel(const __grid_constant__ CUtensorMap tm_k,
                               const __grid_constant__ CUtensorMap tm_v, const DecodeArgs a) {
  using T = typename Cfg::Elt;
  using Geo = typename Cfg::Geo;
  constexpr int W = Cfg::W;
  constexpr int NS = Cfg::NS;
  constexpr int BS = Cfg::BS;
  constexpr int UR = Cfg::UR;
  constexpr int UPB = Cfg::UPB;
  constexpr int D = Cfg::D;
  constexpr int NT = Cfg::kThreads;
  using WarpT = typename std::conditional<Cfg::kMma, MmaWarp<Cfg>, SimtWarp<Cfg>>::type;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kRingBytes);
  int* misc = reinterpret_cast<int*>(smem + Cfg::kRingBytes + Cfg::kBarBytes);
  int* prefix = misc + StreamCfg<Cfg>::kMiscInts;  // [B + 1] units (per KV head) before sequence s
  int* first_unit = prefix + a.num_seqs + 1;      // [B] first unit read, -1: nothing to read

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int B = a.num_seqs;
  const int Hkv = a.num_kv_heads;
  const int G = a.group;
  const int max_tokens = a.max_blocks_per_seq * BS;

  // The merge grid (a programmatic dependent) may be scheduled now; it waits
  // on the device for this grid's completion before it reads anything.
  grid_dependents_launch();

  if (tid == 0) {
    for (int i = 0; i < W * NS; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
    tma_prefetch_descriptor(&tm_k);
    tma_prefetch_descriptor(&tm_v);
  }

  // ---- per-sequence units (per KV head), their exclusive prefix sum, the max ---------
  __shared__ int warp_tot[W];
  __shared__ int warp_max_units[W];
  {
    const int chunk = (B + NT - 1) / NT;
    const int lo = min(B, tid * chunk);
    const int hi = min(B, lo + chunk);
    int mine = 0, biggest = 0;
    for (int i = lo; i < hi; ++i) {
      const int raw = a.context_lens[i];
      const int ctx = clamp_ctx(raw, max_tokens);
      if (ctx != raw && blockIdx.x == 0) report(a.dev_err, PA_DEVERR_CONTEXT_LEN);
      const int ub = stream_first_unit(a, i, ctx, BS);
      first_unit[i] = ub;
      const int u = ub < 0 ? 1 : (ctx + 15) / 16 - ub;
      mine += u;
      biggest = max(biggest, u);
    }
    int incl = mine;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) biggest = max(biggest, __shfl_xor_sync(0xffffffffu, biggest, off));
    if (lane == 31) warp_tot[warp] = incl;
    if (lane == 0) warp_max_units[warp] = biggest;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += warp_tot[w];
    int run = base + incl - mine;
    for (int i = lo; i < hi; ++i) {
      prefix[i] = run;
      const int ub = first_unit[i];
      run += ub < 0 ? 1 : (clamp_ctx(a.context_lens[i], max_tokens) + 15) / 16 - ub;
    }
    if (tid == NT - 1) prefix[B] = base + incl;
    __syncthreads();
  }

  const int U = prefix[B];  // units of each KV head's list
  int umax = 0;
#pragma unroll
  for (int w = 0; w < W; ++w) umax = max(umax, warp_max_units[w]);
  const int wg = static_cast<int>(blockIdx.x) * W + warp;
  const int groups = static_cast<int>(gridDim.x) * W / Hkv;
  const int h = wg % Hkv;   // this warp's KV head
  const int gi = wg / Hkv;  // its group
  const int C = max((U + groups - 1) / groups, (umax + a.max_pieces - 2) / (a.max_pieces - 1));
  const int64_t g_begin = static_cast<int64_t>(gi) * C;
  const int g0 = static_cast<int>(g_begin < U ? g_begin : U);
  const int g1 = static_cast<int>(g_begin + C < U ? g_begin + C : U);
  const int nj = gi < groups ? g1 - g0 : 0;
  if (nj <= 0) {
    if (a.wait_prior_at_exit) grid_dependency_wait();
    return;
  }

  // Sequence of unit g of a KV head's list (last s with prefix[s] <= g) and
  // the unit's index within the sequence's units.
  auto locate = [&](int g, int& s, int& un) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= g) lo = mid; else hi = mid - 1;
    }
    s = lo;
    un = g - prefix[s];
  };

  // TMA row of unit g of head h's list (>= 0), -1 for a unit with nothing to
  // read, -2 for a block id outside the pool.
  auto unit_row = [&](int g) -> int {
    if (g >= g1) return -1;
    int s, un;
    locate(g, s, un);
    const int ub = first_unit[s];
    if (ub < 0) return -1;
    const int u = ub + un;
    const int phys = a.block_tables[static_cast<int64_t>(s) * a.max_blocks_per_seq + u / UPB];
    if (phys < 0 || phys >= a.num_blocks) return -2;
    return (phys * Hkv + h) * BS + (u % UPB) * UR;
  };

  const uint64_t policy = l2_policy(a.l2_hint);
  uint8_t* my_ring = ring + warp * NS * Cfg::kStageBytes;
  uint64_t* my_bars = bars + warp * NS;
  int y_cur = unit_row(g0 + lane);
  int y_nxt = unit_row(g0 + 32 + lane);
  int win = 0;
  uint32_t bad = 0;  // bit per stage: nothing to compute (no data or a bad block id)

  auto issue = [&](int j) {
    const int c = j >> 5;
    if (c != win) {  // advance the window of unit rows by 32 units
      y_cur = y_nxt;
      y_nxt = unit_row(g0 + (c + 1) * 32 + lane);
      win = c;
    }
    const int y = __shfl_sync(0xffffffffu, y_cur, j & 31);
    const uint32_t stage = static_cast<uint32_t>(j) % NS;
    bad = (y >= 0) ? (bad & ~(1u << stage)) : (bad | (1u << stage));
    if (lane == 0) {
      uint64_t* bar = &my_bars[stage];
      fence_proxy_async_smem();
      if (y >= 0) {
        uint8_t* kdst = my_ring + stage * Cfg::kStageBytes;
        uint8_t* vdst = kdst + Geo::kTileBytes;
        mbar_arrive_expect_tx(bar, 2 * Geo::kTileBytes);
#pragma unroll
        for (int c2 = 0; c2 < Geo::kChunks; ++c2) {
          tma_load_2d(kdst + c2 * Geo::kChunkBytes, &tm_k, bar, c2 * Geo::kBoxCols, y, policy);
          tma_load_2d(vdst + c2 * Geo::kChunkBytes, &tm_v, bar, c2 * Geo::kBoxCols, y, policy);
        }
      } else {
        if (y == -2) report(a.dev_err, PA_DEVERR_BLOCK_ID);
        mbar_arrive(bar);  // completes the phase with no data
      }
    }
  };

  const int npre = min(NS, nj);
  for (int j = 0; j < npre; ++j) issue(j);

  // ---- consume the warp's units, segment by segment ---------------------------------
  WarpT st;
  int s = 0, un = 0;
  locate(g0, s, un);
  int us = prefix[s + 1] - prefix[s];
  int seg_start = g0 - un;  // index of the segment's first unit in h's list
  int ctx = 0, ftok = 0, ub = 0;
  const int64_t q_seq_stride = static_cast<int64_t>(a.num_q_heads) * D;
  auto begin_segment = [&]() {
    ctx = clamp_ctx(a.context_lens[s], max_tokens);
    ftok = first_token(a, ctx);
    ub = first_unit[s];
    const T* q_group = reinterpret_cast<const T*>(a.q) + static_cast<int64_t>(s) * q_seq_stride +
                       static_cast<int64_t>(h) * G * D;
    if (s + 1 < B && seg_start + us < g1) {
      // the next segment's query rows (G x D contiguous): into L2 now
      const char* nq = reinterpret_cast<const char*>(q_group + q_seq_stride);
      const int lines = (G * D * static_cast<int>(sizeof(T)) + 127) / 128;
      for (int i = lane; i < lines; i += 32) prefetch_l2(nq + i * 128);
    }
    if constexpr (Cfg::kMma) {
      st.begin(q_group, G, a.scale_log2, lane);
    } else {
      st.begin(q_group, a.scale_log2, lane);
    }
    if (un == 0) {  // this warp holds the segment's first piece: record the count
      const int pieces = (seg_start + us - 1) / C - seg_start / C + 1;
      if (lane == 0) a.seg_pieces[static_cast<int64_t>(s) * Hkv + h] = pieces;
    }
  };
  // Writes the segment out: final rows when this warp covered all of it and
  // no prefix pass contributed, else the partial slot of this warp's piece.
  auto end_segment = [&](bool reached_end) {
    const int base = a.seq_part_base ? a.seq_part_base[s] : 0;
    const int piece = gi - seg_start / C;
    const bool whole = reached_end && seg_start >= g0 && base == 0;
    const int64_t row0 = static_cast<int64_t>(s) * a.num_q_heads + static_cast<int64_t>(h) * G;
    if constexpr (Cfg::kMma) {
      const int g = lane >> 2;
      if (whole) {
        T* o = reinterpret_cast<T*>(a.out) + row0 * D;
        st.store_final(o + g * D, o + (g + 8) * D, g < G, g + 8 < G, lane);
      } else {
        const int64_t pr0 = g < G ? (row0 + g) * a.max_partitions + base + piece : -1;
        const int64_t pr1 = g + 8 < G ? (row0 + g + 8) * a.max_partitions + base + piece : -1;
        st.store_partials(a, pr0, pr1, lane);
      }
    } else {
      if (whole) {
        st.store_final(reinterpret_cast<T*>(a.out) + row0 * D, lane);
      } else {
        st.store_partials(a, row0 * a.max_partitions + base + piece, a.max_partitions, lane);
      }
    }
  };

  begin_segment();
  bool timed_out = false;
  int j = 0;
  for (; j < nj; ++j) {
    if (un == us) {  // the previous unit ended its segment: move to the next one
      end_segment(true);
      seg_start += us;
      ++s;
      us = prefix[s + 1] - prefix[s];
      un = 0;
      begin_segment();
    }
    const uint32_t stage = static_cast<uint32_t>(j) % NS;
    const uint32_t parity = (static_cast<uint32_t>(j) / NS) & 1u;
    const bool okw = mbar_wait_bounded(&my_bars[stage], parity, a.dev_err);
    if (!__all_sync(0xffffffffu, okw)) {
      timed_out = true;
      break;
    }
    if (!(bad & (1u << stage))) {
      const int u0 = (ub + un) * UR;     // first token of the unit
      const int nvalid = min(UR, ctx - u0);
      const int nfirst = ftok - u0;      // > 0 only inside a window's first unit
      if (nfirst < nvalid) {
        uint8_t* kt = my_ring + stage * Cfg::kStageBytes;
        st.block(kt, kt + Geo::kTileBytes, nfirst, nvalid, lane);
      }
    }
    __syncwarp();
    ++un;
    if (j + NS < nj) issue(j + NS);
  }
  if (timed_out) {
    // Give copies still in flight a bounded chance to land before leaving.
    for (int jj = j; jj < min(nj, j + NS); ++jj)
      mbar_wait_bounded(&my_bars[jj % NS], (jj / NS) & 1u, a.dev_err);
  } else {
    end_segment(un == us);
  }
  if (a.wait_prior_at_exit) grid_dependency_wait();
}

}  // namespace pagedkv
