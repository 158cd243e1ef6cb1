// Paged prefill attention on 5th-generation tensor cores (tcgen05 + TMEM).
//
// What is computed is the causal prefill of prefill_kernel.cuh: new token i
// of a sequence at position p attends to tokens 0..p, read through the block
// table ("What is PagedAttention?", How It Works). Many queries share every
// KV tile, so the products are a dense contraction; here they run as
// 128-row tcgen05 MMAs with fp32 accumulators in tensor memory.
//
// An item = two tiles of 128 query rows (query tokens x the KV head's group
// heads) of one sequence, one KV head, one KV partition. Both tiles share
// every K/V chunk, so the tensor core has one tile's work while the other
// tile's softmax runs. A CTA runs one item, or (persistent launch) a list of
// items back to back: the ring, the S buffers and every barrier carry on
// across items, so the next item's loads and first S overlap the end of the
// current one and its epilogue.
//   warp 8 (producer): streams K_j then V_j of each 64-token chunk (four
//     16-token TMA units, 128-byte swizzle: a chunk is one K-major operand
//     for S and one MN-major operand for P V) into a ring of slots, and
//     clears the V rows past the span in the last chunk.
//   warps 9 / 10 (MMA issuers of tile 0 / 1) load the tile's Q (one 3-D TMA
//     box per 64 columns: tokens x group heads x 64, landing as 128-byte
//     swizzled rows in token-major, head-minor order; the next item's as
//     soon as the current item's last S is done), and per chunk j issue:
//       S_t(j+1) = Q_t K_{j+1}^T     (M=128, N=64, K=head_dim)
//       O_t += P_t(j) V_j            (M=128, N=head_dim, K=64, P read from TMEM)
//     The MMA completions an issuer waits for: the P V of two chunks back,
//     before S overwrites the buffer holding that P; the item's last S,
//     before the next Q overwrites this one.
//   warps 0-3 / 4-7 (softmax of tile 0 / 1): thread r owns row r (TMEM lane
//     r). It reads its 64 logits, masks causally where the chunk reaches
//     past the row's position, and keeps a reference max m: P = 2^(x - m)
//     is written back as packed bf16 over the logits it came from (the A
//     operand of P V); m moves only when the chunk's max exceeds it by more
//     than 8 (log2 units, so P <= 2^8), and then O (in TMEM) and l are scaled
//     by 2^(m_old - m_new). The unmasked path runs on packed fp32 pairs
//     (f32x2 FMA/add) and a three-input max. The softmax is bound by each
//     warp's own instruction latency (two softmax warps per SM
//     sub-partition), not by MUFU: moving a share of the exponentials to an
//     FMA-pipe polynomial measured slower at every share tried (1/4, 3/8,
//     1/2). After an item's last chunk the same warps write its output: a
//     full tile of final rows through a 128-byte-swizzled staging buffer and
//     one TMA store per 64 columns, other rows with plain stores.
// TMEM per tile: two 64-column S / P buffers (chunk parity) and head_dim O
// columns; 512 columns for the CTA. The tensor core reads its shared-memory
// operands at about 128 bytes per clock per SM, so P stays out of shared
// memory: per chunk the MMAs read Q and K (S) and V (P V) only. Every
// hand-over is an mbarrier (TMA byte counts, tcgen05.commit, warp arrivals)
// with one barrier per buffer, so no waiter can be lapped by two phases (the
// producer clears a partial chunk's V only after both issuers are past the
// previous clear); every wait is bounded.
#pragma once

#include "prefill_kernel.cuh"

namespace pagedkv {

// ---- packed fp32 pairs (Blackwell f32x2 arithmetic) --------------------------------
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

template <int BS_, int D_, int TILES_, int HALVES_ = 1>
struct TcCfg {
  static constexpr int BS = BS_;
  static constexpr int D = D_;
  static constexpr int ROWS = 128;                      // MMA M: query rows per tile
  static constexpr int TILES = TILES_;                  // tiles per CTA (1 or 2)
  static constexpr int CHUNK = 64;                      // KV tokens per step (N of S, K of P V)
  static constexpr int UR = 16;                         // TMA unit rows
  static constexpr int UPC = CHUNK / UR;                // units per chunk
  static constexpr int KCH = D * 2 / 128;               // 128-byte column chunks of a row
  static constexpr int kQBytes = ROWS * D * 2;          // one tile's Q
  static constexpr int kSlotBytes = CHUNK * D * 2;      // K or V of one chunk
  // Threads per query row in the softmax (1 or 2): with two, each takes half
  // of a chunk's 64 logits and half of O's columns.
  static constexpr int HALVES = HALVES_;
  // ring: K_0 V_0 K_1 V_1 ...; one-tile CTAs run two per SM (TMEM and
  // shared memory for two), so one CTA's prologue and epilogue overlap the
  // other's main loop. Two-tile CTAs with two threads per row keep 7 slots:
  // the eighth's 16 KB went to the halves' exchange buffers.
  static constexpr int NSLOT = TILES == 2 ? (HALVES == 2 ? 7 : 8) : 4;
  static constexpr int kMinBlocks = TILES == 2 ? 1 : 2;
  static constexpr int kBarBytes = 512;
  // Two-tile CTAs stage each tile's normalised output, 64 columns at a time,
  // for one TMA store (one-tile CTAs serve scattered output rows).
  static constexpr bool kTmaOut = TILES == 2;
  static constexpr int kStageBytes = kTmaOut ? TILES * ROWS * 128 : 0;
  // The halves of a row swap row maxima (each chunk) and row sums (each item)
  // through [tile][buffer][half][row] floats, double-buffered.
  static constexpr int kXchgBytes = HALVES == 2 ? TILES * 2 * HALVES * ROWS * 4 : 0;
  static constexpr int kSmem =
      1024 + TILES * kQBytes + NSLOT * kSlotBytes + kStageBytes + kXchgBytes + kBarBytes;
  static constexpr int kTileWarps = 4 * HALVES;         // softmax warps per tile
  static constexpr int kSoftmaxWarps = kTileWarps * TILES;
  static constexpr int kThreads = (kSoftmaxWarps + 1 + TILES) * 32;
  static constexpr uint32_t kTileCols = 256;            // S buffers [0,128), O [128, 128 + D)
  static constexpr uint32_t kTmemCols = TILES * kTileCols;
  static constexpr uint32_t kOCol = 128;
  static constexpr float kRescaleThreshold = 8.f;       // log2 units
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(BS % UR == 0, "block size");
  static_assert(32 % UPC == 0, "a chunk's units lie in one 32-unit id batch");
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static_assert(kTmemCols * kMinBlocks <= 512, "tensor memory");
  static_assert(kSmem * kMinBlocks <= 228 * 1024, "shared memory per SM");
  static_assert(TILES == 1 || TILES == 2, "tiles");
  static_assert(HALVES == 1 || HALVES == 2, "threads per row");
};

// One work item as every role of the CTA sees it.
struct TcItem {
  PrefillItem it;
  int ntiles;    // tiles holding query rows (1 or 2)
  int span0;     // first KV token of the partition
  int span_end;  // KV tokens [span0, span_end) are streamed
  int nchunks;   // CHUNK-token steps over the span
  int vt_last;   // valid rows of the last chunk
};

template <class Cfg>
__device__ __forceinline__ TcItem tc_item(const PrefillArgs& pf, int idx, int tq) {
  TcItem x;
  x.it = pf.items[idx];
  x.ntiles = (Cfg::TILES == 2 && x.it.q_count > tq) ? 2 : 1;
  x.span0 = x.it.block_begin * Cfg::BS;
  x.span_end = min(x.it.block_end * Cfg::BS, x.it.kv_end);
  x.nchunks = x.span_end > x.span0 ? (x.span_end - x.span0 + Cfg::CHUNK - 1) / Cfg::CHUNK : 0;
  x.vt_last = x.nchunks > 0 ? x.span_end - (x.span0 + (x.nchunks - 1) * Cfg::CHUNK) : Cfg::CHUNK;
  return x;
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::kThreads, Cfg::kMinBlocks)
    tc_prefill_kernel(const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_o, const PrefillArgs pf) {
  constexpr int NSLOT = Cfg::NSLOT;
  constexpr int BS = Cfg::BS;
  constexpr int D = Cfg::D;
  constexpr int UR = Cfg::UR;
  constexpr int CHUNK = Cfg::CHUNK;
  constexpr int KCH = Cfg::KCH;
  constexpr int ROWS = Cfg::ROWS;
  constexpr int SMW = Cfg::kSoftmaxWarps;
  const DecodeArgs& a = pf.d;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* qs = smem;                                    // [TILES][KCH][ROWS][128 B]
  uint8_t* slots = qs + Cfg::TILES * Cfg::kQBytes;       // [NSLOT][KCH][CHUNK][128 B]
  uint8_t* stage = slots + NSLOT * Cfg::kSlotBytes;      // [TILES][ROWS][128 B] output staging
  float* xval = reinterpret_cast<float*>(stage + Cfg::kStageBytes);  // [TILES][2][HALVES][ROWS]
  uint64_t* bars = reinterpret_cast<uint64_t*>(stage + Cfg::kStageBytes + Cfg::kXchgBytes);
  uint64_t* kv_full = bars;               // [NSLOT] TMA bytes landed
  uint64_t* kv_empty = bars + NSLOT;      // [NSLOT] both tiles done with the slot
  uint64_t* s_full = bars + 2 * NSLOT;    // [tile][buffer] S MMA done (commit)
  uint64_t* p_full = s_full + 4;          // [tile][buffer] P written (a tile's softmax warps)
  uint64_t* p_free = p_full + 4;          // [tile][buffer] P V MMA done (commit)
  uint64_t* q_full = p_free + 4;          // [tile] Q in shared memory (TMA bytes)
  uint64_t* q_free = q_full + 2;          // [tile] the item's last S MMA done (commit)
  uint64_t* o_last = q_free + 2;          // [tile] every MMA of the item done (commit)
  uint64_t* o_empty = o_last + 2;         // [tile] O read out of TMEM (a tile's softmax warps)
  uint64_t* mma_done = o_empty + 2;       // [tile] every MMA of the CTA done (commit), once
  uint64_t* v_tail = mma_done + 2;        // a last chunk's V tail rows cleared (producer)
  uint64_t* xchg = v_tail + 1;            // [tile][buffer] both halves' values written (threads)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xchg + 4);

  grid_dependents_launch();
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int G = a.group;
  const int Hkv = a.num_kv_heads;
  const int TQ = ROWS / G;  // query tokens per tile
  // This CTA's items, in order.
  const int k_begin = pf.sched_off ? pf.sched_off[blockIdx.x] : static_cast<int>(blockIdx.x);
  const int k_end = pf.sched_off ? pf.sched_off[blockIdx.x + 1] : k_begin + 1;

  if (tid == 0) {
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], Cfg::TILES);  // one arrival per tile's issuer, idle or not
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], Cfg::kTileWarps);
      mbar_init(&p_free[i], 1);
      mbar_init(&xchg[i], Cfg::kTileWarps * 32);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&q_full[t], 1);
      mbar_init(&q_free[t], 1);
      mbar_init(&o_last[t], 1);
      mbar_init(&o_empty[t], Cfg::kTileWarps);
      mbar_init(&mma_done[t], 1);
    }
    mbar_init(v_tail, 1);
    fence_barrier_init();
    tma_prefetch_descriptor(&tm_k);
    tma_prefetch_descriptor(&tm_v);
    tma_prefetch_descriptor(&tm_q);
  }
  if (warp == 0) tmem_alloc(tmem_slot, Cfg::kTmemCols);
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // Every role walks the same items and keeps its own running counts; a
  // barrier's phase parity follows from them:
  //   g  - K/V loads before the item (ring slot g % NSLOT, use g / NSLOT);
  //   cb - chunks of tile t before the item (S / P buffer cb & 1);
  //   nt - items tile t took part in (q_full, q_free, o_last, o_empty);
  //   tails - items with a partial last chunk (v_tail).
  if (warp == SMW) {
    // ---- producer: K_0, V_0, K_1, V_1, ... of every item into the slot ring ----------
    const uint64_t policy = l2_policy(2);  // every query tile of a sequence re-reads its blocks
    int g = 0;
    int prev_tail = -1;  // ring index of the previous partial chunk's V
    bool ok = true;
    for (int idx = k_begin; idx < k_end && ok; ++idx) {
      const TcItem x = tc_item<Cfg>(pf, idx, TQ);
      if (x.nchunks == 0) continue;
      const int32_t* bt = a.block_tables + static_cast<int64_t>(x.it.seq) * a.max_blocks_per_seq;
      // Block ids of the span's 16-token units, 32 units per batch held one per
      // lane, the next batch loaded a batch ahead (a chunk's units never
      // straddle two batches).
      const int nunits = (x.span_end - x.span0 + UR - 1) / UR;
      auto unit_ids = [&](int batch) -> int {
        const int u = batch * 32 + lane;
        return u < nunits ? bt[(x.span0 + u * UR) / BS] : -1;
      };
      int ids = unit_ids(0);
      int ids_next = unit_ids(1);
      int batch = 0;
      for (int i = 0; i < 2 * x.nchunks; ++i) {
        const int j = i >> 1;
        const int gi = g + i;
        const int slot = gi % NSLOT;
        const int use = gi / NSLOT;
        if (use > 0) ok = mbar_wait_bounded(&kv_empty[slot], (use - 1) & 1, a.dev_err);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          g = gi;  // loads issued so far
          break;
        }
        const int c0 = x.span0 + j * CHUNK;
        const int nu = min(Cfg::UPC, (x.span_end - c0 + UR - 1) / UR);  // units holding used tokens
        const int u0 = j * Cfg::UPC;
        if ((u0 >> 5) != batch) {
          batch = u0 >> 5;
          ids = ids_next;
          ids_next = unit_ids(batch + 1);
        }
        int phys_u[Cfg::UPC];
#pragma unroll
        for (int u = 0; u < Cfg::UPC; ++u) phys_u[u] = __shfl_sync(0xffffffffu, ids, (u0 + u) & 31);
        // Every value above is warp-uniform; one elected lane of the converged
        // warp issues the copies.
        if (elect_one()) {
          const CUtensorMap* map = (i & 1) ? &tm_v : &tm_k;
          uint8_t* dst = slots + slot * Cfg::kSlotBytes;
          uint32_t bytes = 0;
#pragma unroll
          for (int u = 0; u < Cfg::UPC; ++u)
            if (u < nu && phys_u[u] >= 0 && phys_u[u] < a.num_blocks) bytes += KCH * UR * 128;
          mbar_arrive_expect_tx(&kv_full[slot], bytes);
#pragma unroll
          for (int u = 0; u < Cfg::UPC; ++u) {
            if (u >= nu) continue;
            const int ph = phys_u[u];
            if (ph < 0 || ph >= a.num_blocks) {
              if (i & 1) report(a.dev_err, PA_DEVERR_BLOCK_ID);  // the unit keeps stale rows
              continue;
            }
            const int32_t y = (ph * Hkv + x.it.kvh) * BS + ((c0 + u * UR) % BS);
#pragma unroll
            for (int c = 0; c < KCH; ++c)
              tma_load_2d(dst + c * (CHUNK * 128) + u * (UR * 128), map, &kv_full[slot], c * 64, y, policy);
          }
        }
        __syncwarp();
      }
      if (!ok) break;
      // Clear V rows [vt_last, CHUNK) of a partial last chunk once its copy
      // landed (stale or unloaded rows; 0 * NaN is NaN), then release its P V.
      // The previous clear must have been waited for by both issuers first
      // (its slot released), so v_tail never runs two phases ahead of a waiter.
      if (x.vt_last < CHUNK) {
        const int gi = g + 2 * x.nchunks - 1;
        bool ready = mbar_wait_bounded(&kv_full[gi % NSLOT], (gi / NSLOT) & 1, a.dev_err);
        if (ready && prev_tail >= 0 && gi - prev_tail < NSLOT)
          ready = mbar_wait_bounded(&kv_empty[prev_tail % NSLOT], (prev_tail / NSLOT) & 1, a.dev_err);
        if (!__all_sync(0xffffffffu, ready)) {
          ok = false;
          g += 2 * x.nchunks;
          break;
        }
        uint8_t* vst = slots + (gi % NSLOT) * Cfg::kSlotBytes;
        const int n16 = (CHUNK - x.vt_last) * KCH * 8;
        for (int e = lane; e < n16; e += 32) {
          const int row = x.vt_last + e / (KCH * 8);
          const int rem = e % (KCH * 8);
          *reinterpret_cast<uint4*>(vst + (rem >> 3) * (CHUNK * 128) + row * 128 + ((rem & 7) << 4)) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(v_tail);
        prev_tail = gi;
      }
      g += 2 * x.nchunks;
    }
    // Every copy issued has landed before the CTA's shared memory is released.
    for (int gi = max(0, g - NSLOT); gi < g; ++gi)
      mbar_wait_bounded(&kv_full[gi % NSLOT], (gi / NSLOT) & 1, a.dev_err);
    __syncwarp();
  } else if (warp > SMW) {
    // ---- MMA issuer of tile t: the whole warp runs the loop (waits are warp-wide,
    // values warp-uniform); one elected lane issues each group of MMAs and commits,
    // and loads the tile's Q (the next item's as soon as this item's last S is done).
    const int t = warp - SMW - 1;
    constexpr uint32_t kIdS = umma_idesc_bf16(ROWS, CHUNK, 0, 0);
    constexpr uint32_t kIdO = umma_idesc_bf16(ROWS, D, 0, 1);
    // Descriptors are built once; a start address moves by adding its
    // offset in 16-byte units (the 14-bit field cannot overflow below 256 KB).
    const uint64_t q_desc = umma_desc_sw128(smem_addr(qs + t * Cfg::kQBytes), 16, 1024);
    const uint64_t k_desc = umma_desc_sw128(smem_addr(slots), 16, 1024);
    const uint64_t v_desc = umma_desc_sw128(smem_addr(slots), CHUNK * 128, 1024);
    const uint32_t s_tmem = tmem + t * Cfg::kTileCols;
    const uint32_t o_tmem = tmem + t * Cfg::kTileCols + Cfg::kOCol;
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity, a.dev_err));
    };
    // Q of tile t of an item: rows past the query tokens of the array read as
    // 0 (the box's out-of-range fill), rows past the item's tokens are masked.
    int q_loads = 0, q_seen = 0;
    auto load_q = [&](const TcItem& y) {
      if (elect_one()) {
        mbar_arrive_expect_tx(&q_full[t], KCH * TQ * G * 128);
        for (int c = 0; c < KCH; ++c)
          tma_load_3d(qs + t * Cfg::kQBytes + c * (ROWS * 128), &tm_q, &q_full[t], c * 64,
                      y.it.q_head0, y.it.q_begin + t * TQ);
      }
      __syncwarp();
      ++q_loads;
    };
    // When Q was packed by a preceding kernel (launched as its programmatic
    // dependent), wait for that grid before the first Q copy.
    grid_dependency_wait();
    int g = 0, cb = 0, nt = 0, tails = 0;
    bool ok = true;
    for (int idx = k_begin; idx < k_end && ok; ++idx) {
      const TcItem x = tc_item<Cfg>(pf, idx, TQ);
      if (x.nchunks == 0) continue;
      const bool tail = x.vt_last < CHUNK;
      if (t >= x.ntiles) {
        // An idle tile still releases every slot of the item.
        for (int i = 0; i < 2 * x.nchunks && ok; ++i) {
          const int gi = g + i;
          ok = wait(&kv_full[gi % NSLOT], (gi / NSLOT) & 1);
          if (ok && elect_one()) mbar_arrive(&kv_empty[gi % NSLOT]);
          __syncwarp();
        }
        g += 2 * x.nchunks;
        tails += tail ? 1 : 0;
        continue;
      }
      if (q_loads == q_seen) load_q(x);
      ok = wait(&q_full[t], q_seen & 1);
      ++q_seen;
      // S_t(j) = Q_t K_j^T into buffer (cb + j) & 1, once the P V that last
      // read that buffer (two chunks back) is done.
      auto issue_s = [&](int j) -> bool {
        const int gi = g + 2 * j, slot = gi % NSLOT, c = cb + j, b = c & 1;
        if (!wait(&kv_full[slot], (gi / NSLOT) & 1)) return false;
        if (c >= 2 && !wait(&p_free[2 * t + b], ((c >> 1) - 1) & 1)) return false;
        tmem_fence_after_sync();
        const uint64_t kd = k_desc + static_cast<uint32_t>((slot * Cfg::kSlotBytes) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_bf16(s_tmem + b * CHUNK, q_desc + (((kk / 4) * (ROWS * 128) + (kk % 4) * 32) >> 4),
                      kd + (((kk / 4) * (CHUNK * 128) + (kk % 4) * 32) >> 4), kIdS, kk > 0);
          umma_commit(&s_full[2 * t + b]);
          umma_commit(&kv_empty[slot]);
        }
        __syncwarp();
        return true;
      };
      // After the item's last S: once it is done, Q's buffer is free and the
      // next item this tile takes part in gets its Q copy started.
      auto after_last_s = [&]() -> bool {
        if (elect_one()) umma_commit(&q_free[t]);
        __syncwarp();
        for (int n = idx + 1; n < k_end; ++n) {
          const TcItem y = tc_item<Cfg>(pf, n, TQ);
          if (y.nchunks == 0 || t >= y.ntiles) continue;
          if (!wait(&q_free[t], nt & 1)) return false;
          load_q(y);
          break;
        }
        return true;
      };
      ok = ok && issue_s(0);
      if (ok && x.nchunks == 1) ok = after_last_s();
      // Issuing whichever of S and P V became ready first measured the same
      // as this fixed order (S of the next chunk, then P V of this one).
      for (int j = 0; j < x.nchunks && ok; ++j) {
        if (j + 1 < x.nchunks) {
          ok = issue_s(j + 1);
          if (ok && j + 2 == x.nchunks) ok = after_last_s();
          if (!ok) break;
        }
        const int gi = g + 2 * j + 1, slot = gi % NSLOT, c = cb + j, b = c & 1;
        ok = wait(&kv_full[slot], (gi / NSLOT) & 1);
        if (ok && tail && j == x.nchunks - 1) ok = wait(v_tail, tails & 1);
        ok = ok && wait(&p_full[2 * t + b], (c >> 1) & 1);
        // The first P V of an item overwrites O: the previous item's O must be read out.
        if (ok && j == 0 && nt > 0) ok = wait(&o_empty[t], (nt - 1) & 1);
        if (!ok) break;
        tmem_fence_after_sync();
        const uint64_t vd = v_desc + static_cast<uint32_t>((slot * Cfg::kSlotBytes) >> 4);
        const uint32_t pa = s_tmem + b * CHUNK;  // P over S: 8 columns per K = 16 step
        if (elect_one()) {
#pragma unroll
          for (int k = 0; k < CHUNK / 16; ++k)
            umma_bf16_ts(o_tmem, pa + k * 8, vd + ((k * 16 * 128) >> 4), kIdO, j > 0 || k > 0);
          umma_commit(&p_free[2 * t + b]);
          umma_commit(&kv_empty[slot]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one()) umma_commit(&o_last[t]);
      __syncwarp();
      g += 2 * x.nchunks;
      cb += x.nchunks;
      tails += tail ? 1 : 0;
      ++nt;
    }
    // Before TMEM and shared memory are released: a Q copy still in flight
    // (after an error), then every MMA this thread issued. elect.sync picks
    // the same lane of the fully active warp every time, so the MMAs above
    // and this commit share one issuing thread.
    if (q_loads > q_seen) wait(&q_full[t], q_seen & 1);
    if (elect_one()) umma_commit(&mma_done[t]);
    __syncwarp();
    wait(&mma_done[t], 0);
  } else {
    // ---- softmax warps: tile t = warp / (4 HALVES). Warp w of the tile reads
    // TMEM lane quarter w % 4 (rows 32 (w % 4) ..); with two threads per row,
    // half hf = w / 4 of the columns: logits 32 hf .. 32 hf + 31 of each chunk,
    // O columns hf D/2 .. of the row. Thread (quarter, lane) owns row r = 32
    // quarter + lane, with its partner thread of the other half; the two swap
    // their row maximum every chunk (and their row sum at the item's end)
    // through xval, completed by xchg (every thread of the tile arrives, so
    // each thread's own store is released by its arrival).
    constexpr int HALF_CHUNK = CHUNK / Cfg::HALVES;
    constexpr int HALF_D = D / Cfg::HALVES;
    const int t = warp / Cfg::kTileWarps;
    const int wt = warp % Cfg::kTileWarps;
    const int hf = wt >> 2;
    const int r = (wt & 3) * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * (wt & 3)) << 16) + t * Cfg::kTileCols;
    float* xt = xval + t * (2 * Cfg::HALVES * ROWS);
    const float sl2 = a.scale_log2;
    int cb = 0, nt = 0, ex = 0;
    bool ok = true;  // warp-uniform
    // Publishes v, waits (bounded) until both halves of the tile published,
    // returns the partner's value. Buffers alternate, so a half can run at
    // most one exchange ahead of its partner's read.
    // The tcgen05 fences order this thread's TMEM loads before the partner's
    // later TMEM stores (P over the buffer's first columns).
    auto exchange = [&](float v, bool& good, float none) -> float {
      good = true;
      if constexpr (Cfg::HALVES == 1) return none;
      const int buf = ex & 1;
      xt[(buf * Cfg::HALVES + hf) * ROWS + r] = v;
      tmem_fence_before_sync();
      mbar_arrive(&xchg[2 * t + buf]);
      good = __all_sync(0xffffffffu, mbar_wait_bounded(&xchg[2 * t + buf], (ex >> 1) & 1, a.dev_err));
      tmem_fence_after_sync();
      const float other = xt[(buf * Cfg::HALVES + (1 - hf)) * ROWS + r];
      ++ex;
      return other;
    };
    for (int idx = k_begin; idx < k_end && ok; ++idx) {
      const TcItem x = tc_item<Cfg>(pf, idx, TQ);
      if (t >= x.ntiles) continue;                         // no row of this tile is a query row
      const PrefillItem& it = x.it;
      const int nchunks = x.nchunks;
      const int span_end = x.span_end;
      const int jq = t * TQ + r / G;                       // query token within the item
      const bool valid = (r / G) < TQ && jq < it.q_count;
      const int lim = valid ? it.p0 + jq : -1;             // last token this row attends to
      float m_used = -INFINITY, l = 0.f;                   // m_used: the same in both halves
      for (int j = 0; j < nchunks; ++j) {
        const int c = cb + j;
        const int b = c & 1;
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s_full[2 * t + b], (c >> 1) & 1, a.dev_err));
        if (!ok) break;
        tmem_fence_after_sync();
        float sv[HALF_CHUNK];
        if constexpr (Cfg::HALVES == 2) {
          tmem_ld32(trow + b * CHUNK + hf * HALF_CHUNK, sv);
        } else {
          tmem_ld64(trow + b * CHUNK, sv);
        }
        const int c0 = x.span0 + j * CHUNK + hf * HALF_CHUNK;  // this half's first token
        // Scaled logits: x = s * scale * log2(e). Only a chunk that reaches
        // past the row's position or the span's end needs the mask.
        const int chunk_last = x.span0 + j * CHUNK + CHUNK - 1;
        const bool whole = chunk_last < span_end && chunk_last <= lim && sl2 > 0.f;
        float mx;
        if (whole) {
          constexpr int NG = HALF_CHUNK / 8;
          float mg[NG];
#pragma unroll
          for (int k = 0; k < NG; ++k) {
            const float* v = sv + 8 * k;
            mg[k] = fmax3(fmax3(v[0], v[1], v[2]), fmax3(v[3], v[4], v[5]), fmaxf(v[6], v[7]));
          }
          mx = mg[0];
#pragma unroll
          for (int k = 1; k < NG; ++k) mx = fmaxf(mx, mg[k]);
          mx *= sl2;
        } else {
          mx = -INFINITY;
#pragma unroll
          for (int i = 0; i < HALF_CHUNK; ++i) {
            const int tk = c0 + i;
            const bool in = tk < span_end && tk <= lim;
            sv[i] = in ? sv[i] * sl2 : -INFINITY;
            mx = fmaxf(mx, sv[i]);
          }
        }
        // Both halves have read this chunk's logits once the exchange completes,
        // so P may then be written over the buffer's first 32 columns.
        bool good;
        mx = fmaxf(mx, exchange(mx, good, -INFINITY));
        ok = good;
        if (!ok) break;
        const bool raise = mx > m_used + Cfg::kRescaleThreshold;
        const bool rescale_o = raise && m_used != -INFINITY;  // only from the item's second chunk on
        if (__any_sync(0xffffffffu, rescale_o)) {
          // O must hold every earlier P V product of the item before it is scaled.
          const int pb = 2 * t + ((c - 1) & 1);
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(&p_free[pb], ((c - 1) >> 1) & 1, a.dev_err));
          if (!ok) break;
          tmem_fence_after_sync();
          const float alpha = rescale_o ? fast_exp2(m_used - mx) : 1.f;
#pragma unroll
          for (int q = 0; q < HALF_D / 16; ++q) {
            float o16[16];
            tmem_ld16(trow + Cfg::kOCol + hf * HALF_D + q * 16, o16);
#pragma unroll
            for (int i = 0; i < 16; ++i) o16[i] *= alpha;
            tmem_st16(trow + Cfg::kOCol + hf * HALF_D + q * 16, o16);
          }
          tmem_fence_before_sync();
          l *= alpha;
        }
        if (raise) m_used = mx;
        // P = 2^(x - m_used) <= 2^8, as packed bf16 pairs: this half's 32
        // tokens go to columns 16 hf .. 16 hf + 15 of the buffer.
        uint32_t pk[HALF_CHUNK / 2];
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
        if (whole) {
          const uint64_t sl2_2 = f2_pack(sl2, sl2);
          const uint64_t nm2 = f2_pack(-m_used, -m_used);
          uint64_t acc2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
          for (int i = 0; i < HALF_CHUNK; i += 2) {
            const uint64_t x2 = f2_fma(f2_pack(sv[i], sv[i + 1]), sl2_2, nm2);
            float x0, x1;
            f2_unpack(x2, x0, x1);
            const float p0 = fast_exp2(x0);
            const float p1 = fast_exp2(x1);
            acc2[(i >> 1) & 1] = f2_add(acc2[(i >> 1) & 1], f2_pack(p0, p1));
            pk[i >> 1] = pack_bf16x2(p0, p1);
          }
          float a0, a1, b0, b1;
          f2_unpack(acc2[0], a0, a1);
          f2_unpack(acc2[1], b0, b1);
          s4[0] = a0; s4[1] = a1; s4[2] = b0; s4[3] = b1;
        } else {
          const float mu = (m_used == -INFINITY) ? 0.f : m_used;  // a row with nothing yet: all p = 0
#pragma unroll
          for (int i = 0; i < HALF_CHUNK; i += 2) {
            const float p0 = fast_exp2(sv[i] - mu);
            const float p1 = fast_exp2(sv[i + 1] - mu);
            s4[(i >> 1) & 3] += p0 + p1;
            pk[i >> 1] = pack_bf16x2(p0, p1);
          }
        }
        l += (s4[0] + s4[1]) + (s4[2] + s4[3]);
        if constexpr (Cfg::HALVES == 2) {
          tmem_st16_bits(trow + b * CHUNK + hf * (HALF_CHUNK / 2), pk);
        } else {
          tmem_st32_bits(trow + b * CHUNK, pk);
        }
        tmem_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[2 * t + b]);
      }
      if (!ok) break;
      // ---- the item's epilogue: O from TMEM, normalised (single partition) or
      // as a partial; then O's columns are handed back for the next item.
      if (nchunks > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&o_last[t], nt & 1, a.dev_err));
        if (!ok) break;
        tmem_fence_after_sync();
      }
      {
        bool good;
        l += exchange(l, good, 0.f);                       // the row sum over both halves
        ok = good;
        if (!ok) break;
      }
      const int64_t tok = !valid ? it.q_begin
                          : it.out_begin >= 0 ? pf.out_tokens[it.out_begin + jq] : it.q_begin + jq;
      const int64_t h = static_cast<int64_t>(it.kvh) * G + (r % G);
      const int64_t row = tok * a.num_q_heads + h;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      // A full tile of final rows goes out by TMA: its rows (token-major,
      // head-minor, as Q came in) are staged 64 columns at a time in the
      // 128-byte swizzle and stored as one box; one thread per tile issues
      // the stores. Each half stages the 16-byte units of its own columns.
      // Partial tiles, scattered rows and partials use plain stores (each
      // thread its row's half).
      const bool tma_out = Cfg::kTmaOut && nchunks > 0 && it.final_out && it.out_begin < 0 &&
                           it.q_count >= (t + 1) * TQ;
      if (tma_out) {
        uint8_t* sbuf = stage + t * (ROWS * 128);
        const bool leader = wt == 0 && lane == 0;
#pragma unroll
        for (int cc = 0; cc < KCH; ++cc) {
          if (leader) bulk_wait_group_read0();  // the previous store has read the buffer
          named_bar_sync(1 + t, Cfg::kTileWarps * 32);
          uint8_t* rowp = sbuf + r * 128;
          const int lo = max(cc * 64, hf * HALF_D), hi = min(cc * 64 + 64, (hf + 1) * HALF_D);
#pragma unroll
          for (int col = 0; col < 64; col += 16) {
            if (cc * 64 + col < lo || cc * 64 + col >= hi) continue;
            float o16[16];
            tmem_ld16(trow + Cfg::kOCol + cc * 64 + col, o16);
#pragma unroll
            for (int p = 0; p < 2; ++p)
              *reinterpret_cast<uint4*>(rowp + ((((col >> 3) + p) ^ (r & 7)) << 4)) =
                  make_uint4(pack_bf16x2(o16[8 * p] * inv, o16[8 * p + 1] * inv),
                             pack_bf16x2(o16[8 * p + 2] * inv, o16[8 * p + 3] * inv),
                             pack_bf16x2(o16[8 * p + 4] * inv, o16[8 * p + 5] * inv),
                             pack_bf16x2(o16[8 * p + 6] * inv, o16[8 * p + 7] * inv));
          }
          fence_proxy_async_smem();
          named_bar_sync(1 + t, Cfg::kTileWarps * 32);
          if (leader) {
            tma_store_3d(&tm_o, sbuf, cc * 64, it.q_head0, it.q_begin + t * TQ);
            bulk_commit_group();
          }
        }
      }
      if (!tma_out) {
#pragma unroll
        for (int q = 0; q < HALF_D / 16; ++q) {
          const int col = hf * HALF_D + q * 16;
          float o16[16];
          if (nchunks > 0) {
            tmem_ld16(trow + Cfg::kOCol + col, o16);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) o16[i] = 0.f;
          }
          if (!valid) continue;
          if (it.final_out) {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + row * D + col);
#pragma unroll
            for (int i = 0; i < 2; ++i)
              dst[i] = make_uint4(pack_bf16x2(o16[8 * i] * inv, o16[8 * i + 1] * inv),
                                  pack_bf16x2(o16[8 * i + 2] * inv, o16[8 * i + 3] * inv),
                                  pack_bf16x2(o16[8 * i + 4] * inv, o16[8 * i + 5] * inv),
                                  pack_bf16x2(o16[8 * i + 6] * inv, o16[8 * i + 7] * inv));
          } else {
            float4* dst = reinterpret_cast<float4*>(a.part_acc + (row * a.max_partitions + it.part) * D + col);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_float4(o16[4 * i], o16[4 * i + 1], o16[4 * i + 2], o16[4 * i + 3]);
          }
        }
      }
      if (valid && !it.final_out && hf == 0) {
        a.part_m[row * a.max_partitions + it.part] = m_used;
        a.part_l[row * a.max_partitions + it.part] = l;
      }
      if (nchunks > 0) {
        tmem_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_empty[t]);
        cb += nchunks;
        ++nt;
      }
    }
  }
  // Output stores complete before the CTA (and its staging memory) ends.
  if (Cfg::kTmaOut && warp < SMW && warp % Cfg::kTileWarps == 0 && lane == 0) bulk_wait_group0();
  tmem_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tmem_fence_after_sync();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace pagedkv
