// Paged prefill attention on 5th-generation tensor cores (tcgen05 + TMEM).
//
// What is computed is the causal prefill of prefill_kernel.cuh: new token i
// of a sequence at position p attends to tokens 0..p, read through the block
// table ("What is PagedAttention?", How It Works). Many queries share every
// KV tile, so the products are a dense contraction and this kernel runs them
// as 128-row tcgen05 MMAs with fp32 accumulators in tensor memory:
//
//   CTA = 128 query rows (query tokens x the KV head's group heads) of one
//   sequence, one KV head, one KV partition; Q stays in shared memory.
//   warp 4 (producer): streams 64-token K/V chunks (four 16-token TMA units,
//     128-byte swizzle, laid out so a chunk is one K-major / MN-major UMMA
//     operand) into an NS-stage ring.
//   warp 5 (MMA issuer, one thread): S_j = Q K_j^T (M=128, N=64, K=head_dim)
//     into one of two TMEM buffers, issued one chunk ahead so the tensor core
//     works while the softmax runs; O += P_j V_j (M=128, N=head_dim, K=64)
//     into the TMEM accumulator once P_j is in shared memory.
//   warps 0-3 (softmax): thread r owns row r (TMEM lane r). It reads its 64
//     logits, applies the causal mask, and keeps a running max m used for
//     both P and O; O is rescaled in TMEM only when the max grows by more
//     than 2^8 (so P <= 256 and O never overflows), and P is written as bf16
//     rows of the next MMA's A operand.
// Each stage of the pipeline is handed over through mbarriers (TMA byte
// counts, tcgen05.commit, warp arrivals); every wait is bounded.
#pragma once

#include "prefill_kernel.cuh"

namespace pagedkv {

template <int BS_, int D_>
struct TcCfg {
  static constexpr int BS = BS_;
  static constexpr int D = D_;
  static constexpr int ROWS = 128;                      // MMA M: query rows per CTA
  static constexpr int CHUNK = 64;                      // MMA N of S: KV tokens per step
  static constexpr int UR = 16;                         // TMA unit rows
  static constexpr int UPC = CHUNK / UR;                // units per chunk
  static constexpr int KCH = D * 2 / 128;               // 128-byte column chunks of a row
  static constexpr int kQBytes = ROWS * D * 2;
  static constexpr int kKVBytes = CHUNK * D * 2;        // K (or V) of one chunk
  static constexpr int kStageBytes = 2 * kKVBytes;
  static constexpr int NS = 3;
  static constexpr int kPBytes = ROWS * CHUNK * 2;      // one P buffer
  static constexpr int kBarBytes = 256;
  static constexpr int kSmem = 1024 + kQBytes + NS * kStageBytes + 2 * kPBytes + kBarBytes;
  static constexpr int kThreads = 6 * 32;
  static constexpr uint32_t kTmemCols = 256;            // S0 [0,64) S1 [64,128) O [128,128+D)
  static constexpr uint32_t kOCol = 128;
  static constexpr float kRescaleThreshold = 8.f;       // log2 units
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(BS % UR == 0, "block size");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

template <class Cfg>
__global__ void __launch_bounds__(Cfg::kThreads, 1)
    tc_prefill_kernel(const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const PrefillArgs pf) {
  constexpr int NS = Cfg::NS;
  constexpr int BS = Cfg::BS;
  constexpr int D = Cfg::D;
  constexpr int UR = Cfg::UR;
  constexpr int CHUNK = Cfg::CHUNK;
  constexpr int KCH = Cfg::KCH;
  constexpr int ROWS = Cfg::ROWS;
  const DecodeArgs& a = pf.d;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* qs = smem;                                    // [KCH][ROWS][128 B]
  uint8_t* stages = qs + Cfg::kQBytes;                   // NS x {K [KCH][CHUNK][128 B], V same}
  uint8_t* pbuf = stages + NS * Cfg::kStageBytes;        // 2 x [ROWS][128 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(pbuf + 2 * Cfg::kPBytes);
  uint64_t* full = bars;            // [NS]  TMA bytes landed
  uint64_t* empty = bars + NS;      // [NS]  PV MMA of the stage done (commit)
  uint64_t* s_full = bars + 2 * NS; // [2]   S MMA done (commit)
  uint64_t* s_free = s_full + 2;    // [2]   S read by the 4 softmax warps
  uint64_t* p_full = s_free + 2;    // [2]   P written by the 4 softmax warps
  uint64_t* p_free = p_full + 2;    // [2]   PV MMA done reading P (commit)
  uint64_t* o_done = p_free + 2;    // [1]   PV MMA done (commit), once per chunk
  uint64_t* o_last = o_done + 1;    // [1]   every MMA of the CTA done (commit), once
  uint64_t* q_full = o_last + 1;    // [1]   Q in shared memory (4 warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_full + 1);

  grid_dependents_launch();
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const PrefillItem it = pf.items[blockIdx.x];
  const int G = a.group;
  const int Hkv = a.num_kv_heads;
  const int span0 = it.block_begin * BS;
  const int span_end = min(it.block_end * BS, it.kv_end);
  const int nchunks = span_end > span0 ? (span_end - span0 + CHUNK - 1) / CHUNK : 0;

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&p_free[i], 1);
    }
    mbar_init(o_done, 1);
    mbar_init(o_last, 1);
    mbar_init(q_full, 4);
    fence_barrier_init();
    tma_prefetch_descriptor(&tm_k);
    tma_prefetch_descriptor(&tm_v);
  }
  if (warp == 0) tmem_alloc(tmem_slot, Cfg::kTmemCols);
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ---- producer: K/V chunks ------------------------------------------------------
    const uint64_t policy = l2_policy(2);  // every query tile of a sequence re-reads its blocks
    const int32_t* bt = a.block_tables + static_cast<int64_t>(it.seq) * a.max_blocks_per_seq;
    int issued = 0;
    for (int j = 0; j < nchunks; ++j) {
      const int st = j % NS;
      bool ok = true;
      if (j >= NS) ok = mbar_wait_bounded(&empty[st], ((j / NS) - 1) & 1, a.dev_err);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int c0 = span0 + j * CHUNK;
      const int nu = min(Cfg::UPC, (span_end - c0 + UR - 1) / UR);  // units holding used tokens
      const int phys_l = (lane < nu) ? bt[(c0 + lane * UR) / BS] : -1;
      int phys_u[Cfg::UPC];
#pragma unroll
      for (int u = 0; u < Cfg::UPC; ++u) phys_u[u] = __shfl_sync(0xffffffffu, phys_l, u);
      if (lane == 0) {
        uint8_t* kst = stages + st * Cfg::kStageBytes;
        uint8_t* vst = kst + Cfg::kKVBytes;
        uint32_t bytes = 0;
#pragma unroll
        for (int u = 0; u < Cfg::UPC; ++u)
          if (u < nu && phys_u[u] >= 0 && phys_u[u] < a.num_blocks) bytes += 2 * KCH * UR * 128;
        mbar_arrive_expect_tx(&full[st], bytes);
#pragma unroll
        for (int u = 0; u < Cfg::UPC; ++u) {
          if (u >= nu) continue;
          const int ph = phys_u[u];
          if (ph < 0 || ph >= a.num_blocks) {
            report(a.dev_err, PA_DEVERR_BLOCK_ID);  // the unit keeps stale rows; the call fails
            continue;
          }
          const int32_t y = (ph * Hkv + it.kvh) * BS + ((c0 + u * UR) % BS);
#pragma unroll
          for (int c = 0; c < KCH; ++c) {
            tma_load_2d(kst + c * (CHUNK * 128) + u * (UR * 128), &tm_k, &full[st], c * 64, y, policy);
            tma_load_2d(vst + c * (CHUNK * 128) + u * (UR * 128), &tm_v, &full[st], c * 64, y, policy);
          }
        }
      }
      issued = j + 1;
    }
    // Every copy issued has landed before the CTA's shared memory is released.
    for (int j = max(0, issued - NS); j < issued; ++j)
      mbar_wait_bounded(&full[j % NS], (j / NS) & 1, a.dev_err);
    __syncwarp();
  } else if (warp == 5) {
    // ---- MMA issuer ------------------------------------------------------------------
    if (lane == 0 && nchunks > 0) {
      constexpr uint32_t kIdS = umma_idesc_bf16(ROWS, CHUNK, 0, 0);
      constexpr uint32_t kIdO = umma_idesc_bf16(ROWS, D, 0, 1);
      const uint32_t qa = smem_addr(qs);
      auto issue_s = [&](int j) -> bool {
        const int st = j % NS, b = j & 1;
        if (!mbar_wait_bounded(&full[st], (j / NS) & 1, a.dev_err)) return false;
        if (j >= 2 && !mbar_wait_bounded(&s_free[b], ((j >> 1) - 1) & 1, a.dev_err)) return false;
        tmem_fence_after_sync();
        const uint32_t ka = smem_addr(stages + st * Cfg::kStageBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = umma_desc_sw128(qa + (kk / 4) * (ROWS * 128) + (kk % 4) * 32, 16, 1024);
          const uint64_t bd = umma_desc_sw128(ka + (kk / 4) * (CHUNK * 128) + (kk % 4) * 32, 16, 1024);
          umma_bf16(tmem + b * CHUNK, ad, bd, kIdS, kk > 0);
        }
        umma_commit(&s_full[b]);
        return true;
      };
      bool ok = mbar_wait_bounded(q_full, 0, a.dev_err) && issue_s(0);
      for (int j = 0; j < nchunks && ok; ++j) {
        // S of the next chunk goes to the tensor core before this chunk's P is ready.
        if (j + 1 < nchunks && !issue_s(j + 1)) break;
        const int st = j % NS, b = j & 1;
        if (!mbar_wait_bounded(&p_full[b], (j >> 1) & 1, a.dev_err)) break;
        tmem_fence_after_sync();
        const uint32_t pa = smem_addr(pbuf + b * Cfg::kPBytes);
        const uint32_t va = smem_addr(stages + st * Cfg::kStageBytes + Cfg::kKVBytes);
#pragma unroll
        for (int t = 0; t < CHUNK / 16; ++t) {
          const uint64_t ad = umma_desc_sw128(pa + t * 32, 16, 1024);
          const uint64_t bd = umma_desc_sw128(va + t * (16 * 128), CHUNK * 128, 1024);
          umma_bf16(tmem + Cfg::kOCol, ad, bd, kIdO, j > 0 || t > 0);
        }
        umma_commit(&empty[st]);
        umma_commit(&p_free[b]);
        umma_commit(o_done);
      }
      // o_last completes once every MMA issued above has; TMEM is freed after it.
      umma_commit(o_last);
      mbar_wait_bounded(o_last, 0, a.dev_err);
    }
    __syncwarp();
  } else {
    // ---- softmax warps: thread r owns query row r (TMEM lane r) -----------------------------
    const int r = tid;
    const int jq = r / G;
    const bool valid = jq < it.q_count;
    const int lim = valid ? it.p0 + jq : -1;  // last token this row attends to
    const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
    {
      const int64_t t = it.q_begin + (valid ? jq : 0);
      const int64_t h = static_cast<int64_t>(it.kvh) * G + (r % G);
      const uint4* src = reinterpret_cast<const uint4*>(
          reinterpret_cast<const __nv_bfloat16*>(a.q) + (t * a.num_q_heads + h) * D);
#pragma unroll
      for (int c = 0; c < D * 2 / 16; ++c) {
        const uint4 v = valid ? src[c] : make_uint4(0u, 0u, 0u, 0u);
        const int cc = c >> 3, w = c & 7;
        *reinterpret_cast<uint4*>(qs + cc * (ROWS * 128) + r * 128 + ((w ^ (r & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full);
    }
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;  // warp-uniform
    for (int j = 0; j < nchunks; ++j) {
      const int st = j % NS, b = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s_full[b], (j >> 1) & 1, a.dev_err));
      if (!ok) break;
      tmem_fence_after_sync();
      float sv[CHUNK];
      {
        float t32[32];
        tmem_ld32(tmem + lane_base + b * CHUNK, t32);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[i] = t32[i];
        tmem_ld32(tmem + lane_base + b * CHUNK + 32, t32);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[32 + i] = t32[i];
      }
      tmem_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[b]);
      const int c0 = span0 + j * CHUNK;
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < CHUNK; ++i) {
        const int tok = c0 + i;
        const bool in = tok < span_end && tok <= lim;  // causal: up to the row's own position
        sv[i] = in ? sv[i] * a.scale_log2 : -INFINITY;
        mx = fmaxf(mx, sv[i]);
      }
      // The reference max moves only when the chunk's max exceeds it by more
      // than the threshold; O and l are then scaled by 2^(old - new).
      const bool raise = mx > m_used + Cfg::kRescaleThreshold;
      const bool rescale_o = raise && m_used != -INFINITY;
      if (__any_sync(0xffffffffu, rescale_o)) {
        // O must hold every earlier P V product before it is scaled.
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(o_done, (j - 1) & 1, a.dev_err));
        if (!ok) break;
        tmem_fence_after_sync();
        const float alpha = rescale_o ? fast_exp2(m_used - mx) : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o32[32];
          tmem_ld32(tmem + lane_base + Cfg::kOCol + c * 32, o32);
#pragma unroll
          for (int i = 0; i < 32; ++i) o32[i] *= alpha;
          tmem_st32(tmem + lane_base + Cfg::kOCol + c * 32, o32);
        }
        tmem_fence_before_sync();
        l *= alpha;
      }
      if (raise) m_used = mx;
      // P = 2^(s - m_used) <= 2^8 as bf16: row r of the A operand of P V.
      if (j >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&p_free[b], ((j >> 1) - 1) & 1, a.dev_err));
        if (!ok) break;
      }
      uint8_t* prow = pbuf + b * Cfg::kPBytes + r * 128;
      float rs = 0.f;
#pragma unroll
      for (int w8 = 0; w8 < CHUNK / 8; ++w8) {
        float p[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float x = sv[w8 * 8 + i];
          p[i] = (x == -INFINITY) ? 0.f : fast_exp2(x - m_used);
          rs += p[i];
        }
        const uint4 pk = make_uint4(pack_bf16x2(p[0], p[1]), pack_bf16x2(p[2], p[3]),
                                    pack_bf16x2(p[4], p[5]), pack_bf16x2(p[6], p[7]));
        *reinterpret_cast<uint4*>(prow + ((w8 ^ (r & 7)) << 4)) = pk;
      }
      l += rs;
      // Rows of V past the span hold stale or unloaded data (0 * NaN is NaN): clear them.
      const int vt = span_end - c0;
      if (vt < CHUNK) {
        uint8_t* vst = stages + st * Cfg::kStageBytes + Cfg::kKVBytes;
        const int n16 = (CHUNK - vt) * KCH * 8;
        for (int x = r; x < n16; x += ROWS) {
          const int row = vt + x / (KCH * 8);
          const int rem = x % (KCH * 8);
          *reinterpret_cast<uint4*>(vst + (rem >> 3) * (CHUNK * 128) + row * 128 + ((rem & 7) << 4)) =
              make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);
    }
    // ---- epilogue: O from TMEM, normalised (single partition) or as a partial --------------
    if (ok && nchunks > 0) ok = __all_sync(0xffffffffu, mbar_wait_bounded(o_last, 0, a.dev_err));
    if (ok) {
      tmem_fence_after_sync();
      const int64_t t = it.q_begin + (valid ? jq : 0);
      const int64_t h = static_cast<int64_t>(it.kvh) * G + (r % G);
      const int64_t row = t * a.num_q_heads + h;
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o32[32];
        if (nchunks > 0) {
          tmem_ld32(tmem + lane_base + Cfg::kOCol + c * 32, o32);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o32[i] = 0.f;
        }
        if (!valid) continue;
        if (it.final_out) {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + row * D + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(pack_bf16x2(o32[8 * i] * inv, o32[8 * i + 1] * inv),
                                pack_bf16x2(o32[8 * i + 2] * inv, o32[8 * i + 3] * inv),
                                pack_bf16x2(o32[8 * i + 4] * inv, o32[8 * i + 5] * inv),
                                pack_bf16x2(o32[8 * i + 6] * inv, o32[8 * i + 7] * inv));
        } else {
          float4* dst = reinterpret_cast<float4*>(a.part_acc + (row * a.max_partitions + it.part) * D + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(o32[4 * i], o32[4 * i + 1], o32[4 * i + 2], o32[4 * i + 3]);
        }
      }
      if (valid && !it.final_out) {
        a.part_m[row * a.max_partitions + it.part] = m_used;
        a.part_l[row * a.max_partitions + it.part] = l;
      }
    }
  }
  tmem_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tmem_fence_after_sync();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace pagedkv
