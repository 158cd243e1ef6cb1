// Paged decode attention kernels for sm_100a (templates; instantiated in
// decode_inst_*.cu).
//
// What is computed: for each sequence s and query head h,
//   out[s][h] = softmax(scale * K_s q) V_s over the first ctx_s tokens of the
// KV head that h reads, gathered in logical order through the sequence's
// block table ("What is PagedAttention?", How It Works / Map Logical to
// Physical Blocks). Blocks are visited in logical order and combined with a
// running (online) max/sum, which reproduces the contiguous-layout result
// ("PagedAttention: Optimizing KV Cache in vLLM", section 3).
//
// How (B200 design; the pages describe no kernel, so all of this is ours):
// * Work item = (sequence, KV head, partition of PB blocks). A CTA of W warps
//   takes an item; the pipeline unit is 16 tokens (one block at block size
//   16, half a block at 32). Warp w walks units w, w+W, w+2W, ... Each warp
//   owns an NS-stage ring in shared memory fed by its lane 0 with 2-D TMA
//   loads (cp.async.bulk.tensor) of the unit's K and V tiles, each
//   completing on an mbarrier. Block ids are prefetched 32 at a time into
//   lane registers, one chunk ahead, so the dependent table load is off the
//   critical path.
// * Tiles land in 128-byte-swizzled layout: each 128-byte column chunk of a
//   tile is one TMA box of block_size rows; unit (16 B) u of row r sits at
//   u ^ (r % 8). Row-wise reads and 8x8 ldmatrix reads are bank-conflict free.
// * fp32 path: CUDA cores. Each lane owns head_dim/32 dims; per-token
//   partial dot products are folded across lanes by a transposing butterfly
//   (block_size values in log2(32) shuffle stages), one exp2 per token, p
//   broadcast by shuffles for the p*V accumulate.
// * bf16 path (any group 1..16, MHA included): tensor cores via mma.sync m16n8k16. The
//   group's query rows (padded to 16) are the A operand held in registers;
//   S = Q K^T comes from ldmatrix'ed K tiles, P stays in registers as the A
//   operand of O += P V with V fragments from ldmatrix.trans.
// * After an item, the warps' (m, l, acc) are merged through shared memory;
//   a sequence that fits one partition is written to `out`, otherwise the
//   partition's (m, l, acc) go to the workspace for the merge kernel, which
//   is launched as a programmatic dependent of this one.
// * Persistent mode (split decode): grid = SMs x occupancy; CTAs pull item
//   tickets from a device counter. Every CTA builds the per-sequence partition
//   prefix sum in shared memory to map a ticket to (s, p, kvh). The last CTA to
//   finish resets the counters to zero for the next call.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>

#include "device_common.cuh"

namespace pagedkv {

struct DecodeArgs {
  const void* q;
  void* out;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* part_m;      // [B][Hq][PMAX], log2-domain running max (scaled logits)
  float* part_l;      // [B][Hq][PMAX], running sum of 2^(logit - m)
  float* part_acc;    // [B][Hq][PMAX][D], unnormalised accumulators
  uint32_t* counters; // [0] ticket, [1] finished CTAs (persistent mode)
  // Shared-prefix decode (nullable otherwise): blocks of each sequence
  // already covered by its group's prefix pass, and the number of partial
  // slots that pass filled before this kernel's partitions.
  const int32_t* seq_skip_blocks;
  const int32_t* seq_part_base;
  // Launched as a programmatic dependent of an independent grid whose
  // results the following merge also reads: wait for it before exiting.
  int wait_prior_at_exit;
  // Sliding window (0 = none): attend to tokens max(0, ctx - window) .. ctx-1.
  int window;
  uint32_t* dev_err;
  int num_seqs;
  int num_q_heads;
  int num_kv_heads;
  int group;
  int num_blocks;
  int max_blocks_per_seq;
  int partition_blocks;  // PB
  int max_partitions;    // PMAX = ceil(max_blocks_per_seq / PB)
  float scale_log2;      // scale * log2(e)
  int persistent;        // 1: ticket loop + partials; 0: item = blockIdx.x, whole context
  int l2_hint;           // L2 policy of the KV stream: 0 normal, 1 evict-first, 2 evict-last
  // Balanced split decode (paged_decode_stream_kernel): the number of pieces
  // each (sequence, KV head) was cut into, written by the kernel and read by
  // the merge ([B][Hkv]; NULL for the other kernels), and the most pieces one
  // (sequence, KV head) may be cut into (its partial slots after the base).
  int32_t* seg_pieces;
  int max_pieces;
};

template <typename T, int BS, int D>
struct TileGeom {
  static constexpr int kElt = static_cast<int>(sizeof(T));
  static constexpr int kRowBytes = D * kElt;
  static constexpr int kChunks = kRowBytes / 128;  // TMA boxes per tile
  static constexpr int kBoxCols = 128 / kElt;      // elements per box row
  static constexpr int kChunkBytes = BS * 128;
  static constexpr int kTileBytes = BS * kRowBytes;
  static_assert(kRowBytes % 128 == 0, "head_dim * element size must be a multiple of 128 bytes");
  static_assert(BS % 16 == 0, "block_size must be a multiple of 16");
  // Byte offset of byte `b` of row `row` inside a swizzled tile.
  __device__ __forceinline__ static uint32_t offset(int row, int b) {
    const int chunk = b >> 7;
    const int within = b & 127;
    return static_cast<uint32_t>(chunk * kChunkBytes + row * 128 +
                                 ((((within >> 4) ^ (row & 7)) << 4) | (within & 15)));
  }
};

constexpr int cmax(int a, int b) { return a > b ? a : b; }
constexpr int cmin(int a, int b) { return a < b ? a : b; }

// G_ > 0: CUDA-core path with compile-time group; G_ == 0: tensor-core path,
// runtime group 1..16 (bf16 only). W_ / NS_: warps per CTA and ring stages
// per warp, 0 = the default below.
template <typename T, int BS_, int D_, int G_, int W_ = 0, int NS_ = 0>
struct DecodeCfg {
  using Elt = T;
  static constexpr int BS = BS_;
  static constexpr int D = D_;
  static constexpr int G = G_;
  static constexpr bool kMma = (G_ == 0);
  // The pipeline moves 16-token units: one unit per block at block size 16,
  // two at block size 32 (each warp then always reads the same half of its
  // blocks), so a stage is the same size whatever the block size.
  static constexpr int UR = 16;
  static constexpr int UPB = BS / UR;
  static_assert(BS % UR == 0, "block_size must be a multiple of 16");
  using Geo = TileGeom<T, UR, D>;
  static constexpr int kStageBytes = 2 * Geo::kTileBytes;
  // Warps per CTA and ring stages per warp. Defaults: four warps (two when
  // two stages each would not fit beside the prefix array) and as many
  // stages, 2..4, as fit in 96 KB, so two CTAs share an SM.
  static constexpr int W = W_ > 0 ? W_ : ((4 * 2 * kStageBytes <= 160 * 1024) ? 4 : 2);
  static constexpr int kThreads = 32 * W;
  static_assert(W % UPB == 0, "warps must cover whole blocks");
  static constexpr int NS = NS_ > 0 ? NS_ : cmin(4, cmax(2, 98304 / (W * kStageBytes)));
  static constexpr int kRingBytes = W * NS * kStageBytes;
  static constexpr int kRowsMax = kMma ? 16 : G;
  static constexpr int kMergeBytes = W * kRowsMax * (D + 2) * 4;
  static constexpr int kMainBytes = cmax(kRingBytes, kMergeBytes);
  static constexpr int kBarBytes = W * NS * 8;
  static constexpr int kMiscInts = 8;
  // Dynamic shared memory = 1024 (alignment slack) + main + barriers + misc
  // + (num_seqs + 1) ints of partition prefix in persistent mode. The merge of
  // a sequence's partitions reuses the main area.
  static constexpr int kFixedSmem = 1024 + kMainBytes + kBarBytes + kMiscInts * 4;
  // 227 KB per CTA, leaving room for the prefix array of up to 4096 sequences.
  static_assert(kFixedSmem + 4097 * 4 <= 227 * 1024, "shared memory budget exceeded");
  static_assert(!kMma || sizeof(T) == 2, "tensor-core path is bf16 only");
  static_assert(kMma || D % 32 == 0, "CUDA-core path needs head_dim % 32 == 0");
};

// Transposing butterfly: on entry every lane holds N partial sums (one per
// token); on exit v[0] holds the full 32-lane sum for token (N == 16 ?
// lane >> 1 : lane). Each stage halves the values a lane keeps while pairing
// lanes across one bit.
template <int N>
__device__ __forceinline__ void transpose_reduce(float (&v)[N], int lane) {
  static_assert(N == 16 || N == 32, "block_size 16 or 32");
#pragma unroll
  for (int half = N / 2, mask = 16; half >= 1; half >>= 1, mask >>= 1) {
    const bool upper = (lane & mask) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
    }
  }
  if constexpr (N == 16) v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
}

// ---------------------------------------------------------------------------
// Per-warp state and per-block math: CUDA-core path.
template <class Cfg>
struct SimtWarp {
  using T = typename Cfg::Elt;
  static constexpr int G = Cfg::G;
  static constexpr int D = Cfg::D;
  static constexpr int BS = Cfg::UR;  // rows per unit
  static constexpr int VEC = D / 32;
  using Geo = typename Cfg::Geo;

  float qf[G][VEC];
  float m[G];
  float l[G];
  float acc[G][VEC];

  __device__ __forceinline__ void begin(const T* q_group, float scale_log2, int lane) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      load_vec_f32<T, VEC>(q_group + h * D + lane * VEC, qf[h]);
#pragma unroll
      for (int j = 0; j < VEC; ++j) {
        qf[h][j] *= scale_log2;
        acc[h][j] = 0.f;
      }
      m[h] = -INFINITY;
      l[h] = 0.f;
    }
  }

  // Tokens nfirst <= t < nvalid of the unit take part (nfirst > 0 only in the
  // first unit of a sliding window).
  __device__ __forceinline__ void block(const uint8_t* kt, uint8_t* vt, int nfirst, int nvalid,
                                        int lane) {
    const int byte_off = lane * VEC * Geo::kElt;
    const int my_token = (BS == 16) ? (lane >> 1) : lane;
    const bool counts = (BS == 32) || ((lane & 1) == 0);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float v[BS];
#pragma unroll
      for (int t = 0; t < BS; ++t) {
        float kf[VEC];
        load_vec_f32<T, VEC>(reinterpret_cast<const T*>(kt + Geo::offset(t, byte_off)), kf);
        float d = 0.f;
#pragma unroll
        for (int j = 0; j < VEC; ++j) d = fmaf(qf[h][j], kf[j], d);
        v[t] = d;
      }
      transpose_reduce<BS>(v, lane);
      const float s = (my_token >= nfirst && my_token < nvalid) ? v[0] : -INFINITY;
      const float m_new = fmaxf(m[h], warp_max(s));
      const float alpha = fast_exp2(m[h] - m_new);
      const float p = fast_exp2(s - m_new);
      l[h] = l[h] * alpha + (counts ? p : 0.f);
      m[h] = m_new;
#pragma unroll
      for (int j = 0; j < VEC; ++j) acc[h][j] *= alpha;
#pragma unroll
      for (int t = 0; t < BS; ++t) {
        if (t >= nfirst && t < nvalid) {  // warp-uniform; rows outside may hold anything
          const float pt = __shfl_sync(0xffffffffu, p, (BS == 16) ? 2 * t : t);
          float vf[VEC];
          load_vec_f32<T, VEC>(reinterpret_cast<const T*>(vt + Geo::offset(t, byte_off)), vf);
#pragma unroll
          for (int j = 0; j < VEC; ++j) acc[h][j] = fmaf(pt, vf[j], acc[h][j]);
        }
      }
    }
  }

  // Writes rows 0..G-1 as final outputs (acc / l) to out_rows (G rows of D
  // contiguous elements); a row with l == 0 gets zeros.
  __device__ __forceinline__ void store_final(T* out_rows, int lane) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float lt = warp_sum(l[h]);
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
#pragma unroll
      for (int j = 0; j < VEC; ++j) out_rows[h * D + lane * VEC + j] = Elt<T>::from_f32(acc[h][j] * inv);
    }
  }

  // Writes rows 0..G-1 as partials (m, l, unnormalised acc) to slots
  // pr0 + h * row_stride.
  __device__ __forceinline__ void store_partials(const DecodeArgs& a, int64_t pr0, int64_t row_stride,
                                                 int lane) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float lt = warp_sum(l[h]);
      const int64_t pr = pr0 + h * row_stride;
      if (lane == 0) {
        a.part_m[pr] = m[h];
        a.part_l[pr] = lt;
      }
#pragma unroll
      for (int j = 0; j < VEC; ++j) a.part_acc[pr * D + lane * VEC + j] = acc[h][j];
    }
  }

  // Writes this warp's state (rows 0..G-1) into the merge area.
  __device__ __forceinline__ void publish(float* sm_m, float* sm_l, float* sm_acc, int lane) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float lt = warp_sum(l[h]);
      if (lane == 0) {
        sm_m[h] = m[h];
        sm_l[h] = lt;
      }
#pragma unroll
      for (int j = 0; j < VEC; ++j) sm_acc[h * D + lane * VEC + j] = acc[h][j];
    }
  }
};

// ---------------------------------------------------------------------------
// Per-warp state and per-block math: tensor-core path (bf16, group <= 16).
template <class Cfg>
struct MmaWarp {
  static constexpr int D = Cfg::D;
  static constexpr int BS = Cfg::UR;  // rows per unit
  static constexpr int KS = D / 16;   // k-steps of S = Q K^T
  static constexpr int NT = BS / 8;   // 8-token n-tiles of S
  static constexpr int ND = D / 8;    // 8-dim n-tiles of O
  using Geo = typename Cfg::Geo;

  uint32_t qa[KS][4];
  float o[ND][4];
  float m[2];
  float l[2];
  float scale_log2;

  __device__ __forceinline__ void begin(const __nv_bfloat16* q_group, int group, float scale,
                                        int lane) {
    const int g = lane >> 2;
    begin_rows(q_group + g * D, q_group + (g + 8) * D, g < group, g + 8 < group, scale, lane);
  }

  // Query rows g and g+8 of this warp's 16-row tile come from row0 / row1
  // (each head_dim contiguous bf16); an invalid row contributes zeros.
  __device__ __forceinline__ void begin_rows(const __nv_bfloat16* row0, const __nv_bfloat16* row1,
                                             bool valid0, bool valid1, float scale, int lane) {
    const int t4 = lane & 3;
    const uint32_t* r0 = reinterpret_cast<const uint32_t*>(row0);
    const uint32_t* r1 = reinterpret_cast<const uint32_t*>(row1);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int c0 = ks * 16 + 2 * t4;
      qa[ks][0] = valid0 ? r0[c0 >> 1] : 0u;
      qa[ks][1] = valid1 ? r1[c0 >> 1] : 0u;
      qa[ks][2] = valid0 ? r0[(c0 + 8) >> 1] : 0u;
      qa[ks][3] = valid1 ? r1[(c0 + 8) >> 1] : 0u;
    }
#pragma unroll
    for (int n = 0; n < ND; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    m[0] = m[1] = -INFINITY;
    l[0] = l[1] = 0.f;
    scale_log2 = scale;
  }

  __device__ __forceinline__ void block(const uint8_t* kt, uint8_t* vt, int nfirst, int nvalid,
                                        int lane) {
    const uint8_t* kts[1] = {kt};
    uint8_t* vts[1] = {vt};
    block_units<1>(kts, vts, nfirst, nvalid, lane);
  }

  // U consecutive 16-token units (tiles kts[u], vts[u]) in one online-softmax
  // step: the U*2 independent S tiles give the tensor pipe more to overlap
  // and the max/sum shuffles are paid once per U*16 tokens. Tokens
  // nfirst <= t < nvalid of the span (counted from its first token) take
  // part; the caller guarantees at least one.
  //
  // kRowLimits (causal prefill): in addition, token t counts for fragment row
  // g only while t <= lim0 and for row g+8 only while t <= lim1; a row with
  // no token in the span keeps its state (guards against -inf - -inf).
  template <int U, bool kRowLimits = false>
  __device__ __forceinline__ void block_units(const uint8_t* const (&kts)[U], uint8_t* const (&vts)[U],
                                              int nfirst, int nvalid, int lane, int lim0 = 0,
                                              int lim1 = 0) {
    const int t4 = lane & 3;
    const int mj = lane >> 3;  // which 8x8 matrix this lane addresses
    const int mr = lane & 7;   // which row of it
    constexpr int NTU = NT * U;

    float s[NTU][4];
#pragma unroll
    for (int n = 0; n < NTU; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t kbase = smem_addr(kts[u]);
#pragma unroll
        for (int sub = 0; sub < BS / 16; ++sub) {
          const int tok = sub * 16 + (mj >> 1) * 8 + mr;
          const int dim = ks * 16 + (mj & 1) * 8;
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4(kbase + Geo::offset(tok, dim * 2), b0, b1, b2, b3);
          mma_bf16_16816(s[u * NT + 2 * sub], qa[ks], b0, b1);
          mma_bf16_16816(s[u * NT + 2 * sub + 1], qa[ks], b2, b3);
        }
      }
    }
    // Scale, mask tokens past the context, online softmax per query row.
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int n = 0; n < NTU; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = n * 8 + 2 * t4 + (e & 1);
        bool in = tok >= nfirst && tok < nvalid;
        if constexpr (kRowLimits) in = in && tok <= ((e < 2) ? lim0 : lim1);
        s[n][e] = in ? s[n][e] * scale_log2 : -INFINITY;
      }
      mx0 = fmaxf(mx0, fmaxf(s[n][0], s[n][1]));
      mx1 = fmaxf(mx1, fmaxf(s[n][2], s[n][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    float mn0 = fmaxf(m[0], mx0);
    float mn1 = fmaxf(m[1], mx1);
    float a0, a1;
    if constexpr (kRowLimits) {
      // A row with nothing valid so far has mn == -inf: keep alpha 1, p 0.
      a0 = (mn0 == -INFINITY) ? 1.f : fast_exp2(m[0] - mn0);
      a1 = (mn1 == -INFINITY) ? 1.f : fast_exp2(m[1] - mn1);
    } else {
      a0 = fast_exp2(m[0] - mn0);
      a1 = fast_exp2(m[1] - mn1);
    }
    m[0] = mn0;
    m[1] = mn1;
    if constexpr (kRowLimits) {
      if (mn0 == -INFINITY) mn0 = 0.f;   // every s of the row is -inf: 2^(-inf) = 0
      if (mn1 == -INFINITY) mn1 = 0.f;
    }
    float r0 = 0.f, r1 = 0.f;
#pragma unroll
    for (int n = 0; n < NTU; ++n) {
      s[n][0] = fast_exp2(s[n][0] - mn0);
      s[n][1] = fast_exp2(s[n][1] - mn0);
      s[n][2] = fast_exp2(s[n][2] - mn1);
      s[n][3] = fast_exp2(s[n][3] - mn1);
      r0 += s[n][0] + s[n][1];
      r1 += s[n][2] + s[n][3];
    }
    l[0] = l[0] * a0 + r0;
    l[1] = l[1] * a1 + r1;
#pragma unroll
    for (int n = 0; n < ND; ++n) {
      o[n][0] *= a0;
      o[n][1] *= a0;
      o[n][2] *= a1;
      o[n][3] *= a1;
    }
    // Rows of V outside [nfirst, nvalid) may hold anything (even NaN bit
    // patterns); p is 0 there but 0 * NaN is NaN, so clear them in shared
    // memory.
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int lo = nfirst - u * BS;   // rows [0, lo) and [hi, BS) are outside
      const int hi = nvalid - u * BS;
      if (lo > 0 || hi < BS) {
        constexpr int kUnitsPerRow = Geo::kRowBytes / 16;
        for (int x = lane; x < BS * kUnitsPerRow; x += 32) {
          const int row = x / kUnitsPerRow;
          if (row < lo || row >= hi) {
            const int b = (x % kUnitsPerRow) * 16;
            *reinterpret_cast<uint4*>(vts[u] + Geo::offset(row, b)) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        fence_proxy_async_smem();  // the stage is refilled by TMA later
        __syncwarp();
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t vbase = smem_addr(vts[u]);
#pragma unroll
      for (int kk = 0; kk < BS / 16; ++kk) {
        const int n0 = u * NT + 2 * kk;
        uint32_t pa[4];
        pa[0] = pack_bf16x2(s[n0][0], s[n0][1]);
        pa[1] = pack_bf16x2(s[n0][2], s[n0][3]);
        pa[2] = pack_bf16x2(s[n0 + 1][0], s[n0 + 1][1]);
        pa[3] = pack_bf16x2(s[n0 + 1][2], s[n0 + 1][3]);
#pragma unroll
        for (int nd = 0; nd < D / 16; ++nd) {
          const int tok = kk * 16 + (mj & 1) * 8 + mr;
          const int dim = nd * 16 + (mj >> 1) * 8;
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4_trans(vbase + Geo::offset(tok, dim * 2), b0, b1, b2, b3);
          mma_bf16_16816(o[2 * nd], pa, b0, b1);
          mma_bf16_16816(o[2 * nd + 1], pa, b2, b3);
        }
      }
    }
  }

  // Writes rows g and g+8 as final outputs (acc / l, bf16) to out0 / out1
  // when valid0 / valid1; a row with l == 0 gets zeros.
  __device__ __forceinline__ void store_final(__nv_bfloat16* out0, __nv_bfloat16* out1, bool valid0,
                                              bool valid1, int lane) {
    const int t4 = lane & 3;
    float l0 = l[0], l1 = l[1];
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float i0 = l0 > 0.f ? 1.f / l0 : 0.f;
    const float i1 = l1 > 0.f ? 1.f / l1 : 0.f;
#pragma unroll
    for (int n = 0; n < ND; ++n) {
      if (valid0)
        *reinterpret_cast<uint32_t*>(out0 + n * 8 + 2 * t4) = pack_bf16x2(o[n][0] * i0, o[n][1] * i0);
      if (valid1)
        *reinterpret_cast<uint32_t*>(out1 + n * 8 + 2 * t4) = pack_bf16x2(o[n][2] * i1, o[n][3] * i1);
    }
  }

  // Writes this warp's rows g (slot pr0) and g+8 (slot pr1) as partials
  // (m, l, unnormalised acc); a negative slot is skipped.
  __device__ __forceinline__ void store_partials(const DecodeArgs& a, int64_t pr0, int64_t pr1,
                                                 int lane) {
    const int t4 = lane & 3;
    float l0 = l[0], l1 = l[1];
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (pr0 >= 0) {
      if (t4 == 0) {
        a.part_m[pr0] = m[0];
        a.part_l[pr0] = l0;
      }
#pragma unroll
      for (int n = 0; n < ND; ++n)
        *reinterpret_cast<float2*>(a.part_acc + pr0 * D + n * 8 + 2 * t4) = make_float2(o[n][0], o[n][1]);
    }
    if (pr1 >= 0) {
      if (t4 == 0) {
        a.part_m[pr1] = m[1];
        a.part_l[pr1] = l1;
      }
#pragma unroll
      for (int n = 0; n < ND; ++n)
        *reinterpret_cast<float2*>(a.part_acc + pr1 * D + n * 8 + 2 * t4) = make_float2(o[n][2], o[n][3]);
    }
  }

  __device__ __forceinline__ void publish(float* sm_m, float* sm_l, float* sm_acc, int group,
                                          int lane) {
    const int g = lane >> 2;
    const int t4 = lane & 3;
    float l0 = l[0], l1 = l[1];
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (g < group) {
      if (t4 == 0) {
        sm_m[g] = m[0];
        sm_l[g] = l0;
      }
#pragma unroll
      for (int n = 0; n < ND; ++n) {
        sm_acc[g * D + n * 8 + 2 * t4] = o[n][0];
        sm_acc[g * D + n * 8 + 2 * t4 + 1] = o[n][1];
      }
    }
    if (g + 8 < group) {
      if (t4 == 0) {
        sm_m[g + 8] = m[1];
        sm_l[g + 8] = l1;
      }
#pragma unroll
      for (int n = 0; n < ND; ++n) {
        sm_acc[(g + 8) * D + n * 8 + 2 * t4] = o[n][2];
        sm_acc[(g + 8) * D + n * 8 + 2 * t4 + 1] = o[n][3];
      }
    }
  }
};

// Number of partitions of a sequence with context length ctx (at least one, so
// that an empty sequence still gets its zero output written).
__device__ __forceinline__ int partitions_of(int ctx, int bs, int pb) {
  const int nb = (ctx + bs - 1) / bs;
  const int p = (nb + pb - 1) / pb;
  return p > 1 ? p : 1;
}

__device__ __forceinline__ int clamp_ctx(int raw, int max_tokens) {
  return (raw < 0 || raw > max_tokens) ? 0 : raw;
}

// Leading blocks of sequence s that a shared-prefix pass already covered:
// at most its full blocks.
__device__ __forceinline__ int first_token(const DecodeArgs& a, int ctx) {
  return (a.window > 0 && ctx > a.window) ? ctx - a.window : 0;
}

__device__ __forceinline__ int skip_blocks(const DecodeArgs& a, int s, int ctx, int bs) {
  int k = first_token(a, ctx) / bs;  // blocks wholly before a sliding window
  if (a.seq_skip_blocks != nullptr) {
    const int full = ctx / bs;
    const int g = a.seq_skip_blocks[s];
    k = max(k, g < 0 ? 0 : (g > full ? full : g));
  }
  return k;
}

// Partitions the split kernel makes for sequence s (its blocks after the
// skipped prefix; at least one).
__device__ __forceinline__ int seq_partitions(const DecodeArgs& a, int s, int max_tokens, int bs) {
  const int ctx = clamp_ctx(a.context_lens[s], max_tokens);
  return partitions_of(ctx - skip_blocks(a, s, ctx, bs) * bs, bs, a.partition_blocks);
}


template <class Cfg>
__global__ void __launch_bounds__(Cfg::kThreads)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const DecodeArgs a) {
  using T = typename Cfg::Elt;
  using Geo = typename Cfg::Geo;
  constexpr int W = Cfg::W;
  constexpr int NS = Cfg::NS;
  constexpr int BS = Cfg::BS;
  constexpr int UR = Cfg::UR;
  constexpr int UPB = Cfg::UPB;
  constexpr int WB = W / UPB;  // warps per unit-half: block lanes
  constexpr int D = Cfg::D;
  constexpr int NT = Cfg::kThreads;
  using WarpT = typename std::conditional<Cfg::kMma, MmaWarp<Cfg>, SimtWarp<Cfg>>::type;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kMainBytes);
  int* misc = reinterpret_cast<int*>(smem + Cfg::kMainBytes + Cfg::kBarBytes);
  int* prefix = misc + Cfg::kMiscInts;  // [num_seqs + 1], persistent mode only
  float* sm_m = reinterpret_cast<float*>(smem);                // [W][rows]
  float* sm_l = sm_m + W * Cfg::kRowsMax;                      // [W][rows]
  float* sm_acc = sm_l + W * Cfg::kRowsMax;                    // [W][rows][D]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int hu = warp % UPB;  // which 16-token half of each block this warp reads
  const int wb = warp / UPB;  // this warp's block lane
  const int B = a.num_seqs;
  const int Hkv = a.num_kv_heads;
  const int G = a.group;
  const int max_tokens = a.max_blocks_per_seq * BS;

  // Let the merge grid (launched as a programmatic dependent) be scheduled
  // now; it waits on the device for this grid's completion before it reads.
  grid_dependents_launch();

  if (tid == 0) {
    for (int i = 0; i < W * NS; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
    tma_prefetch_descriptor(&tm_k);
    tma_prefetch_descriptor(&tm_v);
    misc[0] = 0;  // timeout flag
  }

  int total_items;
  if (a.persistent) {
    // prefix[i] = number of partitions of sequences 0..i-1 (exclusive scan).
    __shared__ int warp_tot[W];
    const int chunk = (B + NT - 1) / NT;
    const int lo = min(B, tid * chunk);
    const int hi = min(B, lo + chunk);
    int mine = 0;
    for (int i = lo; i < hi; ++i) mine += seq_partitions(a, i, max_tokens, BS);
    int incl = mine;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += warp_tot[w];
    int run = base + incl - mine;
    for (int i = lo; i < hi; ++i) {
      prefix[i] = run;
      run += seq_partitions(a, i, max_tokens, BS);
    }
    if (tid == NT - 1) prefix[B] = base + incl;
    __syncthreads();
    total_items = prefix[B] * Hkv;
  } else {
    total_items = B * Hkv;
  }
  __syncthreads();

  const uint64_t policy = l2_policy(a.l2_hint);
  uint32_t gcount = 0;  // units this warp has consumed so far (ring position)

  int item;
  if (a.persistent) {
    if (tid == 0) misc[2] = static_cast<int>(atomicAdd(&a.counters[0], 1u));
    __syncthreads();
    item = misc[2];
  } else {
    item = blockIdx.x;
  }
  int iter = 0;

  while (item < total_items) {
    // Ask for the next ticket now; the atomic's latency overlaps this item.
    if (a.persistent && tid == 0)
      misc[3 + (iter & 1)] = static_cast<int>(atomicAdd(&a.counters[0], 1u));

    // ---- decode the item ----------------------------------------------------
    int s, p, kvh, nparts;
    if (a.persistent) {
      const int pi = item / Hkv;
      kvh = item - pi * Hkv;
      int lo = 0, hi = B - 1;  // last s with prefix[s] <= pi
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= pi) lo = mid; else hi = mid - 1;
      }
      s = lo;
      p = pi - prefix[s];
      nparts = prefix[s + 1] - prefix[s];
    } else {
      s = item / Hkv;
      kvh = item - s * Hkv;
      p = 0;
      nparts = 1;
    }
    const int ctx_raw = a.context_lens[s];
    const int ctx = clamp_ctx(ctx_raw, max_tokens);
    if (ctx != ctx_raw && p == 0 && kvh == 0 && tid == 0) report(a.dev_err, PA_DEVERR_CONTEXT_LEN);
    const int nb = (ctx + BS - 1) / BS;
    const int skip = a.persistent ? skip_blocks(a, s, ctx, BS) : 0;
    const int win_first = a.persistent ? first_token(a, ctx) : 0;
    const int part_base = (a.persistent && a.seq_part_base) ? a.seq_part_base[s] : 0;
    const int b_begin = a.persistent ? skip + p * a.partition_blocks : 0;
    const int b_end = a.persistent ? min(nb, b_begin + a.partition_blocks) : nb;
    const int nblk = max(0, b_end - b_begin);
    // This warp reads half `hu` of blocks b_begin + wb + j*WB.
    const int nbj = (nblk > wb) ? (nblk - wb + WB - 1) / WB : 0;
    int nj = nbj;
    if (UPB > 1 && hu > 0 && nbj > 0) {
      const int last_lb = b_begin + wb + (nbj - 1) * WB;
      if (ctx - last_lb * BS <= hu * UR) nj -= 1;  // the context ends before this half
    }

    // ---- per-warp pipeline over its units -----------------------------------------
    const T* q_group = reinterpret_cast<const T*>(a.q) +
                       (static_cast<int64_t>(s) * a.num_q_heads + static_cast<int64_t>(kvh) * G) * D;
    WarpT st;
    if constexpr (Cfg::kMma) {
      st.begin(q_group, G, a.scale_log2, lane);
    } else {
      st.begin(q_group, a.scale_log2, lane);
    }

    const int32_t* bt = a.block_tables + static_cast<int64_t>(s) * a.max_blocks_per_seq + b_begin + wb;
    int bt_cur = (lane < nbj) ? bt[lane * WB] : -1;
    int bt_nxt = (32 + lane < nbj) ? bt[(32 + lane) * WB] : -1;
    int bt_chunk = 0;
    uint32_t bad = 0;  // bit per stage: the stage's block id was out of range
    uint8_t* my_ring = ring + warp * NS * Cfg::kStageBytes;
    uint64_t* my_bars = bars + warp * NS;

    auto issue = [&](int j) {
      const int c = j >> 5;
      if (c != bt_chunk) {  // advance the block-id window by one chunk
        bt_cur = bt_nxt;
        bt_nxt = ((c + 1) * 32 + lane < nbj) ? bt[((c + 1) * 32 + lane) * WB] : -1;
        bt_chunk = c;
      }
      const int phys = __shfl_sync(0xffffffffu, bt_cur, j & 31);
      const uint32_t stage = (gcount + j) % NS;
      const bool good = phys >= 0 && phys < a.num_blocks;
      bad = good ? (bad & ~(1u << stage)) : (bad | (1u << stage));
      if (lane == 0) {
        uint64_t* bar = &my_bars[stage];
        fence_proxy_async_smem();
        if (good) {
          uint8_t* kdst = my_ring + stage * Cfg::kStageBytes;
          uint8_t* vdst = kdst + Geo::kTileBytes;
          const int32_t y = (phys * Hkv + kvh) * BS + hu * UR;
          mbar_arrive_expect_tx(bar, 2 * Geo::kTileBytes);
#pragma unroll
          for (int c2 = 0; c2 < Geo::kChunks; ++c2) {
            tma_load_2d(kdst + c2 * Geo::kChunkBytes, &tm_k, bar, c2 * Geo::kBoxCols, y, policy);
            tma_load_2d(vdst + c2 * Geo::kChunkBytes, &tm_v, bar, c2 * Geo::kBoxCols, y, policy);
          }
        } else {
          report(a.dev_err, PA_DEVERR_BLOCK_ID);
          mbar_arrive(bar);  // completes the phase with no data
        }
      }
    };

    const int npre = min(NS, nj);
    for (int j = 0; j < npre; ++j) issue(j);
    bool timed_out = false;
    int j = 0;
    for (; j < nj; ++j) {
      const uint32_t g = gcount + j;
      const uint32_t stage = g % NS;
      const uint32_t parity = (g / NS) & 1u;
      const bool okw = mbar_wait_bounded(&my_bars[stage], parity, a.dev_err);
      if (!__all_sync(0xffffffffu, okw)) {
        timed_out = true;
        break;
      }
      if (!(bad & (1u << stage))) {
        const int lb = b_begin + wb + j * WB;  // logical block
        const int u0 = lb * BS + hu * UR;      // first token of the unit
        const int nvalid = min(UR, ctx - u0);
        const int nfirst = win_first - u0;     // > 0 only inside a window's first block
        if (nfirst < nvalid) {                 // a unit wholly before the window is skipped
          uint8_t* kt = my_ring + stage * Cfg::kStageBytes;
          st.block(kt, kt + Geo::kTileBytes, nfirst, nvalid, lane);
        }
      }
      __syncwarp();
      if (j + NS < nj) issue(j + NS);
    }
    if (timed_out) {
      // Give copies still in flight a bounded chance to land before leaving.
      for (int jj = j; jj < min(nj, j + NS); ++jj) {
        const uint32_t g = gcount + jj;
        mbar_wait_bounded(&my_bars[g % NS], (g / NS) & 1u, a.dev_err);
      }
      if (lane == 0) misc[0] = 1;
    }
    gcount += nj;

    // ---- merge the W warps' partial states ------------------------------------------
    __syncthreads();  // every warp is done with the ring; it becomes the merge area
    if constexpr (Cfg::kMma) {
      st.publish(sm_m + warp * Cfg::kRowsMax, sm_l + warp * Cfg::kRowsMax,
                 sm_acc + warp * Cfg::kRowsMax * D, G, lane);
    } else {
      st.publish(sm_m + warp * Cfg::kRowsMax, sm_l + warp * Cfg::kRowsMax,
                 sm_acc + warp * Cfg::kRowsMax * D, lane);
    }
    __syncthreads();
    const bool final_out = (nparts == 1) && (part_base == 0);
    const int64_t row0 = static_cast<int64_t>(s) * a.num_q_heads + static_cast<int64_t>(kvh) * G;
    for (int idx = tid; idx < G * D; idx += NT) {
      const int h = idx / D;
      const int d = idx - h * D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < W; ++w) M = fmaxf(M, sm_m[w * Cfg::kRowsMax + h]);
      float L = 0.f, A = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < W; ++w) {
          const float e = fast_exp2(sm_m[w * Cfg::kRowsMax + h] - M);
          L = fmaf(sm_l[w * Cfg::kRowsMax + h], e, L);
          A = fmaf(sm_acc[(w * Cfg::kRowsMax + h) * D + d], e, A);
        }
      }
      const int64_t row = row0 + h;
      if (final_out) {
        reinterpret_cast<T*>(a.out)[row * D + d] = Elt<T>::from_f32(L > 0.f ? A / L : 0.f);
      } else {
        const int64_t pr = row * a.max_partitions + part_base + p;
        a.part_acc[pr * D + d] = A;
        if (d == 0) {
          a.part_m[pr] = M;
          a.part_l[pr] = L;
        }
      }
    }
    fence_proxy_async_smem();  // generic accesses to the ring precede the next TMA writes
    __syncthreads();  // merge area reads done before the ring is refilled
    if (misc[0]) break;

    if (a.persistent) {
      item = misc[3 + (iter & 1)];
    } else {
      item = total_items;
    }
    ++iter;
  }

  if (a.wait_prior_at_exit) grid_dependency_wait();
  if (a.persistent && tid == 0) {
    // The last CTA to get here resets the counters for the next call; every
    // other CTA has already taken its final ticket.
    __threadfence();
    const uint32_t prev = atomicAdd(&a.counters[1], 1u);
    if (prev == gridDim.x - 1) {
      atomicExch(&a.counters[0], 0u);
      atomicExch(&a.counters[1], 0u);
      __threadfence();
    }
  }
}

// Log-sum-exp merge of partition partials. One warp per (sequence, query
// head) row with more than one partial (rows with one were written by the
// decode kernel), four rows per CTA; no shared memory and no CTA barrier.
// Lane i holds partition p = i (and i + 32, ...)'s m_p and l_p: the warp
// finds M = max_p m_p and L = sum_p l_p 2^(m_p - M) by shuffles. Each lane
// owns head_dim / 32 columns of the output and accumulates
// out = sum_p acc_p 2^(m_p - M) / L in partition order, with the weights
// broadcast from the lanes that hold them. The accumulators of the first
// kMergeBatch partitions are loaded together with every m_p and l_p, before
// M is known, and later ones kMergeBatch at a time, so a row of up to
// kMergeBatch partials costs one dependent round trip to L2 (two up to
// 2 * kMergeBatch).
constexpr int kMergeRowsPerCta = 4;

// VEC consecutive floats (VEC * 4 bytes aligned) in 8- or 16-byte loads.
template <int VEC>
__device__ __forceinline__ void load_f32s(const float* p, float (&v)[VEC]) {
  if constexpr (VEC % 4 == 0) {
#pragma unroll
    for (int q = 0; q < VEC / 4; ++q) {
      const float4 x = reinterpret_cast<const float4*>(p)[q];
      v[4 * q] = x.x; v[4 * q + 1] = x.y; v[4 * q + 2] = x.z; v[4 * q + 3] = x.w;
    }
  } else {
    static_assert(VEC == 2, "head_dim 64, 128 or 256");
    const float2 x = *reinterpret_cast<const float2*>(p);
    v[0] = x.x; v[1] = x.y;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(32 * kMergeRowsPerCta)
    lse_merge_kernel(const DecodeArgs a, int block_size) {
  constexpr int VEC = D / 32;
  // partitions whose accumulators are in flight at once: 64 floats per lane
  constexpr int kMergeBatch = 64 / VEC < 32 ? 64 / VEC : 32;
  grid_dependency_wait();  // the decode grid's partials are complete and visible
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kMergeRowsPerCta + (threadIdx.x >> 5);
  if (row >= static_cast<int64_t>(a.num_seqs) * a.num_q_heads) return;
  const int s = static_cast<int>(row / a.num_q_heads);
  const int base_parts = a.seq_part_base ? a.seq_part_base[s] : 0;
  const int own = a.seg_pieces != nullptr
                      ? a.seg_pieces[static_cast<int64_t>(s) * a.num_kv_heads +
                                     (row - static_cast<int64_t>(s) * a.num_q_heads) / a.group]
                      : seq_partitions(a, s, a.max_blocks_per_seq * block_size, block_size);
  const int np = min(base_parts + own, a.max_partitions);
  if (np <= 1 && base_parts == 0) return;
  const int64_t base = row * a.max_partitions;
  const float* src = a.part_acc + base * D + lane * VEC;

  // first batch of accumulators, then every partition's m and l
  float v[kMergeBatch][VEC];
  const int n_first = min(kMergeBatch, np);
#pragma unroll
  for (int u = 0; u < kMergeBatch; ++u)
    if (u < n_first) load_f32s<VEC>(src + static_cast<int64_t>(u) * D, v[u]);
  const float m_lane = lane < np ? a.part_m[base + lane] : -INFINITY;
  const float l_lane = lane < np ? a.part_l[base + lane] : 0.f;
  float M = m_lane;
  for (int p = lane + 32; p < np; p += 32) M = fmaxf(M, a.part_m[base + p]);
  M = warp_max(M);
  float L = lane < np ? l_lane * fast_exp2(m_lane - M) : 0.f;
  for (int p = lane + 32; p < np; p += 32) L += a.part_l[base + p] * fast_exp2(a.part_m[base + p] - M);
  L = warp_sum(L);

  float acc[VEC];
#pragma unroll
  for (int j = 0; j < VEC; ++j) acc[j] = 0.f;
  for (int p0 = 0; p0 < np; p0 += 32) {
    // this lane's weight for partition p0 + lane, broadcast below
    const float wl = p0 == 0 ? (lane < np ? fast_exp2(m_lane - M) : 0.f)
                             : ((p0 + lane < np) ? fast_exp2(a.part_m[base + p0 + lane] - M) : 0.f);
    const int n = min(32, np - p0);
    for (int k = 0; k < n; k += kMergeBatch) {
      const int cnt = min(kMergeBatch, n - k);
      if (p0 + k > 0) {
#pragma unroll
        for (int u = 0; u < kMergeBatch; ++u)
          if (u < cnt) load_f32s<VEC>(src + static_cast<int64_t>(p0 + k + u) * D, v[u]);
      }
#pragma unroll
      for (int u = 0; u < kMergeBatch; ++u) {
        if (u < cnt) {
          const float w = __shfl_sync(0xffffffffu, wl, k + u);
#pragma unroll
          for (int j = 0; j < VEC; ++j) acc[j] = fmaf(v[u][j], w, acc[j]);
        }
      }
    }
  }
  const float inv = (L > 0.f) ? 1.f / L : 0.f;
  T* dst = reinterpret_cast<T*>(a.out) + row * D + lane * VEC;
#pragma unroll
  for (int j = 0; j < VEC; ++j) dst[j] = Elt<T>::from_f32(acc[j] * inv);
}

}  // namespace pagedkv
