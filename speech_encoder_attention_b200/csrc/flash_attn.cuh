// flash_attn.cuh -- fused multi-head flash attention on Blackwell tensor cores.
//
// Per head:  o_i = sum_{j in A_i} exp(s_ij - m_i) v_j / l_i,  s_ij = scale <q_i, k_j>
// with the running max m and sum l kept in fp32 and no score matrix in memory.
// The edda PR ("Add Edda ASR with DFlash2 speculative decoding", PR
// description) replaces F32 scores materialised for all 1500 frames with flash
// attention over F16 K/V; A_i is every key for the bidirectional encoder
// window, the query's own chunk for the higgs chunked encoder
// ("higgs-audio-v3-stt GGUF", "Architecture note (chunked encoder)"), and the
// query row's ancestor slots for the token-tree verify pass (edda PR
// description, beam search over a token-tree KV cache). The range family
// (FULL, CHUNK, BAND) also takes per-sequence lengths and a causal flag, and
// per-head sinks join the normaliser (drafter PR: causal flag, sliding window,
// attention sinks); those options are a separate compile-time variant (EXT).
//
// Work unit: one 128-row query tile of one (sequence, head) against a range
// of 128-row key/value tiles (the whole sequence, the tile's chunk, or one
// split of the key range). Two CTAs share an SM; for the range masks each CTA
// is persistent and walks units blockIdx.x, blockIdx.x + gridDim.x, ...
//   warps 0-3  softmax: one thread per query row (tensor-memory lane == row,
//              so a row's max and sum never leave the thread); the same
//              threads rescale O when the max grows and write the output.
//   warp 4     TMA producer: Q per unit into a double buffer, K and V tiles
//              through a 2-stage ring, read in place from the (packed)
//              projection buffer through 3-D tensor maps (columns, frames,
//              sequence), so rows past a sequence's end read as zeros.
//   warp 5     tcgen05.mma issuer: S = Q K^T (SS, 128x128x64) into tensor
//              memory, then O += P V (P from tensor memory, V MN-major in
//              shared memory, 128x64x128).
// Tensor memory: S (128 fp32 columns), O (64), P (64 columns of fp16 pairs).
// Between units the next unit's Q load and first S overlap the current
// unit's last softmax, and O is copied to registers before the epilogue's
// stores so the next unit's PV can start.
// Tile skipping: CHUNK walks only the key range of the query tile's chunk(s);
// SLOTMASK skips key tiles whose mask words are zero for every row of the CTA.
// Split-KV: for short query blocks the key range is split over units. Up to 8
// splits of a query tile form a thread-block cluster and merge their
// unnormalised partials through distributed shared memory; more write them to
// the workspace and a combine kernel merges them. Query tiles of at most 32
// rows take the narrow layout (their rows in every lane quadrant, each softmax
// warp a quarter of the key columns, see NARROW below). Every kernel here
// waits (griddepcontrol) after its prologue, so programmatic launches overlap
// that prologue with the previous kernel.
#pragma once

#include "sm100_ptx.cuh"

namespace sea {
namespace fa {

constexpr int BQ = 128;
constexpr int BKV = 128;
constexpr int DH = 64;
constexpr int TILE_BYTES = 128 * DH * 2;  // 16 KB, one 128-row x 64-col fp16 tile
constexpr int MAX_FLAG_WORDS = 16;        // SLOTMASK: up to 512 key tiles (65536 slots)

enum MaskKind : int { kFull = 0, kChunk = 1, kSlotmask = 2, kBand = 3 };

// Division by a launch constant d >= 1 without the integer-divide sequence
// (its reciprocal runs on MUFU, which the softmax keeps saturated): for
// 0 <= n < 2^31, n / d = umulhi(n, m) >> s with l = ceil(log2 d),
// m = ceil(2^(31 + l) / d) and s = l - 1 (division by invariant integers
// using multiplication, Granlund and Montgomery); d = 1 is m = 0. The host
// fills m and s.
struct DivC {
  uint32_t m, s;
  int d;
};

__device__ __forceinline__ int div_c(int n, const DivC& f) {
  return f.m ? static_cast<int>(__umulhi(static_cast<uint32_t>(n), f.m) >> f.s) : n;
}

struct Params {
  int batch, t_q, t_kv, n_heads;
  float scale_log2;  // scale * log2(e)
  int mask_kind;
  int chunk_len;
  const uint32_t* bits;
  int words_per_row;
  // range family: band window, causal flag, optional per-sequence lengths
  int window;
  int causal;
  const int* q_lens;
  const int* kv_lens;
  const float* sinks;  // optional [n_heads] sink logits (units of the scaled scores)
  // query-tile schedule: the query axis is cut into segments of seg_len rows
  // (whole chunks for CHUNK, the whole sequence otherwise), each segment into
  // tiles_per_seg tiles of up to 128 rows.
  int seg_len, tiles_per_seg, q_tiles;
  // key/value split
  int kv_splits, kv_tiles_per_split;
  // work units: batch * n_heads * q_tiles * kv_splits (split fastest)
  int units;
  // the divisions by kv_splits, q_tiles, n_heads, tiles_per_seg, chunk_len
  DivC dv_splits, dv_q_tiles, dv_heads, dv_tiles_per_seg, dv_chunk;
  // outputs
  __half* out;
  int64_t out_stride;
  float* ws_o;   // [splits][batch][heads][t_q][64] unnormalised partial O
  float* ws_ml;  // [splits][batch][heads][t_q][2]  (m in log2 units, l)
  // Split partials merged inside a thread-block cluster (one CTA per split,
  // the cluster = one query tile's splits) instead of through ws_o / ws_ml
  // and the combine kernel.
  int merge;
  uint32_t* err;
  uint64_t limit_ns;
};

// STAGES_: K/V ring depth. Two stages (99.5 KB of shared memory) let two CTAs
// share an SM; launches of at most one CTA per SM (short query blocks) take
// four, so a unit's first four key tiles load at once.
template <int STAGES_ = 2>
struct CfgT {
  static constexpr int SOFTMAX_WARPS = 4;
  static constexpr int SOFTMAX_THREADS = 128;
  static constexpr int PRODUCER_WARP = 4;
  static constexpr int MMA_WARP = 5;
  static constexpr int THREADS = 192;
  static constexpr int MIN_BLOCKS = 2;  // two CTAs per SM (with two stages)
  static constexpr int STAGES = STAGES_;
  static constexpr int TMEM_COLS = 256;
  static constexpr uint32_t S_COL = 0;    // 128 fp32 columns
  static constexpr uint32_t O_COL = 128;  // 64 fp32 columns
  static constexpr uint32_t P_COL = 192;  // 64 columns of fp16 pairs
  static constexpr int OFF_Q = 0;         // two Q buffers
  static constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
  static constexpr int OFF_BARS = OFF_V + STAGES * TILE_BYTES;
  // q_full[2], q_empty[2], k_full[S], v_full[S], kv_empty[S], s_full, s_free,
  // p_full, o_done, o_free, drain, quarters (narrow tiles: the four warps'
  // partials are in shared memory)
  static constexpr int NUM_BARS = 4 + 3 * STAGES + 7;
  static constexpr int OFF_FLAGS = OFF_BARS + 8 * NUM_BARS;
  static constexpr int OFF_MISC = OFF_FLAGS + 4 * MAX_FLAG_WORDS;
  static constexpr int SMEM_BYTES = 1024 + OFF_MISC + 16;
};
using Cfg = CfgT<2>;

// Lazy rescaling: the exponent reference m only moves when a row's max grows
// by more than this (log2 units), so p <= 2^15 fits fp16 and O is rescaled rarely.
constexpr float RESCALE_LIMIT = 15.0f;
constexpr float kLog2e = 1.4426950408889634f;


struct TileGeom {
  int q0;     // first query row (sequence-local)
  int rows;   // valid rows in the tile (0 if none)
};

__device__ __forceinline__ TileGeom q_tile_geom(const Params& p, int qt) {
  TileGeom g{p.t_q, 0};
  if (qt >= p.q_tiles) return g;
  const int seg = div_c(qt, p.dv_tiles_per_seg);
  const int w = qt - seg * p.tiles_per_seg;
  const int seg0 = seg * p.seg_len;
  const int q0 = seg0 + w * BQ;
  const int seg_end = min(seg0 + p.seg_len, p.t_q);
  g.q0 = q0;
  g.rows = max(0, min(BQ, seg_end - q0));
  if (g.rows == 0) g.q0 = p.t_q;
  return g;
}

// Valid query rows and keys of one sequence, and the key position of its query
// row 0 (a query block is the last q positions of its keys).
struct SeqLen {
  int q, kv, off;
};

// EXT: the launch uses lengths, causal, BAND or sinks (a separate compile-time
// variant, so the plain FULL / CHUNK kernel carries none of that code).
template <bool EXT>
__device__ __forceinline__ SeqLen seq_len(const Params& p, int b) {
  SeqLen L{p.t_q, p.t_kv, 0};
  if constexpr (!EXT) return L;
  if (p.q_lens != nullptr) L.q = min(max(__ldg(p.q_lens + b), 0), p.t_q);
  if (p.kv_lens != nullptr) L.kv = min(max(__ldg(p.kv_lens + b), 0), p.t_kv);
  L.off = L.kv - L.q;
  return L;
}

// Keys [lo, hi) that query row i (sequence-local) of the range family may see;
// hi <= lo means none. Both ends are non-decreasing in i.
template <bool EXT>
__device__ __forceinline__ void row_keys(const Params& p, const SeqLen& L, int i, int& lo, int& hi) {
  lo = 0;
  hi = L.kv;
  if constexpr (!EXT) {
    if (p.mask_kind == kChunk) {
      lo = div_c(i, p.dv_chunk) * p.chunk_len;
      hi = min(hi, lo + p.chunk_len);
    }
    return;
  }
  if (i >= L.q) {
    hi = 0;
    return;
  }
  const int pos = i + L.off;
  if (p.mask_kind == kChunk) {
    if (pos < 0) {
      hi = 0;
      return;
    }
    lo = div_c(pos, p.dv_chunk) * p.chunk_len;
    hi = min(hi, lo + p.chunk_len);
  } else if (p.mask_kind == kBand) {
    lo = max(0, pos - p.window + 1);
    hi = min(hi, pos + p.window);
  }
  if (p.causal) hi = min(hi, pos + 1);
}

// One work unit: a query tile of one (sequence, head) and its key-tile range.
struct Unit {
  int b, h, split;
  int q0, rows;          // query rows [q0, q0 + rows) of the sequence
  int kv_lo;             // key index of tile 0
  int j_begin, j_end;    // key tiles [j_begin, j_end) of this unit
};

template <bool EXT>
__device__ __forceinline__ Unit decode_unit(const Params& p, int u) {
  Unit U;
  int r = div_c(u, p.dv_splits);
  U.split = u - r * p.kv_splits;
  const int r2 = div_c(r, p.dv_q_tiles);
  const int qt = r - r2 * p.q_tiles;
  U.b = div_c(r2, p.dv_heads);
  U.h = r2 - U.b * p.n_heads;
  const TileGeom g = q_tile_geom(p, qt);
  U.q0 = g.q0;
  U.rows = g.rows;
  // Keys any valid row of the tile may see: the union of the rows' ranges,
  // which (both ends being monotone) runs from the first row's start to the
  // last valid row's end.
  int lo = 0, hi = 0;
  if (p.mask_kind == kSlotmask) {
    hi = p.t_kv;
  } else if (g.rows > 0) {
    const SeqLen L = seq_len<EXT>(p, U.b);
    const int last = min(g.q0 + g.rows, L.q) - 1;
    if (last >= g.q0) {
      int lo2, hi1;
      row_keys<EXT>(p, L, g.q0, lo, hi1);
      row_keys<EXT>(p, L, last, lo2, hi);
    }
  }
  hi = max(hi, lo);
  U.kv_lo = lo;
  const int n_kv = (hi - lo + BKV - 1) / BKV;
  if (p.kv_splits == 1) {
    U.j_begin = 0;
    U.j_end = n_kv;
  } else {
    U.j_begin = min(n_kv, U.split * p.kv_tiles_per_split);
    U.j_end = min(n_kv, U.j_begin + p.kv_tiles_per_split);
  }
  return U;
}

// SLOT selects the bitmask family (SLOTMASK) at compile time; the range family
// (FULL, CHUNK, BAND, with lengths and causal) carries no bitmask code and runs persistent CTAs. SLOTMASK
// CTAs each own one unit (gridDim.x == units): the tile flags need one pass of
// every row's mask words before any role starts.
//
// NARROW (query tiles of at most 32 rows, one unit per CTA, no key split):
// the tile's rows are loaded four times, into rows 0, 32, 64 and 96 of the Q
// buffer, so every softmax warp holds all of them in its own tensor-memory
// lane quadrant, and warp w takes key columns [32w, 32w + 32) of each key
// tile. Each warp keeps its own running max, sum and O over its quarter of
// the keys (its P columns outside the quarter stay zero, so P V sums only
// its keys); the epilogue merges the four partials through shared memory as
// a split-KV merge does. A thread then exponentiates 32 scores per key tile
// instead of 128, which shortens the per-tile chain of a decode-sized block.
template <bool SLOT, bool EXT, int STAGES = 2, bool NARROW = false>
__global__ void __launch_bounds__(CfgT<STAGES>::THREADS, STAGES == 2 ? 2 : 1)
    flash_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = CfgT<STAGES>;
  constexpr int ST = C::STAGES;
  static_assert(!(SLOT && NARROW), "narrow tiles serve the range masks only");
  constexpr int NC = NARROW ? 32 : BKV;  // score columns a softmax thread holds per key tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::OFF_BARS;
  auto q_full = [&](int i) { return bar0 + 8u * i; };
  auto q_empty = [&](int i) { return bar0 + 8u * (2 + i); };
  auto k_full = [&](int s) { return bar0 + 8u * (4 + s); };
  auto v_full = [&](int s) { return bar0 + 8u * (4 + ST + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (4 + 2 * ST + s); };
  const uint32_t s_full = bar0 + 8u * (4 + 3 * ST);
  const uint32_t s_free = s_full + 8u;
  const uint32_t p_full = s_full + 16u;
  const uint32_t o_done = s_full + 24u;
  const uint32_t o_free = s_full + 32u;
  const uint32_t drain_bar = s_full + 40u;
  const uint32_t quarters_bar = s_full + 48u;
  uint32_t* flags = reinterpret_cast<uint32_t*>(smem + C::OFF_FLAGS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr bool use_flags = SLOT;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full(i), 1);
      mbar_init(q_empty(i), 1);
    }
    for (int s = 0; s < ST; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(p_full, 4);
    mbar_init(o_done, 1);
    mbar_init(o_free, 4);
    mbar_init(drain_bar, 1);
    mbar_init(quarters_bar, 4);
    *abort_flag = 0u;
    fence_barrier_init();
    // The tensor maps are launch parameters, not the previous kernel's data:
    // fetch them before waiting for that kernel.
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (threadIdx.x < MAX_FLAG_WORDS) flags[threadIdx.x] = 0u;
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Everything above touched only this CTA's shared and tensor memory.
  griddep_wait();
  griddep_launch_dependents();
  const WaitCtl wc{abort_flag, p.err, p.limit_ns};
  const int srow = (warp & 3) * 32 + lane;  // softmax: row within the tile == TMEM lane
  // Cluster merge: this CTA's partial O (128 x 64 fp32) and (m, l) per row,
  // in the K/V stages, which no copy or MMA uses once the unit's last P V
  // has completed.
  float* merge_o = reinterpret_cast<float*>(smem + C::OFF_K);
  float2* merge_ml = reinterpret_cast<float2*>(smem + C::OFF_K + BQ * DH * 4);

  // SLOTMASK: mark the key tiles any row of this CTA's (single) unit may see.
  // The producer starts the unit's Q load first: Q does not depend on the
  // flags, and the pass waits on the mask words' global-memory latency.
  bool q_preloaded = false;
  if constexpr (use_flags) {
    const Unit U = decode_unit<EXT>(p, blockIdx.x);
    if (warp == C::PRODUCER_WARP && lane == 0 && U.rows > 0) {
      mbar_arrive_expect_tx(q_full(0), TILE_BYTES);
      tma_load_3d(sbase + C::OFF_Q, &tm_q, q_full(0), U.h * DH, U.q0, U.b);
      q_preloaded = true;
      // Which key tiles load is known only after the pass; meanwhile pull the
      // first ones into L2.
      for (int j = U.j_begin; j < min(U.j_end, U.j_begin + ST); ++j) {
        tma_prefetch_l2_3d(&tm_k, U.h * DH, U.kv_lo + j * BKV, U.b);
        tma_prefetch_l2_3d(&tm_v, U.h * DH, U.kv_lo + j * BKV, U.b);
      }
    }
    if (warp < C::SOFTMAX_WARPS && srow < U.rows) {
      const uint32_t* mrow = p.bits + static_cast<int64_t>(U.q0 + srow) * p.words_per_row;
      for (int j = U.j_begin; j < U.j_end; ++j) {
        const int w0 = j * (BKV / 32);
        uint32_t any = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (w0 + c < p.words_per_row) any |= __ldg(mrow + w0 + c);
        if (any) atomicOr(&flags[j >> 5], 1u << (j & 31));
      }
    }
    __syncthreads();
  }
  auto tile_on = [&](int j) -> bool { return !use_flags || ((flags[j >> 5] >> (j & 31)) & 1u); };

  if (warp == C::PRODUCER_WARP) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int qn = 0, it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        const Unit U = decode_unit<EXT>(p, u);
        if (U.rows == 0 || (!SLOT && U.j_end <= U.j_begin)) continue;  // see the softmax's empty-unit note
        const int qb = qn & 1;
        if (!(q_preloaded && qn == 0)) {
          if (!mbar_wait(q_empty(qb), ((qn >> 1) & 1) ^ 1u, wc)) break;
          mbar_arrive_expect_tx(q_full(qb), TILE_BYTES);
          if constexpr (NARROW) {
            // tm_q's box is 32 rows here: the same rows into each lane quadrant
#pragma unroll
            for (int r = 0; r < 4; ++r)
              tma_load_3d(sbase + C::OFF_Q + qb * TILE_BYTES + r * (TILE_BYTES / 4), &tm_q, q_full(qb), U.h * DH,
                          U.q0, U.b);
          } else {
            tma_load_3d(sbase + C::OFF_Q + qb * TILE_BYTES, &tm_q, q_full(qb), U.h * DH, U.q0, U.b);
          }
        }
        ++qn;
        for (int j = U.j_begin; j < U.j_end; ++j) {
          if (!tile_on(j)) continue;
          const int st = it % ST;
          if (!mbar_wait(kv_empty(st), ((it / ST) & 1) ^ 1u, wc)) {
            ok = false;
            break;
          }
          const int kv0 = U.kv_lo + j * BKV;
          mbar_arrive_expect_tx(k_full(st), TILE_BYTES);
          tma_load_3d(sbase + C::OFF_K + st * TILE_BYTES, &tm_k, k_full(st), U.h * DH, kv0, U.b);
          mbar_arrive_expect_tx(v_full(st), TILE_BYTES);
          tma_load_3d(sbase + C::OFF_V + st * TILE_BYTES, &tm_v, v_full(st), U.h * DH, kv0, U.b);
          ++it;
        }
      }
      // Let the last copies land before the CTA may exit.
      if (qn > 0) mbar_wait_drain(q_full((qn - 1) & 1), ((qn - 1) >> 1) & 1, p.limit_ns);
      for (int i = max(0, it - ST); i < it; ++i) {
        mbar_wait_drain(k_full(i % ST), (i / ST) & 1, p.limit_ns);
        mbar_wait_drain(v_full(i % ST), (i / ST) & 1, p.limit_ns);
      }
    }
  } else if (warp == C::MMA_WARP) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      // Key tile t: S(t) = Q K(t)^T as soon as the softmax has copied S(t-1)
      // out of tensor memory, then O += P(t-1) V(t-1) once the softmax has
      // written P(t-1). Before the first PV of a unit, the softmax must have
      // copied the previous unit's O out (o_free).
      constexpr uint32_t idesc_s = idesc_f16_f32(BQ, BKV, 0, 0);  // Q, K both K-major
      constexpr uint32_t idesc_o = idesc_f16_f32(BQ, DH, 0, 1);   // P K-major (TMEM), V MN-major
      // Descriptors are computed once; advancing K by 16 moves the start
      // address by 32 bytes (Q, K: 2 in descriptor units) or by 16 rows of
      // 128 bytes (V: 128 units); buffers are TILE_BYTES (1024 units) apart.
      const uint64_t q_desc0 = smem_desc_sw128(sbase + C::OFF_Q, 16, 1024);
      const uint64_t k_desc0 = smem_desc_sw128(sbase + C::OFF_K, 16, 1024);
      const uint64_t v_desc0 = smem_desc_sw128(sbase + C::OFF_V, TILE_BYTES, 1024);
      constexpr uint64_t kTileUnits = TILE_BYTES >> 4;
      const uint32_t s_t = tmem_base + C::S_COL, o_t = tmem_base + C::O_COL, p_t = tmem_base + C::P_COL;
      int qn = 0, it = 0;
      bool ok = true;
      // O += P(t) V(t); first == first PV of its unit (overwrites O).
      auto issue_pv = [&](int t, bool first) -> bool {
        const int st = t % ST;
        if (!mbar_wait(v_full(st), (t / ST) & 1, wc)) return false;
        if (first && qn > 1 && !mbar_wait(o_free, (qn - 2) & 1, wc)) return false;
        if (!mbar_wait(p_full, t & 1, wc)) return false;
        tc_fence_after();
        const uint64_t vd = v_desc0 + st * kTileUnits;
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk)
          mma_f16_ts(o_t, p_t + kk * 8, vd + kk * 128, idesc_o, (!first || kk > 0) ? 1u : 0u);
        mma_commit(o_done);
        mma_commit(kv_empty(st));
        return true;
      };
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        const Unit U = decode_unit<EXT>(p, u);
        if (U.rows == 0 || (!SLOT && U.j_end <= U.j_begin)) continue;  // see the softmax's empty-unit note
        const int qb = qn & 1;
        if (!mbar_wait(q_full(qb), (qn >> 1) & 1, wc)) break;
        ++qn;  // qn now counts this unit
        const uint64_t qd = q_desc0 + qb * kTileUnits;
        int prev = -1;
        bool first_pv = true;
        for (int j = U.j_begin; j < U.j_end; ++j) {
          if (!tile_on(j)) continue;
          const int st = it % ST;
          if (!mbar_wait(k_full(st), (it / ST) & 1, wc)) {
            ok = false;
            break;
          }
          if (it > 0 && !mbar_wait(s_free, (it - 1) & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t kd = k_desc0 + st * kTileUnits;
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) mma_f16_ss(s_t, qd + kk * 2, kd + kk * 2, idesc_s, kk > 0 ? 1u : 0u);
          mma_commit(s_full);
          if (prev >= 0) {
            if (!issue_pv(prev, first_pv)) {
              ok = false;
              break;
            }
            first_pv = false;
          }
          prev = it;
          ++it;
        }
        if (!ok) break;
        if (prev >= 0) {
          if (!issue_pv(prev, first_pv)) break;
        } else if (qn > 1 && !mbar_wait(o_free, (qn - 2) & 1, wc)) {
          break;  // a unit without key tiles still consumes its o_free phase
        }
        mma_commit(q_empty(qb));  // Q buffer free once this unit's MMAs finish
      }
      mma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0, p.limit_ns);
    }
  } else if (warp < C::SOFTMAX_WARPS) {
    // ---------------- softmax / correction / epilogue ----------------
    const uint32_t lane_field = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_tmem = tmem_base + C::S_COL + lane_field;
    const uint32_t o_tmem = tmem_base + C::O_COL + lane_field;
    const uint32_t p_tmem = tmem_base + C::P_COL + lane_field;
    const float sl2 = p.scale_log2;
    // NARROW: this warp's key columns of each tile start at cb; its P columns
    // outside them stay zero for the CTA's life.
    const int cb = NARROW ? 32 * (warp & 3) : 0;
    if constexpr (NARROW) {
      uint32_t z[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) z[e] = 0u;
#pragma unroll
      for (int c = 0; c < 8; ++c) tmem_st8_async(p_tmem + c * 8, z);
      tmem_wait_st();
    }
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
      const Unit U = decode_unit<EXT>(p, u);
      if (U.rows == 0) continue;
      const int qrow = NARROW ? lane : srow;  // row within the query tile
      const int row_glob = U.q0 + qrow;       // sequence-local query row
      const bool row_ok = qrow < U.rows;
      if (!SLOT && U.j_end <= U.j_begin) {
        // No key tile (padding rows, rows before the first key, a split past
        // the unit's keys): the rows see no key. In the persistent kernel such
        // a unit touches neither tensor memory nor a barrier in any role, so
        // the softmax cannot complete barrier phases ahead of the MMA thread's
        // parity waits. (A SLOTMASK CTA owns one unit: its empty unit takes
        // the general path.)
        if (row_ok && (!NARROW || (warp & 3) == 0)) {
          const int64_t part =
              ((static_cast<int64_t>(U.split) * p.batch + U.b) * p.n_heads + U.h) * p.t_q + row_glob;
          if (p.kv_splits > 1) {
            float4* dst = p.merge ? reinterpret_cast<float4*>(merge_o + srow * DH)
                                  : reinterpret_cast<float4*>(p.ws_o + part * DH);
#pragma unroll
            for (int v = 0; v < DH / 4; ++v) dst[v] = make_float4(0.f, 0.f, 0.f, 0.f);
            (p.merge ? merge_ml[srow] : reinterpret_cast<float2*>(p.ws_ml)[part]) = make_float2(-INFINITY, 0.f);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<int64_t>(U.b) * p.t_q + row_glob) * p.out_stride +
                                                  U.h * DH);
#pragma unroll
            for (int v = 0; v < DH / 8; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        continue;
      }
      const uint32_t* mask_row =
          (use_flags && row_ok) ? p.bits + static_cast<int64_t>(row_glob) * p.words_per_row : nullptr;
      // Allowed key range of this row for the range family (sequence-local indices).
      int lo_i = 0, hi_i = 0;
      if (!use_flags && row_ok) row_keys<EXT>(p, seq_len<EXT>(p, U.b), row_glob, lo_i, hi_i);
      float m_run = -INFINITY;  // exponent reference (log2 units), lags the true max by <= 15
      float l_run = 0.f;
      int t_unit = 0;  // tiles of this unit done
      for (int j = U.j_begin; j < U.j_end; ++j) {
        if (!tile_on(j)) continue;
        if (!mbar_wait(s_full, it & 1, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float s[NC];
        {
          uint32_t r[NC];
          if constexpr (NARROW)
            tmem_ld32(s_tmem + cb, r);
          else
            tmem_ld128(s_tmem, r);
#pragma unroll
          for (int e = 0; e < NC; ++e) s[e] = __uint_as_float(r[e]);
        }
        // S is in registers: the next tile's S may overwrite it.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);

        const int kv0 = U.kv_lo + j * BKV + cb;  // key index of s[0]
        if constexpr (use_flags) {
          uint32_t wbits[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int wi = (kv0 >> 5) + c;
            wbits[c] = (mask_row != nullptr && wi < p.words_per_row) ? __ldg(mask_row + wi) : 0u;
          }
          const int lim = p.t_kv - kv0;
#pragma unroll
          for (int e = 0; e < 128; ++e)
            if (!((wbits[e >> 5] >> (e & 31)) & 1u) || e >= lim) s[e] = -INFINITY;
        } else {
          // Keys outside the row's range [lo_i, hi_i). Rows past the tile's
          // rows are never stored and need no mask (their scores are finite:
          // zero-filled or real rows).
          const int a = lo_i - kv0;
          const int bnd = hi_i - kv0;
          if (row_ok && (a > 0 || bnd < NC)) {
            if (a <= 0 && bnd >= NC / 2) {
              // Only the end of the range falls in the tile's upper half
              // (the last key tile of a full-range row).
#pragma unroll
              for (int e = NC / 2; e < NC; ++e)
                if (e >= bnd) s[e] = -INFINITY;
            } else {
#pragma unroll
              for (int e = 0; e < NC; ++e)
                if (e < a || e >= bnd) s[e] = -INFINITY;
            }
          }
        }
        // The tile's row max: four independent chains of 3-input max.
        auto row_max = [&]() -> float {
          float mx4[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) mx4[i] = fmaxf(s[i], s[NC - 4 + i]);
#pragma unroll
          for (int e = 4; e < NC - 4; e += 8) {
#pragma unroll
            for (int i = 0; i < 4; ++i) mx4[i] = fmax3(mx4[i], s[e + i], s[e + 4 + i]);
          }
          return fmaxf(fmax3(mx4[0], mx4[1], mx4[2]), mx4[3]);
        };
        // p = 2^(s*scale*log2e - m) on MUFU ex2 (16 lanes per clock per SM),
        // summed in fp32 and written to P as fp16 pairs, 16 keys at a time.
        auto exp_tile = [&](float m_use) -> float {
          const uint64_t sl2x2 = f2_pack(sl2, sl2);
          const uint64_t negm2 = f2_pack(-m_use, -m_use);
          uint64_t acc2[2] = {0ull, 0ull};
#pragma unroll
          for (int c = 0; c < NC / 16; ++c) {
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float x0, x1;
              f2_unpack(f2_fma(f2_pack(s[16 * c + 2 * i], s[16 * c + 2 * i + 1]), sl2x2, negm2), x0, x1);
              const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
              acc2[i & 1] = f2_add(acc2[i & 1], f2_pack(p0, p1));
              pk[i] = pack_half2(p0, p1);
            }
            tmem_st8_async(p_tmem + cb / 2 + c * 8, pk);
          }
          tmem_wait_st();
          float sum0, sum1;
          f2_unpack(f2_add(acc2[0], acc2[1]), sum0, sum1);
          return sum0 + sum1;
        };
        // Move the exponent reference only when the row max grew by more than
        // RESCALE_LIMIT since it was set (lazy rescaling).
        const float mx = row_max();
        const float mx_l2 = mx * sl2;
        const bool grow = mx_l2 > m_run + RESCALE_LIMIT;
        const float m_new = grow ? mx_l2 : m_run;
        const float alpha = grow ? ex2_approx(m_run - m_new) : 1.f;  // 0 while the reference was -inf
        const bool first = t_unit == 0;
        // P and O are still read by this unit's previous PV until it completes
        // (for a unit's first tile the previous unit's epilogue waited already).
        if (!first) {
          if (!mbar_wait(o_done, (it - 1) & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        l_run = l_run * alpha + exp_tile(m_new == -INFINITY ? 0.f : m_new);
        // O holds this unit's earlier PVs (o_done above); this tile's PV is
        // only issued after p_full, so rescale it now.
        if (!first && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t r[32];
            tmem_ld32(o_tmem + c * 32, r);
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(o_tmem + c * 32, r);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        m_run = m_new;
        ++it;
        ++t_unit;
      }
      if (!ok) break;

      // ---------------- epilogue ----------------
      // O / l (or the unnormalised split partial), 32 columns at a time; O is
      // released for the next unit's PV as soon as both halves are in registers.
      const bool have_o = t_unit > 0 && mbar_wait(o_done, (it - 1) & 1, wc);
      if (t_unit > 0 && !have_o) ok = false;
      if (have_o) tc_fence_after();
      if constexpr (NARROW) {
        // The four warps' partials of the tile's rows, merged through shared
        // memory (the K/V stages: this CTA's only unit has no load or MMA
        // left once its last P V is done):
        //   M = max_w m_w,  L = sum_w l_w 2^(m_w - M) [+ 2^(sink*log2e - M)],
        //   o = sum_w O_w 2^(m_w - M) / L.
        // Slot row w*32 + r holds warp w's partial of row r; its 16-byte
        // chunks are rotated by (r mod 16) against bank conflicts.
        float* q_o = reinterpret_cast<float*>(smem + C::OFF_K);
        float2* q_ml = reinterpret_cast<float2*>(smem + C::OFF_K + 4 * 32 * DH * 4);
        const int slot_row = (warp & 3) * 32 + lane;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t r[32];
          if (have_o) {
            tmem_ld32(o_tmem + c * 32, r);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = 0u;
          }
          if (c == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_free);
          }
          float4* dst = reinterpret_cast<float4*>(q_o + slot_row * DH);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[(c * 8 + v) ^ (lane & 15)] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                                         __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
        }
        q_ml[slot_row] = make_float2(m_run, have_o ? l_run : 0.f);
        __syncwarp();
        if (lane == 0) mbar_arrive(quarters_bar);
        if (!mbar_wait(quarters_bar, 0, wc)) {
          ok = false;
          break;
        }
        // Thread (w, lane) writes 16 columns of one row: row slot_row / 4,
        // columns 16 * (slot_row % 4) ...
        const int row = slot_row >> 2, q4 = slot_row & 3;
        if (row < U.rows) {
          float2 ml[4];
          float mx = -INFINITY;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            ml[w] = q_ml[w * 32 + row];
            if (ml[w].y > 0.f) mx = fmaxf(mx, ml[w].x);
          }
          float o[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = 0.f;
          float l = 0.f;
          if (mx != -INFINITY) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              if (ml[w].y > 0.f) {
                const float wgt = ex2_approx(ml[w].x - mx);
                l += ml[w].y * wgt;
                const float4* src = reinterpret_cast<const float4*>(q_o + (w * 32 + row) * DH);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                  const float4 t4 = src[(q4 * 4 + v) ^ (row & 15)];
                  o[4 * v] += t4.x * wgt;
                  o[4 * v + 1] += t4.y * wgt;
                  o[4 * v + 2] += t4.z * wgt;
                  o[4 * v + 3] += t4.w * wgt;
                }
              }
            }
            if constexpr (EXT) {
              if (p.sinks != nullptr) l += ex2_approx(__ldg(p.sinks + U.h) * kLog2e - mx);
            }
          }
          const float inv = l > 0.f ? 1.f / l : 0.f;
          uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<int64_t>(U.b) * p.t_q + U.q0 + row) * p.out_stride +
                                                U.h * DH + 16 * q4);
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            uint4 w4;
            w4.x = pack_half2(o[8 * v + 0] * inv, o[8 * v + 1] * inv);
            w4.y = pack_half2(o[8 * v + 2] * inv, o[8 * v + 3] * inv);
            w4.z = pack_half2(o[8 * v + 4] * inv, o[8 * v + 5] * inv);
            w4.w = pack_half2(o[8 * v + 6] * inv, o[8 * v + 7] * inv);
            dst[v] = w4;
          }
        }
        continue;
      }
      // A sink adds 2^(sink*log2e - m) to the normaliser (split partials get it
      // in the combine step). No visible key: m = -inf, so the output is 0.
      float l_fin = l_run;
      if constexpr (EXT) {
        if (p.sinks != nullptr && p.kv_splits == 1) l_fin += ex2_approx(__ldg(p.sinks + U.h) * kLog2e - m_run);
      }
      const float inv = l_fin > 0.f ? 1.f / l_fin : 0.f;
      const int64_t part =
          ((static_cast<int64_t>(U.split) * p.batch + U.b) * p.n_heads + U.h) * p.t_q + row_glob;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        if (have_o) {
          tmem_ld32(o_tmem + c * 32, r);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = 0u;
        }
        if (c == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(o_free);
        }
        if (!row_ok) continue;
        if (p.kv_splits > 1) {
          float4* dst = p.merge ? reinterpret_cast<float4*>(merge_o + srow * DH + c * 32)
                                : reinterpret_cast<float4*>(p.ws_o + part * DH + c * 32);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                 __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
        } else {
          uint4* dst = reinterpret_cast<uint4*>(
              p.out + (static_cast<int64_t>(U.b) * p.t_q + row_glob) * p.out_stride + U.h * DH + c * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_half2(__uint_as_float(r[8 * v + 0]) * inv, __uint_as_float(r[8 * v + 1]) * inv);
            w.y = pack_half2(__uint_as_float(r[8 * v + 2]) * inv, __uint_as_float(r[8 * v + 3]) * inv);
            w.z = pack_half2(__uint_as_float(r[8 * v + 4]) * inv, __uint_as_float(r[8 * v + 5]) * inv);
            w.w = pack_half2(__uint_as_float(r[8 * v + 6]) * inv, __uint_as_float(r[8 * v + 7]) * inv);
            dst[v] = w;
          }
        }
      }
      if (row_ok && p.kv_splits > 1)
        (p.merge ? merge_ml[srow] : reinterpret_cast<float2*>(p.ws_ml)[part]) = make_float2(m_run, l_run);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (p.merge) {
    // Every CTA of the cluster holds one split's partial of the same query
    // tile. CTA r writes rows r, r + C, r + 2C, ... of the output from all C
    // partials (read through the cluster's shared-memory window):
    //   M = max_s m_s,  L = sum_s l_s 2^(m_s - M) [+ 2^(sink*log2e - M)],
    //   o = sum_s O_s 2^(m_s - M) / L.
    // A thread takes one 4-column chunk of one row at a time and issues the
    // loads of all C partials before using any, so each item costs one round
    // trip through the cluster.
    cluster_sync();
    {
      const Unit U = decode_unit<EXT>(p, blockIdx.x);
      const int nc = p.kv_splits;  // cluster size, at most 8
      const int r = static_cast<int>(cluster_ctarank());
      const int own = U.rows > r ? (U.rows - r + nc - 1) / nc : 0;  // rows this CTA writes
      const uint32_t o_base = smem_u32(merge_o), ml_base = smem_u32(merge_ml);
      float sink_l2 = -INFINITY;
      if constexpr (EXT) {
        if (p.sinks != nullptr) sink_l2 = __ldg(p.sinks + U.h) * kLog2e;
      }
      for (int item = threadIdx.x; item < own * (DH / 4); item += C::THREADS) {
        const int i = r + nc * (item / (DH / 4));  // tile row
        const int c4 = item % (DH / 4);             // 4-column chunk
        float2 ml[8];
        float4 ov[8];
#pragma unroll
        for (int sp = 0; sp < 8; ++sp) {
          if (sp < nc) {
            ml[sp] = ld_shared_cluster_f2(mapa_shared(ml_base + i * 8, sp));
            ov[sp] = ld_shared_cluster_f4(mapa_shared(o_base + (i * DH + 4 * c4) * 4, sp));
          }
        }
        float mx = -INFINITY;
#pragma unroll
        for (int sp = 0; sp < 8; ++sp)
          if (sp < nc && ml[sp].y > 0.f) mx = fmaxf(mx, ml[sp].x);
        float l = 0.f;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        if (mx != -INFINITY) {
#pragma unroll
          for (int sp = 0; sp < 8; ++sp) {
            if (sp < nc && ml[sp].y > 0.f) {
              const float w = ex2_approx(ml[sp].x - mx);
              l += ml[sp].y * w;
              o.x += ov[sp].x * w;
              o.y += ov[sp].y * w;
              o.z += ov[sp].z * w;
              o.w += ov[sp].w * w;
            }
          }
          if (sink_l2 != -INFINITY) l += ex2_approx(sink_l2 - mx);
        }
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint2 h;
        h.x = pack_half2(o.x * inv, o.y * inv);
        h.y = pack_half2(o.z * inv, o.w * inv);
        *reinterpret_cast<uint2*>(p.out + (static_cast<int64_t>(U.b) * p.t_q + U.q0 + i) * p.out_stride + U.h * DH +
                                  4 * c4) = h;
      }
    }
    cluster_sync();  // no CTA leaves while another still reads its partial
  }
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}


// Merges the split-KV partials of one (sequence, head, row) per warp:
//   M = max_s m_s,  L = sum_s l_s 2^(m_s - M) [+ 2^(sink*log2e - M)],
//   o = sum_s O_s 2^(m_s - M) / L.
__global__ void __launch_bounds__(256, 4)
    combine_kernel(const float* __restrict__ ws_o, const float* __restrict__ ws_ml, int splits,
                   int batch, int n_heads, int t_q, const float* __restrict__ sinks, __half* __restrict__ out,
                   int64_t out_stride) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t rows = static_cast<int64_t>(batch) * n_heads * t_q;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (idx >= rows) return;
  const int lane = threadIdx.x & 31;
  const int r = static_cast<int>(idx % t_q);
  const int h = static_cast<int>((idx / t_q) % n_heads);
  const int b = static_cast<int>(idx / (static_cast<int64_t>(t_q) * n_heads));
  const int64_t stride = rows;  // entries between consecutive splits
  const float2* ml_p = reinterpret_cast<const float2*>(ws_ml) + idx;
  const float2* o_p = reinterpret_cast<const float2*>(ws_o + idx * DH) + lane;
  // Lane j holds split 32g + j's (m, l): one round of loads per 32 splits,
  // the max and the sum by warp shuffles.
  float mmax = -INFINITY;
  for (int g = 0; g < splits; g += 32) {
    float m = -INFINITY;
    if (g + lane < splits) {
      const float2 ml = ml_p[(g + lane) * stride];
      if (ml.y > 0.f) m = ml.x;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    mmax = fmaxf(mmax, m);
  }
  float l = 0.f, o0 = 0.f, o1 = 0.f;
  if (mmax != -INFINITY) {
    for (int g = 0; g < splits; g += 32) {
      float w = 0.f, lw = 0.f;
      if (g + lane < splits) {
        const float2 ml = ml_p[(g + lane) * stride];
        if (ml.y > 0.f) {
          w = ex2_approx(ml.x - mmax);
          lw = ml.y * w;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, off);
      l += lw;
      // each lane's two columns of every split in this group, several loads in flight
      const int n = min(32, splits - g);
#pragma unroll 4
      for (int j = 0; j < n; ++j) {
        const float wj = __shfl_sync(0xffffffffu, w, j);
        const float2 ov = o_p[static_cast<int64_t>(g + j) * stride * (DH / 2)];
        o0 += ov.x * wj;
        o1 += ov.y * wj;
      }
    }
    if (sinks != nullptr) l += ex2_approx(__ldg(sinks + h) * kLog2e - mmax);
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  __half2* dst = reinterpret_cast<__half2*>(out + (static_cast<int64_t>(b) * t_q + r) * out_stride + h * DH);
  dst[lane] = __floats2half2_rn(o0 * inv, o1 * inv);
}

}  // namespace fa
}  // namespace sea
