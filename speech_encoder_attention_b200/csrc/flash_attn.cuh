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
// description, beam search over a token-tree KV cache).
//
// One CTA owns NQ query tiles of 128 rows of one (sequence, head) and walks a
// range of 128-row key/value tiles:
//   warps [0, 4*NQ)  softmax: one thread per query row (tensor-memory lane ==
//                    row, so a row's max and sum never leave the thread); the
//                    same threads rescale O when the max grows and write the
//                    normalised output.
//   warp 4*NQ        TMA producer: Q once, then K and V tiles through a
//                    3-stage ring, read in place from the (packed) projection
//                    buffer through 3-D tensor maps (columns, frames, sequence),
//                    so rows past a sequence's end read as zeros.
//   warp 4*NQ+1      tcgen05.mma issuer: S = Q K^T (SS, 128x128x64) into tensor
//                    memory, then O += P V (P from tensor memory, V MN-major in
//                    shared memory, 128x64x128).
// Tensor memory per query tile: S (128 fp32 columns), O (64), P (64 columns of
// packed fp16 pairs).
// Tile skipping: CHUNK walks only the key range of the query tile's chunk(s);
// SLOTMASK skips key tiles whose mask words are zero for every row of the CTA.
// Split-KV: for short query blocks the key range is split over CTAs; each
// writes unnormalised O with its m and l to the workspace and a combine kernel
// merges them.
#pragma once

#include "sm100_ptx.cuh"

namespace sea {
namespace fa {

constexpr int BQ = 128;
constexpr int BKV = 128;
constexpr int DH = 64;
constexpr int TILE_BYTES = 128 * DH * 2;  // 16 KB, one 128-row x 64-col fp16 tile
constexpr int MAX_FLAG_WORDS = 16;        // SLOTMASK: up to 512 key tiles (65536 slots)

enum MaskKind : int { kFull = 0, kChunk = 1, kSlotmask = 2 };

struct Params {
  int batch, t_q, t_kv, n_heads;
  float scale_log2;  // scale * log2(e)
  int mask_kind;
  int chunk_len;
  const uint32_t* bits;
  int words_per_row;
  // query-tile schedule: the query axis is cut into segments of seg_len rows
  // (whole chunks for CHUNK, the whole sequence otherwise), each segment into
  // tiles_per_seg tiles of up to 128 rows.
  int seg_len, tiles_per_seg, q_tiles;
  // key/value split
  int kv_splits, kv_tiles_per_split;
  // outputs
  __half* out;
  int64_t out_stride;
  float* ws_o;   // [splits][batch][heads][t_q][64] unnormalised partial O
  float* ws_ml;  // [splits][batch][heads][t_q][2]  (m in log2 units, l)
  uint32_t* err;
  uint64_t limit_ns;
};

template <int NQ>
struct Cfg {
  // One softmax warpgroup per query tile, one thread per score row.
  static constexpr int SOFTMAX_WARPS = 4 * NQ;
  static constexpr int SOFTMAX_THREADS = 32 * SOFTMAX_WARPS;
  static constexpr int PRODUCER_WARP = SOFTMAX_WARPS;
  static constexpr int MMA_WARP = SOFTMAX_WARPS + 1;
  static constexpr int THREADS = SOFTMAX_THREADS + 64;
  static constexpr int TMEM_COLS = NQ == 1 ? 256 : 512;
  // Single-tile CTAs run two per SM (256 tensor-memory columns and a 2-stage
  // K/V ring each), so one CTA's MMAs fill the other's pipeline drains.
  static constexpr int STAGES = NQ == 1 ? 2 : 3;
  static constexpr int MIN_BLOCKS = NQ == 1 ? 2 : 1;
  // Per query tile q: S (128 fp32 columns), O (64 fp32), P (64 columns of fp16
  // pairs). P has its own columns so the next S can be computed while the
  // softmax of this one runs.
  __host__ __device__ static constexpr uint32_t S_COL(int q) { return 128u * q; }
  __host__ __device__ static constexpr uint32_t O_COL(int q) { return 128u * NQ + 64u * q; }
  __host__ __device__ static constexpr uint32_t P_COL(int q) { return 128u * NQ + 64u * NQ + 64u * q; }
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQ * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
  static constexpr int OFF_BARS = OFF_V + STAGES * TILE_BYTES;
  // q_full, k_full[S], v_full[S], kv_empty[S], s_full[NQ], s_free[NQ], p_full[NQ], o_done[NQ], drain
  static constexpr int NUM_BARS = 1 + 3 * STAGES + 4 * NQ + 1;
  static constexpr int OFF_FLAGS = OFF_BARS + 8 * NUM_BARS;
  static constexpr int OFF_MISC = OFF_FLAGS + 4 * MAX_FLAG_WORDS;
  static constexpr int SMEM_BYTES = 1024 + OFF_MISC + 16;
};

// Lazy rescaling: the exponent reference m only moves when a row's max grows
// by more than this (log2 units), so p <= 2^8 fits fp16 and O is rescaled rarely.
constexpr float RESCALE_THRESHOLD = 8.0f;

// Bit k set: pair k (mod 8) of every 16 keys takes the FMA-pipe exp2 instead
// of MUFU ex2. Measured on B200 the extra instructions cost more than the
// MUFU relief buys in this kernel, so no pair is moved.
constexpr uint32_t POLY_PAIRS = 0x00u;

struct TileGeom {
  int q0;     // first query row (sequence-local)
  int rows;   // valid rows in the tile (0 if none)
};

__device__ __forceinline__ TileGeom q_tile_geom(const Params& p, int qt) {
  TileGeom g{p.t_q, 0};
  if (qt >= p.q_tiles) return g;
  const int seg = qt / p.tiles_per_seg;
  const int w = qt - seg * p.tiles_per_seg;
  const int seg0 = seg * p.seg_len;
  const int q0 = seg0 + w * BQ;
  const int seg_end = min(seg0 + p.seg_len, p.t_q);
  g.q0 = q0;
  g.rows = max(0, min(BQ, seg_end - q0));
  if (g.rows == 0) g.q0 = p.t_q;
  return g;
}

// SLOT selects the bitmask family (SLOTMASK) at compile time; the range family
// (FULL, CHUNK) carries no bitmask code in its inner loop.
template <int NQ, bool SLOT>
__global__ void __launch_bounds__(Cfg<NQ>::THREADS, Cfg<NQ>::MIN_BLOCKS)
    flash_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = Cfg<NQ>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::OFF_BARS;
  const uint32_t q_full = bar0;
  auto k_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto v_full = [&](int s) { return bar0 + 8u * (1 + C::STAGES + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (1 + 2 * C::STAGES + s); };
  auto s_full = [&](int q) { return bar0 + 8u * (1 + 3 * C::STAGES + q); };
  auto s_free = [&](int q) { return bar0 + 8u * (1 + 3 * C::STAGES + NQ + q); };
  auto p_full = [&](int q) { return bar0 + 8u * (1 + 3 * C::STAGES + 2 * NQ + q); };
  auto o_done = [&](int q) { return bar0 + 8u * (1 + 3 * C::STAGES + 3 * NQ + q); };
  const uint32_t drain_bar = bar0 + 8u * (1 + 3 * C::STAGES + 4 * NQ);
  uint32_t* flags = reinterpret_cast<uint32_t*>(smem + C::OFF_FLAGS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x % p.kv_splits;
  const int qgroup = blockIdx.x / p.kv_splits;
  const int h = blockIdx.y;
  const int b = blockIdx.z;

  // Query tiles of this CTA and the key range they need.
  TileGeom geom[NQ];
  int any_rows = 0;
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    geom[q] = q_tile_geom(p, qgroup * NQ + q);
    any_rows |= geom[q].rows;
  }
  if (!any_rows) return;  // uniform for the whole CTA: nothing allocated yet

  int kv_lo = 0, kv_hi = p.t_kv;
  if (p.mask_kind == kChunk) {
    int lo = INT_MAX, hi = 0;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      if (geom[q].rows == 0) continue;
      lo = min(lo, (geom[q].q0 / p.chunk_len) * p.chunk_len);
      const int last = geom[q].q0 + geom[q].rows - 1;
      hi = max(hi, min((last / p.chunk_len + 1) * p.chunk_len, p.t_kv));
    }
    kv_lo = lo;
    kv_hi = hi;
  }
  const int n_kv = (kv_hi - kv_lo + BKV - 1) / BKV;
  const int j_begin = min(n_kv, split * p.kv_tiles_per_split);
  const int j_end = min(n_kv, j_begin + p.kv_tiles_per_split);
  constexpr bool use_flags = SLOT;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    for (int q = 0; q < NQ; ++q) {
      mbar_init(s_full(q), 1);
      mbar_init(s_free(q), 4);
      mbar_init(p_full(q), 4);
      mbar_init(o_done(q), 1);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0u;
    fence_barrier_init();
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
  const WaitCtl wc{abort_flag, p.err, p.limit_ns};

  // Softmax-thread identity (meaningful for warp < SOFTMAX_WARPS).
  const int sq = min(warp >> 2, NQ - 1);     // query tile of this thread
  const int srow = (warp & 3) * 32 + lane;   // row within the tile == TMEM lane
  const int row_glob = geom[sq].q0 + srow;   // sequence-local query row
  const bool row_ok = warp < C::SOFTMAX_WARPS && srow < geom[sq].rows;
  const uint32_t* mask_row =
      (use_flags && row_ok) ? p.bits + static_cast<int64_t>(row_glob) * p.words_per_row : nullptr;

  // SLOTMASK: mark key tiles that any row of this CTA may see.
  if constexpr (use_flags) {
    if (mask_row != nullptr) {
      for (int j = j_begin; j < j_end; ++j) {
        const int w0 = j * (BKV / 32);
        uint32_t any = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (w0 + c < p.words_per_row) any |= __ldg(mask_row + w0 + c);
        if (any) atomicOr(&flags[j >> 5], 1u << (j & 31));
      }
    }
    __syncthreads();
  }
  auto tile_on = [&](int j) -> bool { return !use_flags || ((flags[j >> 5] >> (j & 31)) & 1u); };

  if (warp == C::PRODUCER_WARP) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(q_full, NQ * TILE_BYTES);
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        tma_load_3d(sbase + C::OFF_Q + q * TILE_BYTES, &tm_q, q_full, h * DH, geom[q].q0, b);
      int it = 0;
      for (int j = j_begin; j < j_end; ++j) {
        if (!tile_on(j)) continue;
        const int st = it % C::STAGES;
        const uint32_t ph = (it / C::STAGES) & 1;
        if (!mbar_wait(kv_empty(st), ph ^ 1u, wc)) break;
        const int kv0 = kv_lo + j * BKV;
        mbar_arrive_expect_tx(k_full(st), TILE_BYTES);
        tma_load_3d(sbase + C::OFF_K + st * TILE_BYTES, &tm_k, k_full(st), h * DH, kv0, b);
        mbar_arrive_expect_tx(v_full(st), TILE_BYTES);
        tma_load_3d(sbase + C::OFF_V + st * TILE_BYTES, &tm_v, v_full(st), h * DH, kv0, b);
        ++it;
      }
      // Let the copies land before the CTA may exit.
      mbar_wait_drain(q_full, 0, p.limit_ns);
      for (int i = max(0, it - C::STAGES); i < it; ++i) {
        mbar_wait_drain(k_full(i % C::STAGES), (i / C::STAGES) & 1, p.limit_ns);
        mbar_wait_drain(v_full(i % C::STAGES), (i / C::STAGES) & 1, p.limit_ns);
      }
    }
  } else if (warp == C::MMA_WARP) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      // Key tile i: S_q(i) = Q_q K(i)^T as soon as the softmax of query tile q
      // has copied S_q(i-1) out of tensor memory, then O_q += P_q(i-1) V(i-1)
      // once that softmax has written P_q(i-1).
      constexpr uint32_t idesc_s = idesc_f16_f32(BQ, BKV, 0, 0);  // Q, K both K-major
      constexpr uint32_t idesc_o = idesc_f16_f32(BQ, DH, 0, 1);   // P K-major (TMEM), V MN-major
      // Descriptors are computed once; advancing K by 16 moves the start
      // address by 32 bytes (Q, K: 2 in descriptor units) or by 16 rows of
      // 128 bytes (V: 128 units); stages are TILE_BYTES (1024 units) apart.
      const uint64_t q_desc0 = smem_desc_sw128(sbase + C::OFF_Q, 16, 1024);
      const uint64_t k_desc0 = smem_desc_sw128(sbase + C::OFF_K, 16, 1024);
      const uint64_t v_desc0 = smem_desc_sw128(sbase + C::OFF_V, TILE_BYTES, 1024);
      constexpr uint64_t kTileUnits = TILE_BYTES >> 4;
      bool ok = mbar_wait(q_full, 0, wc);
      int it = 0;
      int prev_st = 0;
      auto issue_pv = [&](int st, int idx) -> bool {
        if (!mbar_wait(v_full(st), (idx / C::STAGES) & 1, wc)) return false;
        const uint64_t vd = v_desc0 + st * kTileUnits;
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          if (!mbar_wait(p_full(q), idx & 1, wc)) return false;
          tc_fence_after();
          const uint32_t o_t = tmem_base + C::O_COL(q), p_t = tmem_base + C::P_COL(q);
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk)
            mma_f16_ts(o_t, p_t + kk * 8, vd + kk * 128, idesc_o, (idx > 0 || kk > 0) ? 1u : 0u);
          mma_commit(o_done(q));
        }
        mma_commit(kv_empty(st));
        return true;
      };
      for (int j = j_begin; j < j_end && ok; ++j) {
        if (!tile_on(j)) continue;
        const int st = it % C::STAGES;
        if (!mbar_wait(k_full(st), (it / C::STAGES) & 1, wc)) {
          ok = false;
          break;
        }
        const uint64_t kd = k_desc0 + st * kTileUnits;
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          if (it > 0 && !mbar_wait(s_free(q), (it - 1) & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t qd = q_desc0 + q * kTileUnits;
          const uint32_t s_t = tmem_base + C::S_COL(q);
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) mma_f16_ss(s_t, qd + kk * 2, kd + kk * 2, idesc_s, kk > 0 ? 1u : 0u);
          mma_commit(s_full(q));
        }
        if (!ok) break;
        if (it > 0 && !issue_pv(prev_st, it - 1)) {
          ok = false;
          break;
        }
        prev_st = st;
        ++it;
      }
      if (ok && it > 0) issue_pv(prev_st, it - 1);
      mma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0, p.limit_ns);
    }
  } else if (warp < C::SOFTMAX_WARPS) {
    // ---------------- softmax / correction / epilogue ----------------
    const int q = sq;
    const uint32_t lane_field = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_tmem = tmem_base + C::S_COL(q) + lane_field;
    const uint32_t o_tmem = tmem_base + C::O_COL(q) + lane_field;
    const uint32_t p_tmem = tmem_base + C::P_COL(q) + lane_field;
    // Allowed key range of this row for FULL / CHUNK (sequence-local indices).
    int lo_i = 0, hi_i = p.t_kv;
    if (p.mask_kind == kChunk) {
      lo_i = (row_glob / p.chunk_len) * p.chunk_len;
      hi_i = min(lo_i + p.chunk_len, p.t_kv);
    }
    if (!row_ok) {
      lo_i = 0;
      hi_i = 0;
    }
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;  // exponent reference (log2 units), lags the true max by < 8
    float l_run = 0.f;
    int it = 0;
    bool ok = true;
    for (int j = j_begin; j < j_end; ++j) {
      if (!tile_on(j)) continue;
      if (!mbar_wait(s_full(q), it & 1, wc)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[128];
      {
        uint32_t r[128];
        tmem_ld128(s_tmem, r);
#pragma unroll
        for (int e = 0; e < 128; ++e) s[e] = __uint_as_float(r[e]);
      }
      // S is in registers: the next tile's S may overwrite it.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free(q));

      const int kv0 = kv_lo + j * BKV;  // key index of s[0]
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
        const int a = lo_i - kv0;
        const int bnd = hi_i - kv0;
        if (a > 0 || bnd < BKV) {
#pragma unroll
          for (int e = 0; e < 128; ++e)
            if (e < a || e >= bnd) s[e] = -INFINITY;
        }
      }
      // row max: eight independent chains of 3-input max, then a short tree
      float mx;
      {
        float mx8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = s[i];
#pragma unroll
        for (int e = 8; e < 128; e += 16) {
#pragma unroll
          for (int i = 0; i < 8; ++i) mx8[i] = fmax3(mx8[i], s[e + i], s[e + 8 + i]);
        }
        mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
      }
      const float mx_l2 = mx * sl2;
      // Move the reference only when the max grew by more than the threshold.
      const bool grow = mx_l2 > m_run + RESCALE_THRESHOLD;
      const float m_new = grow ? mx_l2 : m_run;
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = grow ? ex2_approx(m_run - m_use) : 1.f;
      // P and O are still read by the previous tile's PV until it completes.
      if (it > 0) {
        if (!mbar_wait(o_done(q), (it - 1) & 1, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      // p = 2^(s*scale*log2e - m), summed in fp32 and written to P as fp16
      // pairs, 32 keys at a time. MUFU ex2 serves 16 lanes per clock per SM;
      // pairs picked by POLY_PAIRS take the FMA-pipe exp2 instead.
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      const uint64_t negm2 = f2_pack(-m_use, -m_use);
      uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0, x1, p0, p1;
          f2_unpack(f2_fma(f2_pack(s[32 * c + 2 * i], s[32 * c + 2 * i + 1]), sl2x2, negm2), x0, x1);
          if ((POLY_PAIRS >> (i & 7)) & 1) {
            exp2_poly_x2(x0, x1, p0, p1);
          } else {
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          acc2[i & 3] = f2_add(acc2[i & 3], f2_pack(p0, p1));
          pk[i] = pack_half2(p0, p1);
        }
        tmem_st16_async(p_tmem + c * 16, pk);
      }
      tmem_wait_st();
      float sum0, sum1;
      f2_unpack(f2_add(f2_add(acc2[0], acc2[1]), f2_add(acc2[2], acc2[3])), sum0, sum1);
      l_run = l_run * alpha + (sum0 + sum1);
      // O holds the PV of every earlier tile (o_done above), and this tile's
      // PV is only issued after p_full, so rescale it now.
      if (it > 0 && __any_sync(0xffffffffu, grow)) {
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
      if (lane == 0) mbar_arrive(p_full(q));
      m_run = m_new;
      ++it;
    }

    // ---------------- epilogue ----------------
    // O / l (or the unnormalised split partial), 32 columns at a time.
    const bool have_o = ok && it > 0 && mbar_wait(o_done(q), (it - 1) & 1, wc);
    if (have_o) tc_fence_after();
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    const int64_t part =
        ((static_cast<int64_t>(split) * p.batch + b) * p.n_heads + h) * p.t_q + row_glob;
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      uint32_t r[32];
      if (have_o) {
        tmem_ld32(o_tmem + c * 32, r);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = 0u;
      }
      if (!row_ok) continue;
      if (p.kv_splits > 1) {
        float4* dst = reinterpret_cast<float4*>(p.ws_o + part * DH + c * 32);
#pragma unroll
        for (int v = 0; v < 8; ++v)
          dst[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                               __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
      } else {
        uint4* dst = reinterpret_cast<uint4*>(
            p.out + (static_cast<int64_t>(b) * p.t_q + row_glob) * p.out_stride + h * DH + c * 32);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 u;
          u.x = pack_half2(__uint_as_float(r[8 * v + 0]) * inv, __uint_as_float(r[8 * v + 1]) * inv);
          u.y = pack_half2(__uint_as_float(r[8 * v + 2]) * inv, __uint_as_float(r[8 * v + 3]) * inv);
          u.z = pack_half2(__uint_as_float(r[8 * v + 4]) * inv, __uint_as_float(r[8 * v + 5]) * inv);
          u.w = pack_half2(__uint_as_float(r[8 * v + 6]) * inv, __uint_as_float(r[8 * v + 7]) * inv);
          dst[v] = u;
        }
      }
    }
    if (row_ok && p.kv_splits > 1) reinterpret_cast<float2*>(p.ws_ml)[part] = make_float2(m_run, l_run);
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// Merges the split-KV partials of one (sequence, head, row) per warp:
//   M = max_s m_s,  L = sum_s l_s 2^(m_s - M),  o = sum_s O_s 2^(m_s - M) / L.
__global__ void __launch_bounds__(256)
    combine_kernel(const float* __restrict__ ws_o, const float* __restrict__ ws_ml, int splits,
                   int batch, int n_heads, int t_q, __half* __restrict__ out, int64_t out_stride) {
  const int64_t rows = static_cast<int64_t>(batch) * n_heads * t_q;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (idx >= rows) return;
  const int lane = threadIdx.x & 31;
  const int r = static_cast<int>(idx % t_q);
  const int h = static_cast<int>((idx / t_q) % n_heads);
  const int b = static_cast<int>(idx / (static_cast<int64_t>(t_q) * n_heads));
  const int64_t stride = rows;  // entries between consecutive splits
  float mmax = -INFINITY;
  for (int s = 0; s < splits; ++s) {
    const float2 ml = reinterpret_cast<const float2*>(ws_ml)[idx + s * stride];
    if (ml.y > 0.f) mmax = fmaxf(mmax, ml.x);
  }
  float l = 0.f, o0 = 0.f, o1 = 0.f;
  if (mmax != -INFINITY) {
    for (int s = 0; s < splits; ++s) {
      const float2 ml = reinterpret_cast<const float2*>(ws_ml)[idx + s * stride];
      if (!(ml.y > 0.f)) continue;
      const float w = ex2_approx(ml.x - mmax);
      l += ml.y * w;
      const float2 ov = reinterpret_cast<const float2*>(ws_o + (idx + s * stride) * DH)[lane];
      o0 += ov.x * w;
      o1 += ov.y * w;
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  __half2* dst = reinterpret_cast<__half2*>(out + (static_cast<int64_t>(b) * t_q + r) * out_stride + h * DH);
  dst[lane] = __floats2half2_rn(o0 * inv, o1 * inv);
}

}  // namespace fa
}  // namespace sea
