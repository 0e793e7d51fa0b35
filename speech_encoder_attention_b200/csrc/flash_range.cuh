// flash_range.cuh -- flash attention for the range masks (FULL, CHUNK, BAND,
// with per-sequence lengths, a causal flag and per-head sinks) on Blackwell.
//
// Same computation as flash_attn.cuh -- o_i = sum_{j in A_i} 2^(x_ij) v_j / l_i,
// x_ij = s_ij * scale * log2(e) - m_i, over the key interval A_i of each query
// row -- laid out for one CTA per SM:
//
//   warps 0-7   softmax. Warp w owns 16 rows of the 128-row query tile: tensor
//               memory lanes 32(w%4) + 16(w/4) ... +15 (a warp may only touch
//               its own lane quadrant, w%4). Scores are read with the 16x256b
//               shape, so each row lies in four consecutive threads and its
//               max and sum are two xor-shuffles; each thread holds 2 rows x
//               32 columns. The same warps write a unit's output one key tile
//               into the next unit (O is double-buffered), when its last P V
//               has long completed, reading O in the same layout, so a row's
//               sum is already in the threads that hold the row.
//   warp 8      TMA producer: Q per unit (double buffer), K and V tiles through
//               a 4-stage ring, in place from the packed projection buffer.
//   warp 9      tcgen05.mma issuer: S(t) = Q K(t)^T, then O += P(t-2) V(t-2).
// Ten warps keep three per SM sub-partition at most, so a thread may hold 168
// registers (an SMSP has 16K).
//
// Tensor memory (512 columns): S in two 128-column buffers, P in two 64-column
// buffers, O in two 64-column buffers. With S and P double-buffered the tensor
// core computes S(t+1) and P(t-1) V(t-1) while the softmax works on tile t;
// with O double-buffered the epilogue of one unit overlaps the next unit.
//
// Softmax per key tile. The exponent reference m_i lags the true running max:
// the first tile of a unit sets it to that tile's row max; later tiles compute
// their exponentials against the current reference straight away and keep the
// tile's row max on the side. Only if some row's max exceeds its reference by
// more than RESCALE_LIMIT (2^15 still fits fp16 P; never for data whose logits
// stay within 10 natural units of the first tile's) does the warp take the
// slow path: new references from the row max, the tile recomputed from
// registers, O and the partial sums rescaled. The common path therefore has no
// serial max phase before its exponentials.
//
// A compile-time share of the exponentials (POLY_REPS) runs on the FMA pipe
// (exp2_poly_x2) instead of MUFU ex2.
#pragma once

#include "flash_attn.cuh"
#include "sm100_ptx.cuh"

#ifndef SEA_POLY_REPS
#define SEA_POLY_REPS 0x0000u
#endif

namespace sea {
namespace fr {

using fa::BKV;
using fa::BQ;
using fa::DH;
using fa::Params;
using fa::SeqLen;
using fa::TILE_BYTES;
using fa::Unit;

// A reference may lag the row max by this much (log2 units): p <= 2^15 fits fp16.
constexpr float RESCALE_LIMIT = 15.0f;

// Bit j set: the 8-column repetition j (of 16) of every score tile takes the
// FMA-pipe exp2 instead of MUFU ex2.
constexpr uint32_t POLY_REPS = SEA_POLY_REPS;

// K/V ring depth (each stage one 16 KB K tile and one 16 KB V tile).
#ifndef SEA_KV_STAGES
#define SEA_KV_STAGES 4
#endif

// How many key tiles behind S the P V products are issued (1 or 2).
#ifndef SEA_PV_LAG
#define SEA_PV_LAG 2
#endif
constexpr int PV_LAG = SEA_PV_LAG;

struct Cfg {
  static constexpr int SOFTMAX_WARPS = 8;
  static constexpr int PRODUCER_WARP = 8;
  static constexpr int MMA_WARP = 9;
  static constexpr int THREADS = 320;
  static constexpr int STAGES = SEA_KV_STAGES;  // K/V ring depth
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t S_COL = 0;    // S buffer b at S_COL + 128 b
  static constexpr uint32_t P_COL = 256;  // P buffer b at P_COL + 64 b
  static constexpr uint32_t O_COL = 384;  // O buffer b at O_COL + 64 b
  static constexpr int OFF_Q = 0;         // two Q buffers
  static constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
  static constexpr int OFF_BARS = OFF_V + STAGES * TILE_BYTES;
  // q_full[2], q_empty[2], k_full[S], v_full[S], kv_empty[S], s_full[2], s_free[2],
  // p_full[2], pv_done[2], o_full[2], o_free[2], drain
  static constexpr int NUM_BARS = 4 + 3 * STAGES + 12 + 1;
  static constexpr int OFF_MISC = OFF_BARS + 8 * NUM_BARS;
  static constexpr int SMEM_BYTES = 1024 + OFF_MISC + 16;
};

// One thread's share of a 16-row slice of a score tile in the 16x256b layout
// (fp32 bit patterns): r[4j + 2h + e] is row (h ? r1 : r0), column
// 8j + 2(lane%4) + e.
struct Slice {
  uint32_t r[64];
  __device__ __forceinline__ float v(int i) const { return __uint_as_float(r[i]); }
};

// Exponentials of one score tile slice against references m_use[h] (log2
// units): P written to tensor memory as fp16 pairs (16x128b, four
// repetitions per store), row sums of this slice returned in sum[h].
__device__ __forceinline__ void exp_tile(const Slice& s, float sl2, const float (&m_use)[2], uint32_t p_addr,
                                         float (&sum)[2]) {
  const uint64_t sl2x2 = f2_pack(sl2, sl2);
  const uint64_t negm[2] = {f2_pack(-m_use[0], -m_use[0]), f2_pack(-m_use[1], -m_use[1])};
  uint64_t acc[2][2] = {{0ull, 0ull}, {0ull, 0ull}};
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    uint32_t pk[8];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int j = 4 * g + jj;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float x0, x1, p0, p1;
        f2_unpack(f2_fma(f2_pack(s.v(4 * j + 2 * h), s.v(4 * j + 2 * h + 1)), sl2x2, negm[h]), x0, x1);
        if ((POLY_REPS >> j) & 1u) {
          exp2_poly_x2(x0, x1, p0, p1);
        } else {
          p0 = ex2_approx(x0);
          p1 = ex2_approx(x1);
        }
        acc[h][j & 1] = f2_add(acc[h][j & 1], f2_pack(p0, p1));
        pk[2 * jj + h] = pack_half2(p0, p1);
      }
    }
    tmem_st16x128b_x4(p_addr + 16 * g, pk);
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float a0, a1;
    f2_unpack(f2_add(acc[h][0], acc[h][1]), a0, a1);
    sum[h] = a0 + a1;
  }
}

// Per-thread max of each of the two rows' 32 values.
__device__ __forceinline__ void slice_max(const Slice& s, float (&mx)[2]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float a = s.v(2 * h), b = s.v(2 * h + 1);
#pragma unroll
    for (int j = 1; j < 16; j += 2) {
      a = fmax3(a, s.v(4 * j + 2 * h), s.v(4 * j + 2 * h + 1));
      if (j + 1 < 16) b = fmax3(b, s.v(4 * (j + 1) + 2 * h), s.v(4 * (j + 1) + 2 * h + 1));
    }
    mx[h] = fmaxf(a, b);
  }
}

__device__ __forceinline__ float quad_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
}

__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v + __shfl_xor_sync(0xffffffffu, v, 2);
}

template <bool EXT>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    flash_range_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = Cfg;
  constexpr int ST = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::OFF_BARS;
  auto q_full = [&](int i) { return bar0 + 8u * i; };
  auto q_empty = [&](int i) { return bar0 + 8u * (2 + i); };
  auto k_full = [&](int s) { return bar0 + 8u * (4 + s); };
  auto v_full = [&](int s) { return bar0 + 8u * (4 + ST + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (4 + 2 * ST + s); };
  const uint32_t bar1 = bar0 + 8u * (4 + 3 * ST);
  auto s_full = [&](int b) { return bar1 + 8u * b; };
  auto s_free = [&](int b) { return bar1 + 8u * (2 + b); };
  auto p_full = [&](int b) { return bar1 + 8u * (4 + b); };
  auto pv_done = [&](int b) { return bar1 + 8u * (6 + b); };
  auto o_full = [&](int b) { return bar1 + 8u * (8 + b); };
  auto o_free = [&](int b) { return bar1 + 8u * (10 + b); };
  const uint32_t drain_bar = bar1 + 8u * 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full(i), 1);
      mbar_init(q_empty(i), 1);
      mbar_init(s_full(i), 1);
      mbar_init(s_free(i), C::SOFTMAX_WARPS);
      mbar_init(p_full(i), C::SOFTMAX_WARPS);
      mbar_init(pv_done(i), 1);
      mbar_init(o_full(i), 1);
      mbar_init(o_free(i), C::SOFTMAX_WARPS);
    }
    for (int s = 0; s < ST; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0u;
    fence_barrier_init();
    // The tensor maps are launch parameters, not the previous kernel's data:
    // fetch them before waiting for that kernel.
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
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

  // Units every role skips: no query row, or (range masks) no key tile. The
  // softmax warps write such a unit's rows directly; no barrier is touched.
  auto has_tiles = [](const Unit& U) { return U.rows > 0 && U.j_end > U.j_begin; };

  if (warp == C::PRODUCER_WARP) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int nu = 0, it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        const Unit U = fa::decode_unit<EXT>(p, u);
        if (!has_tiles(U)) continue;
        const int qb = nu & 1;
        if (!mbar_wait(q_empty(qb), ((nu >> 1) & 1) ^ 1u, wc)) break;
        mbar_arrive_expect_tx(q_full(qb), TILE_BYTES);
        tma_load_3d(sbase + C::OFF_Q + qb * TILE_BYTES, &tm_q, q_full(qb), U.h * DH, U.q0, U.b);
        ++nu;
        for (int j = U.j_begin; j < U.j_end; ++j, ++it) {
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
        }
      }
      // Let the last copies land before the CTA may exit.
      if (nu > 0) mbar_wait_drain(q_full((nu - 1) & 1), ((nu - 1) >> 1) & 1, p.limit_ns);
      for (int i = max(0, it - ST); i < it; ++i) {
        mbar_wait_drain(k_full(i % ST), (i / ST) & 1, p.limit_ns);
        mbar_wait_drain(v_full(i % ST), (i / ST) & 1, p.limit_ns);
      }
    }
  } else if (warp == C::MMA_WARP) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc_s = idesc_f16_f32(BQ, BKV, 0, 0);  // Q, K both K-major
      constexpr uint32_t idesc_o = idesc_f16_f32(BQ, DH, 0, 1);   // P K-major (TMEM), V MN-major
      const uint64_t q_desc0 = smem_desc_sw128(sbase + C::OFF_Q, 16, 1024);
      const uint64_t k_desc0 = smem_desc_sw128(sbase + C::OFF_K, 16, 1024);
      const uint64_t v_desc0 = smem_desc_sw128(sbase + C::OFF_V, TILE_BYTES, 1024);
      constexpr uint64_t kTileUnits = TILE_BYTES >> 4;
      struct Pending {
        int t, nu;
        bool first, last, valid;
      };
      Pending pend{0, 0, false, false, false};
      // O(nu) += P(t) V(t); the first PV of a unit overwrites O.
      auto issue_pv = [&](const Pending& pd) -> bool {
        const int st = pd.t % ST;
        if (!mbar_wait(v_full(st), (pd.t / ST) & 1, wc)) return false;
        if (pd.first && !mbar_wait(o_free(pd.nu & 1), ((pd.nu >> 1) & 1) ^ 1u, wc)) return false;
        if (!mbar_wait(p_full(pd.t & 1), (pd.t >> 1) & 1, wc)) return false;
        tc_fence_after();
        const uint64_t vd = v_desc0 + st * kTileUnits;
        const uint32_t o_t = tmem_base + C::O_COL + 64u * (pd.nu & 1);
        const uint32_t p_t = tmem_base + C::P_COL + 64u * (pd.t & 1);
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk)
          mma_f16_ts(o_t, p_t + kk * 8, vd + kk * 128, idesc_o, (!pd.first || kk > 0) ? 1u : 0u);
        mma_commit(pv_done(pd.t & 1));
        mma_commit(kv_empty(st));
        if (pd.last) mma_commit(o_full(pd.nu & 1));
        return true;
      };
      // S(t) and P(t-2) V(t-2) become ready together (the softmax's end of
      // tile t-2 frees S buffer t%2 and fills P buffer t%2); S(t) goes first
      // so the scores the softmax prefetches next are not queued behind a PV.
      Pending pend2{0, 0, false, false, false};  // the older of two pending PVs
      int nu = 0, it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        const Unit U = fa::decode_unit<EXT>(p, u);
        if (!has_tiles(U)) continue;
        const int qb = nu & 1;
        if (!mbar_wait(q_full(qb), (nu >> 1) & 1, wc)) break;
        const uint64_t qd = q_desc0 + qb * kTileUnits;
        for (int j = U.j_begin; j < U.j_end; ++j, ++it) {
          const int st = it % ST;
          const int sb = it & 1;
          if (!mbar_wait(k_full(st), (it / ST) & 1, wc) || !mbar_wait(s_free(sb), ((it >> 1) & 1) ^ 1u, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t kd = k_desc0 + st * kTileUnits;
          const uint32_t s_t = tmem_base + C::S_COL + 128u * sb;
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) mma_f16_ss(s_t, qd + kk * 2, kd + kk * 2, idesc_s, kk > 0 ? 1u : 0u);
          mma_commit(s_full(sb));
          const Pending cur{it, nu, j == U.j_begin, j == U.j_end - 1, true};
          if constexpr (PV_LAG == 2) {
            if (pend2.valid && !issue_pv(pend2)) {
              ok = false;
              break;
            }
            pend2 = pend;
          } else {
            if (pend.valid && !issue_pv(pend)) {
              ok = false;
              break;
            }
          }
          pend = cur;
        }
        if (!ok) break;
        mma_commit(q_empty(qb));  // Q buffer free once this unit's S products finish
        ++nu;
      }
      if (ok && pend2.valid) ok = issue_pv(pend2);
      if (ok && pend.valid) issue_pv(pend);
      mma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0, p.limit_ns);
    }
  } else if (warp < C::SOFTMAX_WARPS) {
    // ---------------- softmax (and the deferred epilogue) ----------------
    const int qd = warp & 3;                        // lane quadrant
    const int L0 = 32 * qd + 16 * (warp >> 2);      // first row (tensor-memory lane) of this warp
    const int rr[2] = {L0 + (lane >> 2), L0 + (lane >> 2) + 8};
    const int cpair = 2 * (lane & 3);
    const uint32_t lane_field = static_cast<uint32_t>(L0) << 16;
    const float sl2 = p.scale_log2;
    // A unit whose output is still to be written: its O buffer, and this
    // thread's rows' references and sums.
    struct Done {
      int u, nu;  // work unit (decoded again when written) and its O buffer
      float m[2], l[2];
      bool valid;
    };
    Done done{};
    done.valid = false;
    // Writes a finished unit's rows of this warp: waits for its last P V,
    // reads O in the scores' layout (rows rr[h], columns 8j + cpair + e),
    // frees the buffer, divides by the row sums (or writes the unnormalised
    // split partial with m and l).
    auto epilogue = [&](const Done& d) -> bool {
      const int ob = d.nu & 1;
      if (!mbar_wait(o_full(ob), (d.nu >> 1) & 1, wc)) return false;
      tc_fence_after();
      uint32_t o[32];
      tmem_ld16x256b_x8(tmem_base + C::O_COL + 64u * ob + lane_field, o);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free(ob));
      const Unit U = fa::decode_unit<EXT>(p, d.u);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (rr[h] >= U.rows) continue;
        const int row_glob = U.q0 + rr[h];
        if (p.kv_splits > 1) {
          const int64_t part =
              ((static_cast<int64_t>(U.split) * p.batch + U.b) * p.n_heads + U.h) * p.t_q + row_glob;
          float* dst = p.ws_o + part * DH + cpair;
#pragma unroll
          for (int j8 = 0; j8 < 8; ++j8)
            *reinterpret_cast<float2*>(dst + 8 * j8) =
                make_float2(__uint_as_float(o[4 * j8 + 2 * h]), __uint_as_float(o[4 * j8 + 2 * h + 1]));
          if ((lane & 3) == 0) reinterpret_cast<float2*>(p.ws_ml)[part] = make_float2(d.m[h], d.l[h]);
        } else {
          float l = d.l[h];
          // A sink adds 2^(sink*log2e - m) to the normaliser. No visible key:
          // m = -inf and l = 0, so the output is 0.
          if constexpr (EXT) {
            if (p.sinks != nullptr && d.m[h] != -INFINITY)
              l += ex2_approx(__ldg(p.sinks + U.h) * fa::kLog2e - d.m[h]);
          }
          const float inv = l > 0.f ? 1.f / l : 0.f;
          uint32_t* dst = reinterpret_cast<uint32_t*>(p.out + (static_cast<int64_t>(U.b) * p.t_q + row_glob) *
                                                                   p.out_stride + U.h * DH + cpair);
#pragma unroll
          for (int j8 = 0; j8 < 8; ++j8)
            dst[4 * j8] = pack_half2(__uint_as_float(o[4 * j8 + 2 * h]) * inv,
                                     __uint_as_float(o[4 * j8 + 2 * h + 1]) * inv);
        }
      }
      return true;
    };
    int nu = 0, it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
      const Unit U = fa::decode_unit<EXT>(p, u);
      if (U.rows == 0) continue;
      if (!has_tiles(U)) {
        // No key tile: the rows see no key (zero output, or an empty partial).
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (rr[h] >= U.rows) continue;
          const int row_glob = U.q0 + rr[h];
          if (p.kv_splits > 1) {
            const int64_t part =
                ((static_cast<int64_t>(U.split) * p.batch + U.b) * p.n_heads + U.h) * p.t_q + row_glob;
            float* dst = p.ws_o + part * DH + cpair;
#pragma unroll
            for (int j8 = 0; j8 < 8; ++j8) *reinterpret_cast<float2*>(dst + 8 * j8) = make_float2(0.f, 0.f);
            if ((lane & 3) == 0) reinterpret_cast<float2*>(p.ws_ml)[part] = make_float2(-INFINITY, 0.f);
          } else {
            uint32_t* dst = reinterpret_cast<uint32_t*>(p.out + (static_cast<int64_t>(U.b) * p.t_q + row_glob) *
                                                                     p.out_stride + U.h * DH + cpair);
#pragma unroll
            for (int j8 = 0; j8 < 8; ++j8) dst[4 * j8] = 0u;
          }
        }
        continue;
      }
      const bool warp_active = L0 < U.rows;
      // key interval [lo, hi) of each of the thread's rows (sequence-local keys)
      int lo[2] = {0, 0}, hi[2] = {0, 0};
      {
        const SeqLen L = fa::seq_len<EXT>(p, U.b);
#pragma unroll
        for (int h = 0; h < 2; ++h)
          if (rr[h] < U.rows) fa::row_keys<EXT>(p, L, U.q0 + rr[h], lo[h], hi[h]);
      }
      float m_ref[2] = {-INFINITY, -INFINITY};  // exponent reference (log2 units)
      float l_part[2] = {0.f, 0.f};             // this thread's share of the row sums
      Slice s;
      for (int j = U.j_begin; j < U.j_end; ++j, ++it) {
        const int sb = it & 1;
        const bool first = j == U.j_begin;
        const uint32_t s_addr = tmem_base + C::S_COL + 128u * sb + lane_field;
        const uint32_t p_addr = tmem_base + C::P_COL + 64u * sb + lane_field;
        if (first) {
          if (!mbar_wait(s_full(sb), (it >> 1) & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          tmem_ld16x256b_x16(s_addr, s.r);
        }
        tmem_wait_ld64(s.r);
        if (warp_active) {
          const int kv0 = U.kv_lo + j * BKV;
          int a[2], bnd[2];
          bool need = false;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            a[h] = lo[h] - kv0;
            bnd[h] = hi[h] - kv0;
            need |= a[h] > 0 || bnd[h] < BKV;
          }
          if (__any_sync(0xffffffffu, need)) {
#pragma unroll
            for (int j8 = 0; j8 < 16; ++j8)
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const int col = 8 * j8 + cpair + e;
                  if (col < a[h] || col >= bnd[h]) s.r[4 * j8 + 2 * h + e] = 0xff800000u;  // -inf
                }
          }
          if (first) {
            float mx[2];
            slice_max(s, mx);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float rm = quad_max(mx[h]);
              m_ref[h] = rm == -INFINITY ? -INFINITY : rm * sl2;
            }
          }
          // P buffer sb was last read by the PV of tile it - 2.
          if (it >= 2 && !mbar_wait(pv_done(sb), ((it >> 1) & 1) ^ 1u, wc)) {
            ok = false;
            break;
          }
          float m_use[2], sum[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) m_use[h] = m_ref[h] == -INFINITY ? 0.f : m_ref[h];
          exp_tile(s, sl2, m_use, p_addr, sum);
          bool slow = false;
          float mx[2] = {-INFINITY, -INFINITY};
          if (!first) {
            slice_max(s, mx);
            const bool fail = mx[0] * sl2 > m_ref[0] + RESCALE_LIMIT || mx[1] * sl2 > m_ref[1] + RESCALE_LIMIT;
            slow = __any_sync(0xffffffffu, fail);
          }
          if (!slow) {
            l_part[0] += sum[0];
            l_part[1] += sum[1];
          } else {
            // Rare: a row's max outgrew its reference. New references from
            // the row maxima, the tile recomputed, O and the sums rescaled.
            float alpha[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float rm = quad_max(mx[h]) * sl2;
              if (rm > m_ref[h] + RESCALE_LIMIT) {
                alpha[h] = ex2_approx(m_ref[h] - rm);  // 0 while the reference was -inf
                m_ref[h] = rm;
              } else {
                alpha[h] = 1.f;
              }
              m_use[h] = m_ref[h] == -INFINITY ? 0.f : m_ref[h];
            }
            tmem_wait_st();
            exp_tile(s, sl2, m_use, p_addr, sum);
#pragma unroll
            for (int h = 0; h < 2; ++h) l_part[h] = l_part[h] * alpha[h] + sum[h];
            // O holds this unit's earlier tiles once the previous PV completes.
            if (!mbar_wait(pv_done((it - 1) & 1), ((it - 1) >> 1) & 1, wc)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t o_addr = tmem_base + C::O_COL + 64u * (nu & 1) + lane_field;
            uint32_t o[32];
            tmem_ld16x256b_x8(o_addr, o);
#pragma unroll
            for (int j8 = 0; j8 < 8; ++j8)
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int e = 0; e < 2; ++e)
                  o[4 * j8 + 2 * h + e] = __float_as_uint(__uint_as_float(o[4 * j8 + 2 * h + e]) * alpha[h]);
            tmem_st16x256b_x8(o_addr, o);
          }
        }
        // The previous unit's output, one tile into this one: its last P V has
        // had a tile's time to complete.
        if (first && done.valid) {
          if (!epilogue(done)) {
            ok = false;
            break;
          }
          done.valid = false;
        }
        // Prefetch the next tile's scores of this unit (S double-buffered).
        if (j + 1 < U.j_end) {
          if (!mbar_wait(s_full(sb ^ 1), ((it + 1) >> 1) & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          tmem_ld16x256b_x16(tmem_base + C::S_COL + 128u * (sb ^ 1) + lane_field, s.r);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        // p_full before s_free: once S(t+2) is issued (s_free complete), every
        // warp has arrived on p_full(t) too.
        if (lane == 0) {
          mbar_arrive(p_full(sb));
          mbar_arrive(s_free(sb));
        }
      }
      if (!ok) break;
      // Row sums (four threads per row) and references for the epilogue.
      done = Done{u, nu, {m_ref[0], m_ref[1]}, {quad_sum(l_part[0]), quad_sum(l_part[1])}, true};
      ++nu;
    }
    if (ok && done.valid) epilogue(done);
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace fr
}  // namespace sea
