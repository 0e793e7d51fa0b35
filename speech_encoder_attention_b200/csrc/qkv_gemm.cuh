// qkv_gemm.cuh -- the packed QKV projection on Blackwell tensor cores.
//
//   qkv[r, j] = sum_c x[r, c] * W[j, c] + bias[j],   bias = [b_q | 0 | b_v]
//
// The edda PR ("Add Edda ASR with DFlash2 speculative decoding", PR
// description) packs the three projections into one; this is that single GEMM
// with the q/v bias folded into its epilogue (Whisper's key projection has no
// bias).
//
// Design (one persistent CTA per SM, 192 threads):
//   warp 0      TMA producer: x and W tiles (64-wide K slices, 128-byte swizzle)
//               into a 4-stage shared-memory ring.
//   warp 1      tcgen05.mma issuer (one thread): 128xBNx16 f16 MMAs (BN = 256 or
//               192) into one of two fp32 accumulators in tensor memory, so the
//               epilogue of tile i overlaps the main loop of tile i+1.
//   warps 2..5  epilogue: tcgen05.ld 32 columns at a time, add the bias in fp32,
//               round to fp16, stage a 32x32 box per warp in swizzled shared
//               memory and write it with a TMA store.
// Both operands are K-major (x rows and W rows are contiguous along d_model).
#pragma once

#include "sm100_ptx.cuh"

namespace sea {
namespace gemm {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int EPI_COLS = 32;
constexpr int A_BYTES = BM * BK * 2;
constexpr int EPI_BUF_BYTES = 32 * EPI_COLS * 2;  // one 32-row x 32-col fp16 box
constexpr int EPI_BYTES = 4 * 2 * EPI_BUF_BYTES;  // 4 warps, double buffered
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 512;  // two accumulators of up to 256 fp32 columns

// Output tile width and pipeline depth. 128x256 tiles with a 4-stage ring
// suit large row counts; 128x192 tiles (5 stages in the same shared memory)
// are ~11 % less efficient per flop but cut the idle part of the last wave
// when the tile count is small (the host picks by estimated waves).
template <int BN_, int STAGES_>
struct Shape {
  static constexpr int BN = BN_;
  static constexpr int STAGES = STAGES_;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int OFF_STAGES = 0;
  static constexpr int OFF_EPI = OFF_STAGES + STAGES * STAGE_BYTES;
  static constexpr int OFF_BARS = OFF_EPI + EPI_BYTES;
  // barriers: full[STAGES], empty[STAGES], tfull[2], tempty[2], drain
  static constexpr int NUM_BARS = 2 * STAGES + 5;
  static constexpr int OFF_MISC = OFF_BARS + 8 * NUM_BARS;  // tmem base, abort flag
  static constexpr int SMEM_BYTES = 1024 + OFF_MISC + 16;   // + slack to align the base to 1 KB
};
using WideTiles = Shape<256, 4>;
using NarrowTiles = Shape<192, 5>;

struct Args {
  const __half* b_q;
  const __half* b_v;
  int m, n, k, d_model;
  uint32_t* err;
  uint64_t limit_ns;
};

__device__ __forceinline__ void load_bias32(const Args& a, int n_c, float (&bias)[32]) {
  const __half* src = nullptr;
  const int region = n_c / a.d_model;
  if (region == 0)
    src = a.b_q ? a.b_q + n_c : nullptr;
  else if (region == 2)
    src = a.b_v ? a.b_v + (n_c - 2 * a.d_model) : nullptr;
  if (src == nullptr) {
#pragma unroll
    for (int i = 0; i < 32; ++i) bias[i] = 0.f;
    return;
  }
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    uint4 u = __ldg(s4 + v);
    const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __half22float2(h[i]);
      bias[8 * v + 2 * i] = f.x;
      bias[8 * v + 2 * i + 1] = f.y;
    }
  }
}

template <class S>
__global__ void __launch_bounds__(THREADS, 1)
    qkv_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                    const __grid_constant__ CUtensorMap tm_out, const Args args) {
  constexpr int BN = S::BN;
  constexpr int STAGES = S::STAGES;
  constexpr int STAGE_BYTES = S::STAGE_BYTES;
  constexpr int OFF_STAGES = S::OFF_STAGES;
  constexpr int OFF_EPI = S::OFF_EPI;
  constexpr int OFF_BARS = S::OFF_BARS;
  constexpr int OFF_MISC = S::OFF_MISC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + OFF_BARS;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tiles_m = (args.m + BM - 1) / BM;
  const int tiles_n = (args.n + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int kblocks = (args.k + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 4);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0u;
    fence_barrier_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_out);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Everything above touched only this CTA's shared and tensor memory.
  griddep_wait();
  griddep_launch_dependents();
  const WaitCtl wc{abort_flag, args.err, args.limit_ns};

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        const int m0 = (tile / tiles_n) * BM;
        const int n0 = (tile % tiles_n) * BN;
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, wc)) {
            ok = false;
            break;
          }
          const uint32_t sa = sbase + OFF_STAGES + stage * STAGE_BYTES;
          mbar_arrive_expect_tx(full_bar(stage), STAGE_BYTES);
          tma_load_2d(sa, &tm_x, full_bar(stage), kb * BK, m0);
          tma_load_2d(sa + A_BYTES, &tm_w, full_bar(stage), kb * BK, n0);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      // Let the last copies land before the CTA can exit (they are already
      // complete on the normal path).
      for (int i = 0; i < STAGES && i < issued; ++i) {
        if (--stage < 0) {
          stage = STAGES - 1;
          phase ^= 1u;
        }
        mbar_wait_drain(full_bar(stage), phase, args.limit_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = idesc_f16_f32(BM, BN, 0, 0);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, wc)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = sbase + OFF_STAGES + stage * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(sb + kk * 32, 16, 1024);
            mma_f16_ss(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          mma_commit(empty_bar(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) mma_commit(tfull_bar(acc));
      }
      // Every MMA issued above has finished once this arrives.
      mma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0, args.limit_ns);
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int quad = warp & 3;  // tensor-memory lane quadrant this warp may access
    const uint32_t lane_field = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t ebuf = sbase + OFF_EPI + (warp - 2) * 2 * EPI_BUF_BYTES;
    uint32_t chunk_count = 0;
    int local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!mbar_wait(tfull_bar(acc), acc_phase, wc)) break;
      tc_fence_after();
      const int m0 = (tile / tiles_n) * BM;
      const int n0 = (tile % tiles_n) * BN;
      const int row0 = m0 + quad * 32;
#pragma unroll 1
      for (int c = 0; c < BN / EPI_COLS; ++c) {
        const int n_c = n0 + c * EPI_COLS;
        if (n_c >= args.n) break;
        uint32_t r[32];
        tmem_ld32(tmem_base + acc * BN + c * EPI_COLS + lane_field, r);
        float bias[32];
        load_bias32(args, n_c, bias);
        uint32_t h[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          h[i] = pack_half2(__uint_as_float(r[2 * i]) + bias[2 * i],
                            __uint_as_float(r[2 * i + 1]) + bias[2 * i + 1]);
        const uint32_t buf = ebuf + (chunk_count & 1u) * EPI_BUF_BYTES;
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
        // Row `lane` of the 32x32 box, 64 bytes, in the 64-byte swizzle TMA expects.
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint32_t addr = buf + lane * 64 + ((v ^ ((lane >> 1) & 3)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(h[4 * v]),
                       "r"(h[4 * v + 1]), "r"(h[4 * v + 2]), "r"(h[4 * v + 3])
                       : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < args.m) {
          tma_store_2d(&tm_out, buf, n_c, row0);
          bulk_commit_group();
        }
        ++chunk_count;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
    }
    if (lane == 0) bulk_wait_group_all();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace gemm
}  // namespace sea

namespace sea {
namespace gemm {

// ---------------------------------------------------------------------------
// CTA-pair variant: 256 x 256 output tiles computed by two SMs with
// cta_group::2 MMAs (M = 256, N = 256, K = 16). CTA r of the pair owns tile
// rows [128 r, 128 r + 128): it loads its 128 rows of x and its 128 rows of W
// (the MMA splits B along N between the pair), holds its rows' accumulator in
// its own tensor memory and writes them. Per SM this reads half the operand
// bytes per flop of the 128 x 256 single-CTA tile. Roles as in
// qkv_gemm_kernel; the pair leader's thread issues the MMAs, whose
// completions are signalled to both CTAs' barriers; the peer's epilogue
// releases an accumulator by arriving on the leader's barrier. No TMA load
// is multicast: each CTA loads only its own halves.
// ---------------------------------------------------------------------------
struct PairShape {
  static constexpr int BN = 256;  // tile columns (the pair's N)
  static constexpr int STAGES = 6;
  static constexpr int HALF_BYTES = 128 * BK * 2;  // one CTA's 128 rows of a 64-wide K slice
  static constexpr int STAGE_BYTES = 2 * HALF_BYTES;  // its x half + its W half
  static constexpr int OFF_STAGES = 0;
  static constexpr int OFF_EPI = OFF_STAGES + STAGES * STAGE_BYTES;
  static constexpr int OFF_BARS = OFF_EPI + EPI_BYTES;
  // barriers: full[STAGES], empty[STAGES], tfull[2], tempty[2], drain
  static constexpr int NUM_BARS = 2 * STAGES + 5;
  static constexpr int OFF_MISC = OFF_BARS + 8 * NUM_BARS;
  static constexpr int SMEM_BYTES = 1024 + OFF_MISC + 16;
};

__global__ void __launch_bounds__(THREADS, 1)
    qkv_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                         const __grid_constant__ CUtensorMap tm_out, const Args args) {
  using S = PairShape;
  constexpr int BN = S::BN;
  constexpr int STAGES = S::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + S::OFF_BARS;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + S::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: pair leader
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;
  const int tiles_m = (args.m + 2 * BM - 1) / (2 * BM);
  const int tiles_n = (args.n + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int kblocks = (args.k + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 8);  // the leader's: four epilogue warps of each CTA
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0u;
    fence_barrier_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_out);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before either signals the other's
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();
  griddep_launch_dependents();
  const WaitCtl wc{abort_flag, args.err, args.limit_ns};

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int tile = pair; tile < num_tiles; tile += num_pairs) {
        const int m0 = (tile / tiles_n) * 2 * BM + static_cast<int>(rank) * BM;
        const int n0 = (tile % tiles_n) * BN + static_cast<int>(rank) * (BN / 2);
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, wc)) {
            ok = false;
            break;
          }
          const uint32_t sa = sbase + S::OFF_STAGES + stage * S::STAGE_BYTES;
          const uint32_t leader_full = mapa_shared(full_bar(stage), 0);
          if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 2 * S::STAGE_BYTES);
          tma_load_2d_pair(sa, &tm_x, leader_full, kb * BK, m0);
          tma_load_2d_pair(sa + S::HALF_BYTES, &tm_w, leader_full, kb * BK, n0);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      // Let this CTA's last copies land before it can exit: once the leader's
      // MMAs that read a stage completed, its bytes had arrived.
      for (int i = 0; i < STAGES && i < issued; ++i) {
        if (--stage < 0) {
          stage = STAGES - 1;
          phase ^= 1u;
        }
        mbar_wait_drain(empty_bar(stage), phase, args.limit_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (pair leader) ----------------
      constexpr uint32_t idesc = idesc_f16_f32(2 * BM, BN, 0, 0);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs, ++local) {
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait_cluster(tempty_bar(acc), acc_phase ^ 1u, wc)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = sbase + S::OFF_STAGES + stage * S::STAGE_BYTES;
          const uint32_t sb = sa + S::HALF_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(sb + kk * 32, 16, 1024);
            mma_f16_ss_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          mma_commit_pair(empty_bar(stage), 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) mma_commit_pair(tfull_bar(acc), 0x3);
      }
      mma_commit_pair(drain_bar, 0x1);
      mbar_wait_drain(drain_bar, 0, args.limit_ns);
    }
  } else {
    // ---------------- epilogue (warps 2..5, both CTAs) ----------------
    const int quad = warp & 3;
    const uint32_t lane_field = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t ebuf = sbase + S::OFF_EPI + (warp - 2) * 2 * EPI_BUF_BYTES;
    uint32_t chunk_count = 0;
    int local = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!mbar_wait_cluster(tfull_bar(acc), acc_phase, wc)) break;
      tc_fence_after();
      const int m0 = (tile / tiles_n) * 2 * BM + static_cast<int>(rank) * BM;
      const int n0 = (tile % tiles_n) * BN;
      const int row0 = m0 + quad * 32;
#pragma unroll 1
      for (int c = 0; c < BN / EPI_COLS; ++c) {
        const int n_c = n0 + c * EPI_COLS;
        if (n_c >= args.n) break;
        uint32_t r[32];
        tmem_ld32(tmem_base + acc * BN + c * EPI_COLS + lane_field, r);
        float bias[32];
        load_bias32(args, n_c, bias);
        uint32_t h[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          h[i] = pack_half2(__uint_as_float(r[2 * i]) + bias[2 * i], __uint_as_float(r[2 * i + 1]) + bias[2 * i + 1]);
        const uint32_t buf = ebuf + (chunk_count & 1u) * EPI_BUF_BYTES;
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint32_t addr = buf + lane * 64 + ((v ^ ((lane >> 1) & 3)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(h[4 * v]), "r"(h[4 * v + 1]),
                       "r"(h[4 * v + 2]), "r"(h[4 * v + 3])
                       : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < args.m) {
          tma_store_2d(&tm_out, buf, n_c, row0);
          bulk_commit_group();
        }
        ++chunk_count;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive(tempty_bar(acc));
        else
          mbar_arrive_remote(mapa_shared(tempty_bar(acc), 0));
      }
    }
    if (lane == 0) bulk_wait_group_all();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA frees tensor memory the pair's MMAs may still use
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace gemm
}  // namespace sea
