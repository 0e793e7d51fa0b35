// qkv_q8.cuh -- the packed QKV projection with Q8_0 weights (decoder path).
//
//   qkv[r, j] = sum_c x[r, c] * W[j, c] + bias[j],   bias = [b_q | 0 | b_v],
//   W[j, 32b + t] = d[j, b] * q[j, b, t]
//
// The edda PR ("Add Edda ASR with DFlash2 speculative decoding", results
// table) runs its decoder with Q8_0 weights. A Q8_0 weight row is a run of
// 34-byte blocks: a little-endian fp16 scale d, then 32 signed bytes q.
//
// Shapes: the decoder projects a few hundred rows at most (the verify block
// is 5 beams x 16 rows), so the kernel is bound by reading the weights once.
// One CTA per (128-row tile, 32 output columns): 3 * d_model / 32 CTAs cover
// the SMs even for a single row tile.
//
// Design (192 threads per CTA):
//   warp 0      TMA producer: the 32 weight rows' 8 blocks per K step of 256
//               weights (272 raw bytes each) into a 6-stage ring whose first
//               loads all start at once (a CTA reads each weight byte once,
//               from HBM, so their latency is paid once rather than per K
//               step), and per K step x as four 64-column slices (128-byte
//               swizzle) into a 2-stage ring.
//   warp 1      tcgen05.mma issuer (one thread): 128x32x16 f16 MMAs into 32
//               fp32 tensor-memory columns.
//   warps 2..5  dequantize each stage's raw blocks into an fp16 operand tile in
//               the MMA's 128-byte-swizzled K-major layout (thread: one weight
//               row, 64 weights), then the epilogue: add the bias in fp32,
//               round to fp16, store.
#pragma once

#include "sm100_ptx.cuh"

namespace sea {
namespace q8 {

constexpr int BM = 128;
constexpr int BN = 32;
constexpr int BKQ = 256;                  // weights per K step (8 Q8_0 blocks)
constexpr int QBLOCK = 32;                // weights per Q8_0 block
constexpr int QBLOCK_BYTES = 34;          // fp16 scale + 32 int8
constexpr int RAW_ROW_BYTES = (BKQ / QBLOCK) * QBLOCK_BYTES;  // 272
constexpr int STAGES = 2;                 // x and dequantized-operand ring
constexpr int WSTAGES = 6;                // raw weight-block ring
constexpr int A_BYTES = BM * BKQ * 2;     // 64 KB: four 128x64 fp16 slices
constexpr int A_SLICE = BM * 64 * 2;      // 16 KB
constexpr int RAW_BYTES = BN * RAW_ROW_BYTES;  // 8704
constexpr int RAW_PAD = 9216;
constexpr int B_BYTES = BN * BKQ * 2;     // 16 KB: four 32x64 fp16 slices
constexpr int B_SLICE = BN * 64 * 2;      // 4 KB
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 32;

constexpr int OFF_A = 0;                              // [STAGES] x tiles
constexpr int OFF_B = OFF_A + STAGES * A_BYTES;       // [STAGES] dequantized W operands
constexpr int OFF_RAW = OFF_B + STAGES * B_BYTES;     // [WSTAGES] raw weight blocks
constexpr int OFF_BARS = OFF_RAW + WSTAGES * RAW_PAD;
// a_full[S], b_ready[S], ab_empty[S], raw_full[W], raw_empty[W], acc_full, drain
constexpr int NUM_BARS = 3 * STAGES + 2 * WSTAGES + 2;
constexpr int OFF_MISC = OFF_BARS + 8 * NUM_BARS;
constexpr int SMEM_BYTES = 1024 + OFF_MISC + 16;

struct Args {
  const __half* b_q;
  const __half* b_v;
  __half* out;
  int64_t out_stride;
  int m, d_model;
  uint32_t* err;
  uint64_t limit_ns;
};

__global__ void __launch_bounds__(THREADS, 1)
    qkv_q8_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                  const Args args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + OFF_BARS;
  auto a_full = [&](int s) { return bar0 + 8u * s; };
  auto b_ready = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto ab_empty = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };  // MMA done with x and B of stage s
  auto raw_full = [&](int w) { return bar0 + 8u * (3 * STAGES + w); };
  auto raw_empty = [&](int w) { return bar0 + 8u * (3 * STAGES + WSTAGES + w); };
  const uint32_t acc_full = bar0 + 8u * (3 * STAGES + 2 * WSTAGES);
  const uint32_t drain_bar = acc_full + 8u;
  auto stage_a = [&](int s) { return sbase + OFF_A + s * A_BYTES; };
  auto stage_b = [&](int s) { return sbase + OFF_B + s * B_BYTES; };
  auto stage_raw = [&](int w) { return sbase + OFF_RAW + w * RAW_PAD; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * BM;
  const int n0 = blockIdx.y * BN;
  const int ksteps = args.d_model / BKQ;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(a_full(s), 1);
      mbar_init(b_ready(s), 4);
      mbar_init(ab_empty(s), 1);
    }
    for (int w = 0; w < WSTAGES; ++w) {
      mbar_init(raw_full(w), 1);
      mbar_init(raw_empty(w), 4);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0u;
    fence_barrier_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
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
      // Raw blocks of K step kb into slot kb % WSTAGES once the dequantization
      // of step kb - WSTAGES has read it (the raw map counts 2-byte units:
      // 136 per 8 blocks).
      int issued_w = 0, issued = 0;
      auto load_w = [&](int kb) -> bool {
        const int w = kb % WSTAGES;
        if (kb >= WSTAGES && !mbar_wait(raw_empty(w), ((kb / WSTAGES) - 1) & 1, wc)) return false;
        mbar_arrive_expect_tx(raw_full(w), RAW_BYTES);
        tma_load_2d(stage_raw(w), &tm_w, raw_full(w), kb * (RAW_ROW_BYTES / 2), n0);
        ++issued_w;
        return true;
      };
      bool ok = true;
      for (int kb = 0; kb < min(ksteps, WSTAGES) && ok; ++kb) ok = load_w(kb);
      for (int kb = 0; kb < ksteps && ok; ++kb) {
        const int s = kb % STAGES;
        if (!mbar_wait(ab_empty(s), ((kb / STAGES) & 1) ^ 1u, wc)) break;
        mbar_arrive_expect_tx(a_full(s), A_BYTES);
#pragma unroll
        for (int a = 0; a < BKQ / 64; ++a)
          tma_load_2d(stage_a(s) + a * A_SLICE, &tm_x, a_full(s), kb * BKQ + a * 64, m0);
        ++issued;
        if (kb + WSTAGES < ksteps) ok = load_w(kb + WSTAGES);
      }
      // Let the last copies land before the CTA may exit.
      for (int i = max(0, issued - STAGES); i < issued; ++i)
        mbar_wait_drain(a_full(i % STAGES), (i / STAGES) & 1, args.limit_ns);
      for (int i = max(0, issued_w - WSTAGES); i < issued_w; ++i)
        mbar_wait_drain(raw_full(i % WSTAGES), (i / WSTAGES) & 1, args.limit_ns);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = idesc_f16_f32(BM, BN, 0, 0);  // x and W both K-major
      bool ok = true;
      for (int kb = 0; kb < ksteps; ++kb) {
        const int s = kb % STAGES;
        const uint32_t par = (kb / STAGES) & 1;
        if (!mbar_wait(a_full(s), par, wc) || !mbar_wait(b_ready(s), par, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BKQ / 16; ++kk) {
          const int slice = kk >> 2, within = kk & 3;
          const uint64_t ad = smem_desc_sw128(stage_a(s) + slice * A_SLICE + within * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(stage_b(s) + slice * B_SLICE + within * 32, 16, 1024);
          mma_f16_ss(tmem_base, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        mma_commit(ab_empty(s));
      }
      if (ok) mma_commit(acc_full);
      mma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0, args.limit_ns);
    }
  } else {
    // ---------------- dequantize, then epilogue ----------------
    const int t = threadIdx.x - 64;  // 0..127
    const int r = t >> 2;            // weight row within the 32-row tile
    const int qq = t & 3;            // 64-weight quarter of the K step == operand slice
    bool ok = true;
    for (int kb = 0; kb < ksteps; ++kb) {
      const int s = kb % STAGES, w = kb % WSTAGES;
      if (!mbar_wait(raw_full(w), (kb / WSTAGES) & 1, wc)) {
        ok = false;
        break;
      }
      // this thread's two blocks: 34-byte records, so 2-byte loads (plain C++
      // loads, ordered after the barrier wait, which the compiler may batch)
      const uint16_t* raw16 = reinterpret_cast<const uint16_t*>(
          smem + (stage_raw(w) - sbase) + r * RAW_ROW_BYTES + 2 * qq * QBLOCK_BYTES);
      const uint32_t dst_row = stage_b(s) + qq * B_SLICE + r * 128;
      uint16_t words[2][17];
#pragma unroll
      for (int bb = 0; bb < 2; ++bb)
#pragma unroll
        for (int i = 0; i < 17; ++i) words[bb][i] = raw16[bb * (QBLOCK_BYTES / 2) + i];
      // the raw slot may be refilled once every warp has read it; the operand
      // stage once the MMAs of step kb - STAGES are done
      __syncwarp();
      if (lane == 0) mbar_arrive(raw_empty(w));
      if (kb >= STAGES && !mbar_wait(ab_empty(s), ((kb / STAGES) - 1) & 1, wc)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int bb = 0; bb < 2; ++bb) {
        const float d = __half2float(__ushort_as_half(words[bb][0]));
        uint32_t h[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint16_t u = words[bb][1 + i];
          const float lo = static_cast<float>(static_cast<int8_t>(u & 0xFF)) * d;
          const float hi = static_cast<float>(static_cast<int8_t>(u >> 8)) * d;
          h[i] = pack_half2(lo, hi);
        }
        // 32 weights = four 16-byte chunks of the 128-byte row, 128-byte swizzle
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int ch = 4 * bb + c;
          const uint32_t addr = dst_row + ((ch ^ (r & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(h[4 * c]), "r"(h[4 * c + 1]),
                       "r"(h[4 * c + 2]), "r"(h[4 * c + 3])
                       : "memory");
        }
      }
      fence_proxy_async_smem();  // generic-proxy stores -> visible to the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(b_ready(s));
    }
    if (ok && mbar_wait(acc_full, 0, wc)) {
      tc_fence_after();
      const int row = (warp & 3) * 32 + lane;  // tensor-memory lane == output row in the tile
      uint32_t v[32];
      tmem_ld32(tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16), v);
      const int gr = m0 + row;
      if (gr < args.m) {
        const int region = n0 / args.d_model;  // 0: q, 1: k (no bias), 2: v
        const __half* bias = region == 0   ? (args.b_q ? args.b_q + n0 : nullptr)
                             : region == 2 ? (args.b_v ? args.b_v + (n0 - 2 * args.d_model) : nullptr)
                                           : nullptr;
        uint4* dst = reinterpret_cast<uint4*>(args.out + static_cast<int64_t>(gr) * args.out_stride + n0);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float b[8];
          if (bias != nullptr) {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(bias) + c);
            const __half2* hb = reinterpret_cast<const __half2*>(&u);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 f = __half22float2(hb[i]);
              b[2 * i] = f.x;
              b[2 * i + 1] = f.y;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) b[i] = 0.f;
          }
          uint4 o;
          o.x = pack_half2(__uint_as_float(v[8 * c + 0]) + b[0], __uint_as_float(v[8 * c + 1]) + b[1]);
          o.y = pack_half2(__uint_as_float(v[8 * c + 2]) + b[2], __uint_as_float(v[8 * c + 3]) + b[3]);
          o.z = pack_half2(__uint_as_float(v[8 * c + 4]) + b[4], __uint_as_float(v[8 * c + 5]) + b[5]);
          o.w = pack_half2(__uint_as_float(v[8 * c + 6]) + b[6], __uint_as_float(v[8 * c + 7]) + b[7]);
          dst[c] = o;
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace q8
}  // namespace sea
