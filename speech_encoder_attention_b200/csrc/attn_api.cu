// attn_api.cu -- the C ABI of libattn.so (declared in include/attn.h).
//
// Host side of the library: argument validation, the launch plan (query-tile
// schedule, key/value split), TMA tensor-map encoding and kernel launches.
// Everything is enqueued on the caller's stream; nothing here allocates device
// memory or synchronises (except the two debug entry points, which say so).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn.h"
#include "flash_attn.cuh"
#include "qkv_gemm.cuh"
#include "qkv_q8.cuh"
#include "sm100_ptx.cuh"

namespace {

// Device-side error word: kernels OR kErrTimeout into it when a bounded wait
// gives up. One copy per device.
__device__ uint32_t g_error_word = 0;

// Waits on a barrier nothing will complete, so the bounded-wait path can be
// tested without hanging or faulting the GPU.
__global__ void timeout_probe_kernel(uint32_t* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    sea::mbar_init(sea::smem_u32(&bar), 1);
    abort_flag = 0u;
    sea::fence_barrier_init();
  }
  __syncthreads();
  const sea::WaitCtl wc{&abort_flag, err, limit_ns};
  sea::mbar_wait(sea::smem_u32(&bar), 0, wc);
}

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ok = false;       // sm_100 device, attributes set
  int num_sms = 0;
  uint32_t* err = nullptr;  // address of g_error_word on this device
};

std::mutex g_mutex;
DeviceInfo g_dev[kMaxDevices];
bool g_dev_init[kMaxDevices] = {};

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// Raises the dynamic shared-memory limit of the attention kernel's four
// variants with a K/V ring of ST stages.
template <int ST>
bool set_attention_smem() {
  constexpr int bytes = sea::fa::CfgT<ST>::SMEM_BYTES;
  return cudaFuncSetAttribute(sea::fa::flash_attn_kernel<false, false, ST>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess &&
         cudaFuncSetAttribute(sea::fa::flash_attn_kernel<false, true, ST>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess &&
         cudaFuncSetAttribute(sea::fa::flash_attn_kernel<true, false, ST>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess &&
         cudaFuncSetAttribute(sea::fa::flash_attn_kernel<true, true, ST>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess &&
         (ST != 4 || (cudaFuncSetAttribute(sea::fa::flash_attn_kernel<false, false, 4, true>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess &&
                      cudaFuncSetAttribute(sea::fa::flash_attn_kernel<false, true, 4, true>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess));
}

// The attention kernel variant for a mask family, the options and the ring depth.
template <int ST>
auto attention_kernel(bool slot, bool ext) {
  return slot ? (ext ? sea::fa::flash_attn_kernel<true, true, ST> : sea::fa::flash_attn_kernel<true, false, ST>)
              : (ext ? sea::fa::flash_attn_kernel<false, true, ST> : sea::fa::flash_attn_kernel<false, false, ST>);
}

// The narrow-tile variant (range family, four stages).
auto narrow_attention_kernel(bool ext) {
  return ext ? sea::fa::flash_attn_kernel<false, true, 4, true> : sea::fa::flash_attn_kernel<false, false, 4, true>;
}

// Per-device set-up: checks for an sm_100 part, records the SM count and the
// error-word address, and raises the dynamic shared-memory limits once.
attn_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_dev[dev];
  if (!g_dev_init[dev]) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    g_dev_init[dev] = true;
    if (major != 10 || minor != 0) return ATTN_ERR_UNSUPPORTED;
    void* err = nullptr;
    if (cudaGetSymbolAddress(&err, g_error_word) != cudaSuccess) return ATTN_ERR_CUDA;
    if (cudaFuncSetAttribute(sea::gemm::qkv_gemm_kernel<sea::gemm::WideTiles>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             sea::gemm::WideTiles::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(sea::gemm::qkv_gemm_kernel<sea::gemm::NarrowTiles>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             sea::gemm::NarrowTiles::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(sea::gemm::qkv_gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             sea::gemm::PairShape::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(sea::q8::qkv_q8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             sea::q8::SMEM_BYTES) != cudaSuccess ||
        !set_attention_smem<2>() || !set_attention_smem<4>())
      return ATTN_ERR_CUDA;
    d.num_sms = sms;
    d.err = static_cast<uint32_t*>(err);
    d.ok = true;
  }
  if (!d.ok) return ATTN_ERR_UNSUPPORTED;
  *out = &d;
  return ATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Byte range [lo, hi) touched by a row-major fp16 matrix.
struct Range {
  uintptr_t lo, hi;
};
Range mat_range(const void* p, int64_t rows, int64_t cols, int64_t stride) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  return {lo, lo + static_cast<uintptr_t>(((rows - 1) * stride + cols) * 2)};
}
bool overlaps(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

bool encode_2d(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint64_t stride_bytes,
               uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {stride_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Raw Q8_0 rows as 2-byte units (the 34-byte blocks are not 4-byte aligned;
// 8 blocks = 272 bytes = 136 units = one box row), no swizzle.
bool encode_q8_rows(CUtensorMap* m, const void* ptr, uint64_t units_per_row, uint64_t rows, uint32_t box_units,
                    uint32_t box_rows) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {units_per_row, rows};
  cuuint64_t strides[1] = {units_per_row * 2};
  cuuint32_t box[2] = {box_units, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// (columns, frames, sequence) view of a [batch*t, >=cols] matrix: rows past a
// sequence's end read as zeros instead of the next sequence's frames.
bool encode_seq_3d(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t t, uint64_t batch,
                   uint64_t row_stride_elems, uint32_t box_rows = 128) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {cols, t, batch};
  cuuint64_t strides[2] = {row_stride_elems * 2, row_stride_elems * 2 * t};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct FaPlan {
  int seg_len, tiles_per_seg, q_tiles;
  int n_kv_max;
  int kv_splits, kv_tiles_per_split;
  bool merge;  // splits merged inside a thread-block cluster (no workspace)
  size_t ws_bytes;
};

// Splits up to this many are merged through distributed shared memory in a
// cluster of that many CTAs (the portable cluster size); more need the
// workspace and the combine kernel.
constexpr int kMaxClusterSplits = 8;

int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

// Multiplier and shift for sea::fa::div_c (division by a launch constant).
sea::fa::DivC make_divc(int d) {
  sea::fa::DivC f{0u, 0u, d};
  if (d <= 1) return f;
  int l = 0;
  while ((int64_t(1) << l) < d) ++l;  // ceil(log2 d)
  f.m = static_cast<uint32_t>(((uint64_t(1) << (31 + l)) + static_cast<uint64_t>(d) - 1) / static_cast<uint64_t>(d));
  f.s = static_cast<uint32_t>(l - 1);
  return f;
}

// Launch plan shared by attn_forward and attn_workspace_size.
FaPlan plan_forward(int batch, int t_q, int t_kv, int n_heads, int mask_kind, int chunk_len, int num_sms) {
  FaPlan pl{};
  const bool chunked = mask_kind == sea::fa::kChunk && chunk_len < t_q;
  if (chunked) {
    // Segments of whole chunks: one chunk when it is at least a tile long,
    // otherwise as many whole chunks as fit in 128 rows.
    pl.seg_len = chunk_len >= sea::fa::BQ ? chunk_len : (sea::fa::BQ / chunk_len) * chunk_len;
    pl.tiles_per_seg = ceil_div(pl.seg_len, sea::fa::BQ);
    pl.q_tiles = ceil_div(t_q, pl.seg_len) * pl.tiles_per_seg;
    pl.n_kv_max = ceil_div(pl.seg_len, sea::fa::BKV) + 1;
  } else {
    pl.seg_len = t_q;
    pl.tiles_per_seg = ceil_div(t_q, sea::fa::BQ);
    pl.q_tiles = pl.tiles_per_seg;
    pl.n_kv_max = ceil_div(t_kv, sea::fa::BKV);
  }
  pl.kv_splits = 1;
  pl.kv_tiles_per_split = pl.n_kv_max;
  const int64_t base_units = static_cast<int64_t>(batch) * n_heads * pl.q_tiles;
  // CHUNK tiles already fill the GPU; the split serves short query blocks.
  if (mask_kind != sea::fa::kChunk && base_units * 2 <= num_sms && pl.n_kv_max >= 2) {
    int splits = static_cast<int>(std::min<int64_t>(pl.n_kv_max, std::max<int64_t>(1, num_sms / base_units)));
    const int per = ceil_div(pl.n_kv_max, splits);
    splits = ceil_div(pl.n_kv_max, per);
    if (splits > 1) {
      pl.kv_splits = splits;
      pl.kv_tiles_per_split = per;
      pl.merge = splits <= kMaxClusterSplits;
      if (!pl.merge) {
        const size_t rows = static_cast<size_t>(splits) * batch * n_heads * t_q;
        pl.ws_bytes = rows * sea::fa::DH * sizeof(float) + rows * 2 * sizeof(float);
      }
    }
  }
  return pl;
}

// Query tiles of at most 32 rows with no key split and at most one unit per
// SM take the narrow layout (the rows in every lane quadrant, each softmax
// warp a quarter of the key columns); the range masks only.
bool narrow_tiles(const FaPlan& pl, int mask_kind, int64_t units, int num_sms) {
  return mask_kind != sea::fa::kSlotmask && pl.kv_splits == 1 && pl.tiles_per_seg == 1 && pl.seg_len <= 32 &&
         units <= num_sms;
}

// Launches with programmatic stream serialization: the kernel may start its
// prologue while the previous kernel in the stream finishes; every kernel of
// this library waits (griddepcontrol.wait) before it touches global memory.
// cluster_x > 1 launches thread-block clusters of that many CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                               unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  unsigned n = 1;
  if (cluster_x > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  return launch_pdl_cluster(kernel, grid, block, smem, stream, 1u, std::forward<Args>(args)...);
}


// Row counts from which the projection runs on CTA pairs (256 x 256 tiles,
// cta_group::2): large enough that the pair tiles fill the GPU.
constexpr int64_t kPairMinRows = 4096;
constexpr int kPairTileN = 512;  // plan code for the pair kernel (tile 256 rows x 256 columns)

// Projection tile width by estimated time: waves of 128x256 tiles against
// waves of 128x192 tiles, which cost ~0.835 of a wide tile each (measured on
// B200).
int gemm_tile_n(int64_t rows, int64_t n, int num_sms) {
  using namespace sea::gemm;
  if (rows >= kPairMinRows && n % PairShape::BN == 0) return kPairTileN;
  const int64_t m_tiles = ceil_div(rows, BM);
  const int64_t waves_wide = (m_tiles * ceil_div(n, WideTiles::BN) + num_sms - 1) / num_sms;
  const int64_t waves_narrow = (m_tiles * ceil_div(n, NarrowTiles::BN) + num_sms - 1) / num_sms;
  const bool narrow = n % NarrowTiles::BN == 0 && waves_narrow * 835 < waves_wide * 1000;
  return narrow ? NarrowTiles::BN : WideTiles::BN;
}

bool valid_mat(const attn_mat& m, int64_t cols) {
  return m.ptr != nullptr && aligned16(m.ptr) && m.row_stride >= cols && (m.row_stride % 8) == 0;
}

// Argument checks of the attention entry points: pure host arithmetic on the
// arguments, no CUDA call. ATTN_OK or ATTN_ERR_INVALID.
attn_status validate_attention(attn_mat q, attn_mat k, attn_mat v, int32_t batch, int32_t t_q, int32_t t_kv,
                               int32_t n_heads, int32_t head_dim, const attn_mask& mask, const float* sinks,
                               float scale, attn_mat out, const void* workspace, size_t workspace_bytes) {
  if (batch <= 0 || t_q <= 0 || t_kv <= 0 || n_heads <= 0) return ATTN_ERR_INVALID;
  if (head_dim != sea::fa::DH) return ATTN_ERR_INVALID;
  if (batch > 65535 || n_heads > 65535) return ATTN_ERR_INVALID;
  if (static_cast<int64_t>(batch) * t_q > INT32_MAX || static_cast<int64_t>(batch) * t_kv > INT32_MAX)
    return ATTN_ERR_INVALID;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID;
  const int64_t cols = static_cast<int64_t>(n_heads) * head_dim;
  if (!valid_mat(q, cols) || !valid_mat(k, cols) || !valid_mat(v, cols) || !valid_mat(out, cols))
    return ATTN_ERR_INVALID;
  auto misaligned4 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 3u) != 0; };
  if ((mask.flags & ~ATTN_FLAG_NO_SPLIT) != 0) return ATTN_ERR_INVALID;
  if (mask.causal != 0 && mask.causal != 1) return ATTN_ERR_INVALID;
  if (mask.kind != ATTN_MASK_BAND && mask.window != 0) return ATTN_ERR_INVALID;
  if (misaligned4(mask.q_lens) || misaligned4(mask.kv_lens) || misaligned4(sinks)) return ATTN_ERR_INVALID;
  if (mask.kind == ATTN_MASK_CHUNK) {
    if (mask.chunk_len <= 0 || t_q != t_kv) return ATTN_ERR_INVALID;
  } else if (mask.kind == ATTN_MASK_SLOTMASK) {
    if (mask.bits == nullptr || misaligned4(mask.bits)) return ATTN_ERR_INVALID;
    if (t_kv > sea::fa::MAX_FLAG_WORDS * 32 * sea::fa::BKV) return ATTN_ERR_INVALID;
    if (mask.words_per_row < (t_kv + 31) / 32) return ATTN_ERR_INVALID;
    // the bits define the allowed set alone
    if (mask.causal != 0 || mask.q_lens != nullptr || mask.kv_lens != nullptr) return ATTN_ERR_INVALID;
  } else if (mask.kind == ATTN_MASK_BAND) {
    if (mask.window <= 0) return ATTN_ERR_INVALID;
  } else if (mask.kind != ATTN_MASK_FULL) {
    return ATTN_ERR_INVALID;
  }
  const Range ro = mat_range(out.ptr, static_cast<int64_t>(batch) * t_q, cols, out.row_stride);
  if (overlaps(ro, mat_range(q.ptr, static_cast<int64_t>(batch) * t_q, cols, q.row_stride)) ||
      overlaps(ro, mat_range(k.ptr, static_cast<int64_t>(batch) * t_kv, cols, k.row_stride)) ||
      overlaps(ro, mat_range(v.ptr, static_cast<int64_t>(batch) * t_kv, cols, v.row_stride)))
    return ATTN_ERR_INVALID;
  if (workspace != nullptr && !aligned16(workspace)) return ATTN_ERR_INVALID;
  if (workspace == nullptr && workspace_bytes != 0) return ATTN_ERR_INVALID;
  return ATTN_OK;
}

attn_status launch_attention(attn_mat q, attn_mat k, attn_mat v, int32_t batch, int32_t t_q, int32_t t_kv,
                             int32_t n_heads, int32_t head_dim, attn_mask mask, const float* sinks, float scale,
                             attn_mat out, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (attn_status st = validate_attention(q, k, v, batch, t_q, t_kv, n_heads, head_dim, mask, sinks, scale, out,
                                          workspace, workspace_bytes);
      st != ATTN_OK)
    return st;
  const int64_t cols = static_cast<int64_t>(n_heads) * head_dim;

  DeviceInfo* dev = nullptr;
  if (attn_status st = device_info(&dev); st != ATTN_OK) return st;

  FaPlan pl = plan_forward(batch, t_q, t_kv, n_heads, mask.kind, mask.chunk_len, dev->num_sms);
  if (mask.flags & ATTN_FLAG_NO_SPLIT) {
    pl.kv_splits = 1;
    pl.kv_tiles_per_split = pl.n_kv_max;
    pl.merge = false;
    pl.ws_bytes = 0;
  }
  if (pl.kv_splits > 1 && !pl.merge) {
    if (workspace == nullptr) {
      pl.kv_splits = 1;  // caller opted out of the split: same result, one CTA per key range
      pl.kv_tiles_per_split = pl.n_kv_max;
      pl.ws_bytes = 0;
    } else if (workspace_bytes < pl.ws_bytes) {
      return ATTN_ERR_INVALID;
    }
  }

  const int64_t units = static_cast<int64_t>(batch) * n_heads * pl.q_tiles * pl.kv_splits;
  if (units > INT32_MAX) return ATTN_ERR_INVALID;
  const bool narrow = narrow_tiles(pl, mask.kind == ATTN_MASK_SLOTMASK ? sea::fa::kSlotmask : sea::fa::kFull, units,
                                   dev->num_sms);
  CUtensorMap tq, tk, tv;
  if (!encode_seq_3d(&tq, q.ptr, cols, t_q, batch, q.row_stride, narrow ? 32 : 128) ||
      !encode_seq_3d(&tk, k.ptr, cols, t_kv, batch, k.row_stride) ||
      !encode_seq_3d(&tv, v.ptr, cols, t_kv, batch, v.row_stride))
    return ATTN_ERR_CUDA;

  sea::fa::Params p{};
  p.batch = batch;
  p.t_q = t_q;
  p.t_kv = t_kv;
  p.n_heads = n_heads;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.mask_kind = mask.kind;
  p.chunk_len = (mask.kind == ATTN_MASK_CHUNK && mask.chunk_len < t_q) ? mask.chunk_len : t_q;
  if (mask.kind == ATTN_MASK_CHUNK && mask.chunk_len >= t_q) p.mask_kind = sea::fa::kFull;
  p.bits = mask.kind == ATTN_MASK_SLOTMASK ? mask.bits : nullptr;
  p.words_per_row = mask.kind == ATTN_MASK_SLOTMASK ? mask.words_per_row : 0;
  // |p_i - j| never exceeds t_q + t_kv, so a wider window changes nothing.
  p.window = mask.kind == ATTN_MASK_BAND
                 ? static_cast<int>(std::min<int64_t>(mask.window, static_cast<int64_t>(t_q) + t_kv + 1))
                 : 0;
  p.causal = mask.causal;
  p.q_lens = mask.q_lens;
  p.kv_lens = mask.kv_lens;
  p.sinks = sinks;
  p.seg_len = pl.seg_len;
  p.tiles_per_seg = pl.tiles_per_seg;
  p.q_tiles = pl.q_tiles;
  p.kv_splits = pl.kv_splits;
  p.kv_tiles_per_split = pl.kv_tiles_per_split;
  p.dv_splits = make_divc(p.kv_splits);
  p.dv_q_tiles = make_divc(p.q_tiles);
  p.dv_heads = make_divc(p.n_heads);
  p.dv_tiles_per_seg = make_divc(p.tiles_per_seg);
  p.dv_chunk = make_divc(p.chunk_len);
  p.out = static_cast<__half*>(out.ptr);
  p.out_stride = out.row_stride;
  float* ws = static_cast<float*>(workspace);
  const size_t ws_rows = static_cast<size_t>(pl.kv_splits) * batch * n_heads * t_q;
  p.ws_o = pl.kv_splits > 1 && !pl.merge ? ws : nullptr;
  p.ws_ml = pl.kv_splits > 1 && !pl.merge ? ws + ws_rows * sea::fa::DH : nullptr;
  p.merge = pl.merge ? 1 : 0;
  p.err = dev->err;
  p.limit_ns = sea::kDefaultTimeoutNs;

  p.units = static_cast<int>(units);
  const bool slot = p.mask_kind == sea::fa::kSlotmask;
  // The lengths / causal / BAND / sinks code is compiled into its own variant.
  const bool ext = p.mask_kind == sea::fa::kBand || p.causal != 0 || p.q_lens != nullptr ||
                   p.kv_lens != nullptr || p.sinks != nullptr;
  const int threads = sea::fa::Cfg::THREADS;
  cudaError_t err;
  // A merged split runs one unit per CTA, the splits of a query tile (units
  // next to each other) forming one cluster.
  const unsigned cluster = pl.merge ? static_cast<unsigned>(pl.kv_splits) : 1u;
  // At most one CTA per SM: a four-stage K/V ring (a short unit's key tiles
  // all load at once); otherwise two CTAs per SM with two stages each.
  const bool deep = units <= dev->num_sms;
  if (narrow) {
    err = launch_pdl(narrow_attention_kernel(ext), dim3(p.units), dim3(threads), sea::fa::CfgT<4>::SMEM_BYTES, stream,
                     tq, tk, tv, p);
  } else if (slot || deep) {
    // One unit per CTA (SLOTMASK: its tile flags need a pass over every row's words).
    if (deep)
      err = launch_pdl_cluster(attention_kernel<4>(slot, ext), dim3(p.units), dim3(threads),
                               sea::fa::CfgT<4>::SMEM_BYTES, stream, cluster, tq, tk, tv, p);
    else
      err = launch_pdl_cluster(attention_kernel<2>(slot, ext), dim3(p.units), dim3(threads),
                               sea::fa::CfgT<2>::SMEM_BYTES, stream, cluster, tq, tk, tv, p);
  } else {
    // Persistent: Cfg::MIN_BLOCKS CTAs per SM walk the units.
    const int grid = static_cast<int>(std::min<int64_t>(units, int64_t(sea::fa::Cfg::MIN_BLOCKS) * dev->num_sms));
    err = launch_pdl(attention_kernel<2>(false, ext), dim3(grid), dim3(threads), sea::fa::Cfg::SMEM_BYTES, stream, tq,
                     tk, tv, p);
  }
  if (err != cudaSuccess) return ATTN_ERR_CUDA;
  if (pl.kv_splits > 1 && !pl.merge) {
    const int64_t rows = static_cast<int64_t>(batch) * n_heads * t_q;
    if (launch_pdl(sea::fa::combine_kernel, dim3(ceil_div(rows, 8)), dim3(256), 0, stream,
                   static_cast<const float*>(p.ws_o), static_cast<const float*>(p.ws_ml), pl.kv_splits, batch,
                   n_heads, t_q, sinks, p.out, p.out_stride) != cudaSuccess)
      return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

// ---------------------------------------------------------------------------
// Fixed scratch for attn_cross_static_scratch (no allocation by the caller).
// ---------------------------------------------------------------------------

constexpr size_t kStaticScratchBytes = size_t(4) << 20;  // 4 MiB per device

// Split-KV partials (unnormalised O, running max and sum) of
// attn_cross_static_scratch. Every device that loads this library's device
// code holds these 4 MiB until the process exits. In host code the name below
// only stands in for the symbol; its device address comes from
// cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

void* g_static_scratch_ptr[kMaxDevices] = {};

// Once per device, with that device current: resolve the scratch address.
attn_status static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_static_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || ptr == nullptr) return ATTN_ERR_CUDA;
    g_static_scratch_ptr[dev] = ptr;
  }
  *out = g_static_scratch_ptr[dev];
  return ATTN_OK;
}

}  // namespace

extern "C" {

attn_status attn_qkv_pack(attn_mat x, const void* w_qkv, const void* b_q, const void* b_v, int64_t rows,
                          int32_t d_model, attn_mat qkv_out, attn_stream_t stream) {
  if (rows <= 0 || rows > INT32_MAX) return ATTN_ERR_INVALID;
  if (d_model <= 0 || d_model % 64 != 0 || d_model > 65536) return ATTN_ERR_INVALID;
  if (!valid_mat(x, d_model) || !valid_mat(qkv_out, 3 * static_cast<int64_t>(d_model))) return ATTN_ERR_INVALID;
  if (w_qkv == nullptr || !aligned16(w_qkv)) return ATTN_ERR_INVALID;
  if ((b_q != nullptr && !aligned16(b_q)) || (b_v != nullptr && !aligned16(b_v))) return ATTN_ERR_INVALID;
  const int64_t n = 3 * static_cast<int64_t>(d_model);
  const Range ro = mat_range(qkv_out.ptr, rows, n, qkv_out.row_stride);
  if (overlaps(ro, mat_range(x.ptr, rows, d_model, x.row_stride)) ||
      overlaps(ro, mat_range(w_qkv, n, d_model, d_model)))
    return ATTN_ERR_INVALID;

  DeviceInfo* dev = nullptr;
  if (attn_status st = device_info(&dev); st != ATTN_OK) return st;

  CUtensorMap tx, tw, to;
  using namespace sea::gemm;
  const int64_t m_tiles = ceil_div(rows, BM);
  const int bn = gemm_tile_n(rows, n, dev->num_sms);
  const bool pair = bn == kPairTileN;
  const bool narrow = bn == NarrowTiles::BN;
  // A pair CTA loads 128 rows of W (its half of the 256-column tile).
  const uint32_t w_box_rows = pair ? PairShape::BN / 2 : static_cast<uint32_t>(bn);
  if (!encode_2d(&tx, x.ptr, d_model, rows, x.row_stride * 2, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&tw, w_qkv, d_model, n, static_cast<uint64_t>(d_model) * 2, BK, w_box_rows,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&to, qkv_out.ptr, n, rows, qkv_out.row_stride * 2, EPI_COLS, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return ATTN_ERR_CUDA;
  Args a{};
  a.b_q = static_cast<const __half*>(b_q);
  a.b_v = static_cast<const __half*>(b_v);
  a.m = static_cast<int>(rows);
  a.n = static_cast<int>(n);
  a.k = d_model;
  a.d_model = d_model;
  a.err = dev->err;
  a.limit_ns = sea::kDefaultTimeoutNs;
  cudaError_t err;
  if (pair) {
    const int64_t tiles = ceil_div(rows, 2 * BM) * ceil_div(n, PairShape::BN);
    const int pairs = static_cast<int>(std::min<int64_t>(tiles, dev->num_sms / 2));
    err = launch_pdl_cluster(qkv_gemm_pair_kernel, dim3(2 * pairs), dim3(THREADS), PairShape::SMEM_BYTES, stream, 2u,
                             tx, tw, to, a);
  } else {
    const int64_t tiles = m_tiles * ceil_div(n, bn);
    const int grid = static_cast<int>(std::min<int64_t>(tiles, dev->num_sms));
    err = narrow ? launch_pdl(qkv_gemm_kernel<NarrowTiles>, dim3(grid), dim3(THREADS), NarrowTiles::SMEM_BYTES, stream,
                              tx, tw, to, a)
                 : launch_pdl(qkv_gemm_kernel<WideTiles>, dim3(grid), dim3(THREADS), WideTiles::SMEM_BYTES, stream, tx,
                              tw, to, a);
  }
  if (err != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

attn_status attn_qkv_pack_q8_0(attn_mat x, const void* w_q8_0, const void* b_q, const void* b_v, int64_t rows,
                               int32_t d_model, attn_mat qkv_out, attn_stream_t stream) {
  using namespace sea::q8;
  if (rows <= 0 || rows > INT32_MAX) return ATTN_ERR_INVALID;
  if (d_model <= 0 || d_model % BKQ != 0 || d_model > 65536) return ATTN_ERR_INVALID;
  if (!valid_mat(x, d_model) || !valid_mat(qkv_out, 3 * static_cast<int64_t>(d_model))) return ATTN_ERR_INVALID;
  if (w_q8_0 == nullptr || !aligned16(w_q8_0)) return ATTN_ERR_INVALID;
  if ((b_q != nullptr && !aligned16(b_q)) || (b_v != nullptr && !aligned16(b_v))) return ATTN_ERR_INVALID;
  const int64_t n = 3 * static_cast<int64_t>(d_model);
  const int64_t row_bytes = static_cast<int64_t>(d_model) / QBLOCK * QBLOCK_BYTES;
  const Range ro = mat_range(qkv_out.ptr, rows, n, qkv_out.row_stride);
  const Range rw{reinterpret_cast<uintptr_t>(w_q8_0), reinterpret_cast<uintptr_t>(w_q8_0) + n * row_bytes};
  if (overlaps(ro, mat_range(x.ptr, rows, d_model, x.row_stride)) || overlaps(ro, rw)) return ATTN_ERR_INVALID;

  DeviceInfo* dev = nullptr;
  if (attn_status st = device_info(&dev); st != ATTN_OK) return st;

  CUtensorMap tx, tw;
  if (!encode_2d(&tx, x.ptr, d_model, rows, x.row_stride * 2, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_q8_rows(&tw, w_q8_0, row_bytes / 2, n, RAW_ROW_BYTES / 2, BN))
    return ATTN_ERR_CUDA;
  Args a{};
  a.b_q = static_cast<const __half*>(b_q);
  a.b_v = static_cast<const __half*>(b_v);
  a.out = static_cast<__half*>(qkv_out.ptr);
  a.out_stride = qkv_out.row_stride;
  a.m = static_cast<int>(rows);
  a.d_model = d_model;
  a.err = dev->err;
  a.limit_ns = sea::kDefaultTimeoutNs;
  const dim3 grid(ceil_div(rows, BM), static_cast<unsigned>(n / BN));
  if (launch_pdl(qkv_q8_kernel, grid, dim3(THREADS), SMEM_BYTES, stream, tx, tw, a) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return ATTN_OK;
}

attn_status attn_forward(attn_mat q, attn_mat k, attn_mat v, int32_t batch, int32_t t_q, int32_t t_kv,
                         int32_t n_heads, int32_t head_dim, attn_mask mask, float scale, attn_mat out,
                         void* workspace, size_t workspace_bytes, attn_stream_t stream) {
  return launch_attention(q, k, v, batch, t_q, t_kv, n_heads, head_dim, mask, nullptr, scale, out, workspace,
                          workspace_bytes, stream);
}

attn_status attn_forward_sinks(attn_mat q, attn_mat k, attn_mat v, int32_t batch, int32_t t_q, int32_t t_kv,
                               int32_t n_heads, int32_t head_dim, attn_mask mask, const float* sinks, float scale,
                               attn_mat out, void* workspace, size_t workspace_bytes, attn_stream_t stream) {
  return launch_attention(q, k, v, batch, t_q, t_kv, n_heads, head_dim, mask, sinks, scale, out, workspace,
                          workspace_bytes, stream);
}

attn_status attn_cross(attn_mat q, attn_mat k_enc, attn_mat v_enc, int32_t batch, int32_t t_q, int32_t t_enc,
                       int32_t n_heads, int32_t head_dim, float scale, attn_mat out, void* workspace,
                       size_t workspace_bytes, attn_stream_t stream) {
  attn_mask full{};
  full.kind = ATTN_MASK_FULL;
  return launch_attention(q, k_enc, v_enc, batch, t_q, t_enc, n_heads, head_dim, full, nullptr, scale, out,
                          workspace, workspace_bytes, stream);
}

attn_status attn_cross_static_scratch(attn_mat q, attn_mat k_enc, attn_mat v_enc, int32_t batch, int32_t t_q,
                                      int32_t t_enc, int32_t n_heads, int32_t head_dim, float scale, attn_mat out,
                                      attn_stream_t stream) {
  attn_mask full{};
  full.kind = ATTN_MASK_FULL;
  // The arguments are checked before the device is queried, so an invalid
  // call returns ATTN_ERR_INVALID without any CUDA call, as attn_cross does.
  if (attn_status st = validate_attention(q, k_enc, v_enc, batch, t_q, t_enc, n_heads, head_dim, full, nullptr,
                                          scale, out, nullptr, 0);
      st != ATTN_OK)
    return st;
  DeviceInfo* dev = nullptr;
  if (attn_status st = device_info(&dev); st != ATTN_OK) return st;
  void* scratch = nullptr;
  if (attn_status st = static_scratch(&scratch); st != ATTN_OK) return st;
  // Same launch as attn_cross with the fixed scratch as its workspace: a split
  // that needs more than kStaticScratchBytes is rejected (ATTN_ERR_INVALID)
  // before anything is launched. Every partial the combine step reads is
  // written earlier in the same call, so nothing has to be cleared.
  return launch_attention(q, k_enc, v_enc, batch, t_q, t_enc, n_heads, head_dim, full, nullptr, scale, out,
                          scratch, kStaticScratchBytes, stream);
}

size_t attn_workspace_size(int32_t batch, int32_t t_q, int32_t t_kv, int32_t n_heads, int32_t head_dim,
                           int32_t mask_kind) {
  if (batch <= 0 || t_q <= 0 || t_kv <= 0 || n_heads <= 0 || head_dim != sea::fa::DH) return 0;
  if (mask_kind == ATTN_MASK_CHUNK) return 0;
  DeviceInfo* dev = nullptr;
  if (device_info(&dev) != ATTN_OK) return 0;
  return plan_forward(batch, t_q, t_kv, n_heads, mask_kind, 0, dev->num_sms).ws_bytes;
}

const char* attn_status_string(attn_status status) {
  switch (status) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID: return "ATTN_ERR_INVALID: invalid argument, nothing launched";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED: needs an sm_100 (B200) device";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA: a CUDA call or kernel launch failed";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT: a kernel's bounded wait expired";
  }
  return "ATTN_ERR_UNKNOWN";
}

attn_status attn_debug_error_word(attn_stream_t stream, uint32_t* word_out) {
  DeviceInfo* dev = nullptr;
  if (attn_status st = device_info(&dev); st != ATTN_OK) return st;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return ATTN_ERR_CUDA;
  uint32_t w = 0;
  if (cudaMemcpy(&w, dev->err, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_ERR_CUDA;
  const uint32_t zero = 0;
  if (cudaMemcpy(dev->err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return ATTN_ERR_CUDA;
  if (word_out) *word_out = w;
  return w ? ATTN_ERR_TIMEOUT : ATTN_OK;
}

attn_status attn_debug_plan(int32_t batch, int32_t t_q, int32_t t_kv, int32_t n_heads, int32_t mask_kind,
                            int32_t chunk_len, int32_t num_sms, int64_t proj_rows, int32_t d_model,
                            attn_plan_info* out) {
  if (out == nullptr || batch <= 0 || t_q <= 0 || t_kv <= 0 || n_heads <= 0 || num_sms <= 0) return ATTN_ERR_INVALID;
  if (mask_kind < ATTN_MASK_FULL || mask_kind > ATTN_MASK_BAND) return ATTN_ERR_INVALID;
  if (mask_kind == ATTN_MASK_CHUNK && chunk_len <= 0) return ATTN_ERR_INVALID;
  const int kind = (mask_kind == ATTN_MASK_CHUNK && chunk_len >= t_q) ? ATTN_MASK_FULL : mask_kind;
  const FaPlan pl = plan_forward(batch, t_q, t_kv, n_heads, kind, chunk_len, num_sms);
  out->seg_len = pl.seg_len;
  out->tiles_per_seg = pl.tiles_per_seg;
  out->q_tiles = pl.q_tiles;
  out->kv_splits = pl.kv_splits;
  out->kv_tiles_per_split = pl.kv_tiles_per_split;
  out->units = static_cast<int64_t>(batch) * n_heads * pl.q_tiles * pl.kv_splits;
  out->workspace_bytes = pl.ws_bytes;
  out->cluster_merge = pl.merge ? 1 : 0;
  out->narrow = narrow_tiles(pl, kind == ATTN_MASK_SLOTMASK ? sea::fa::kSlotmask : sea::fa::kFull, out->units, num_sms)
                    ? 1
                    : 0;
  out->proj_tile_n = (proj_rows > 0 && d_model > 0) ? gemm_tile_n(proj_rows, 3 * static_cast<int64_t>(d_model), num_sms)
                                                    : 0;
  return ATTN_OK;
}

attn_status attn_debug_timeout_probe(int64_t limit_ns, attn_stream_t stream) {
  if (limit_ns < 1000 || limit_ns > 1000000000) return ATTN_ERR_INVALID;
  DeviceInfo* dev = nullptr;
  if (attn_status st = device_info(&dev); st != ATTN_OK) return st;
  timeout_probe_kernel<<<1, 32, 0, stream>>>(dev->err, static_cast<uint64_t>(limit_ns));
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

}  // extern "C"
