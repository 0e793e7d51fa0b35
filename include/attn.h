/*
 * attn.h -- C ABI of libattn.so: the Whisper-style attention pass on B200 (sm_100a).
 *
 * The pass has two stages, both hand-written CUDA kernels for sm_100a:
 *   1. a packed QKV projection (one GEMM instead of three), and
 *   2. fused multi-head flash attention with fp16 K/V, an fp32 online softmax
 *      and no score matrix in memory, under one of three masks.
 * Sources (page titles and sections):
 *   - "Add Edda ASR with DFlash2 speculative decoding" (audio.cpp PR #1223), PR
 *     description: the encoder packs QKV and runs flash attention over F16 K/V
 *     instead of materialising F32 scores for all 1500 frames; block verification
 *     of an anchor plus up to 15 drafted tokens against KV slots indexed by
 *     position; a token-tree KV cache whose mask rows admit only ancestors; the
 *     drafter's flash cross-attention.
 *   - "higgs-audio-v3-stt GGUF" model card, "Architecture note (chunked encoder)":
 *     4 s chunks encoded independently with within-chunk attention.
 *   - BuzzASR "danish" discussion #1: the Whisper encoder is fully bidirectional;
 *     a shortened 500-position encoder input (1000 mel frames).
 *   - "Add causal attention and attention sinks to DFlash" (the drafter PR):
 *     block-internal attention that is non-causal unless the model says causal,
 *     an optional sliding window, and optional per-head attention sinks.
 *
 * Conventions for every entry point
 *   - All tensors are IEEE fp16 (binary16) in device memory unless stated.
 *   - A matrix is passed as attn_mat {ptr, row_stride}: element (r, c) lives at
 *     ptr[r * row_stride + c]; row_stride counts elements. Sequence b of a batch
 *     of sequences of length t occupies rows [b*t, (b+1)*t).
 *   - Head h of a [rows, n_heads*64] matrix uses columns [64h, 64h+64).
 *   - The caller owns every buffer, including the workspace. The library
 *     allocates no device memory, keeps no per-call state and never
 *     synchronises: all work is enqueued on `stream` in order and the call
 *     returns immediately.
 *   - Arguments are validated on the host before anything is launched. An
 *     invalid argument returns ATTN_ERR_INVALID and launches nothing; there is
 *     no fallback path. A launch failure returns ATTN_ERR_CUDA.
 *   - Device pointers must be 16-byte aligned and row strides multiples of 8
 *     elements (the tensor-memory-accelerator copies need 16-byte strides).
 *   - Kernels are launched with programmatic stream serialization: each one
 *     may start its prologue while the previous kernel in the stream finishes,
 *     and waits for that kernel's completion before touching global memory.
 *     Ordering on the stream is unchanged for the caller; a caller's own kernel
 *     that is itself launched programmatically after one of these must wait
 *     (griddepcontrol.wait) before reading this library's outputs.
 *   - No C++ exception crosses this interface.
 */
#ifndef SEA_ATTN_H
#define SEA_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st *attn_stream_t;

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID = 1,     /* bad argument; nothing was launched */
  ATTN_ERR_UNSUPPORTED = 2, /* valid request this library does not serve (e.g. no sm_100 device) */
  ATTN_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  ATTN_ERR_TIMEOUT = 4      /* a kernel's bounded wait expired (see attn_debug_error_word) */
} attn_status;

/* attn_mask.flags bits */
enum {
  ATTN_FLAG_NO_SPLIT = 1  /* never split the key range over several CTAs (one
                             CTA per query tile: a fixed summation order) */
};

typedef enum {
  ATTN_MASK_FULL = 0,     /* every key: the bidirectional encoder window */
  ATTN_MASK_CHUNK = 1,    /* keys in the query's chunk of chunk_len frames */
  ATTN_MASK_SLOTMASK = 2, /* keys whose bit is set in the query row's bitmask */
  ATTN_MASK_BAND = 3      /* keys within `window` positions of the query (sliding window) */
} attn_mask_kind;

/*
 * FULL, CHUNK and BAND form the range family. For sequence b with Q valid
 * query rows and KV valid keys (q_lens[b] and kv_lens[b], or t_q and t_kv when
 * the pointer is NULL), query row i sits at key position p_i = i + KV - Q: a
 * query block is the last Q positions of its keys (the same row index when
 * t_q == t_kv and no lengths are given). Row i may see key j iff
 *   i < Q and j < KV                          (padding never attends nor is seen)
 *   and CHUNK: floor(p_i / chunk_len) == floor(j / chunk_len)
 *   and BAND:  |p_i - j| < window
 *   and, if causal, j <= p_i.
 * Rows with no visible key (including padding rows i >= Q) yield zeros.
 */
typedef struct {
  int32_t kind;            /* attn_mask_kind */
  int32_t chunk_len;       /* CHUNK: frames per chunk, > 0. Chunks start at frame 0
                              of each sequence; the last one may be short. */
  const uint32_t *bits;    /* SLOTMASK: device pointer, [t_q, words_per_row] uint32.
                              Slot j of row i is allowed iff bit (j % 32) of word
                              i*words_per_row + j/32 is set (LSB first). Shared by
                              all heads and all sequences of the batch. 4-byte aligned. */
  int32_t words_per_row;   /* SLOTMASK: >= ceil(t_kv / 32) */
  int32_t window;          /* BAND: >= 1 (values above t_q + t_kv act as t_q + t_kv);
                              0 for every other kind */
  int32_t causal;          /* 0 or 1; 1 also requires j <= p_i (range family only) */
  int32_t flags;           /* 0 or ATTN_FLAG_NO_SPLIT */
  const int32_t *q_lens;   /* range family, optional: device pointer, [batch] int32,
                              valid query rows per sequence; NULL = t_q. Values are
                              clamped to [0, t_q] on the device. 4-byte aligned. */
  const int32_t *kv_lens;  /* same for the keys; NULL = t_kv; clamped to [0, t_kv] */
} attn_mask;

typedef struct {
  void *ptr;               /* device pointer (read-only for inputs) */
  int64_t row_stride;      /* elements between consecutive rows */
} attn_mat;

/*
 * attn_qkv_pack -- the packed QKV projection
 *   qkv[r, j] = sum_c x[r, c] * W[j, c] + bias[j],  bias = [b_q | 0 | b_v]
 * Source: the edda PR description ("packs QKV"): one projection with the packed
 * weight W = [W_q; W_k; W_v] instead of three. As in Whisper, the key projection
 * has no bias.
 *   x        [rows, d_model]    fp16, row_stride >= d_model
 *   w_qkv    [3*d_model, d_model] fp16, contiguous (q rows, k rows, v rows)
 *   b_q, b_v [d_model] fp16, may be NULL (treated as zero)
 *   qkv_out  [rows, 3*d_model]  fp16, row_stride >= 3*d_model; must not overlap x or W
 * d_model must be a positive multiple of 64 and rows >= 1. Accumulates in fp32,
 * adds the bias in fp32 and rounds once to fp16 (round to nearest even).
 */
attn_status attn_qkv_pack(attn_mat x, const void *w_qkv, const void *b_q, const void *b_v,
                          int64_t rows, int32_t d_model, attn_mat qkv_out, attn_stream_t stream);

/*
 * attn_qkv_pack_q8_0 -- the packed QKV projection with Q8_0 weights
 *   qkv[r, j] = sum_c x[r, c] * W[j, c] + bias[j],  bias = [b_q | 0 | b_v],
 *   W[j, 32b + t] = d[j, b] * q[j, b, t]
 * Source: the edda PR's results table (decoder run with Q8_0 weights). The
 * pages name the GGUF Q8_0 type without defining it; its published layout is
 * taken: each weight row is d_model/32 blocks of 34 bytes, a little-endian
 * fp16 scale d followed by 32 signed bytes q (the GGUF tensor's row order).
 * Meant for the decoder's few rows (a verify block): one CTA per 128 rows x 32
 * output columns reads each weight row once.
 *   x        [rows, d_model] fp16, row_stride >= d_model
 *   w_q8_0   [3*d_model rows of d_model/32 * 34 bytes], contiguous, 16-byte
 *            aligned (q rows, k rows, v rows)
 *   b_q, b_v [d_model] fp16 or NULL (zero)
 *   qkv_out  [rows, 3*d_model] fp16, row_stride >= 3*d_model; must not overlap x or W
 * d_model must be a positive multiple of 256 (a K step is 8 blocks = 272 bytes,
 * a multiple of the 16 bytes a tensor-memory-accelerator row needs). Each
 * weight is dequantized to fp16 (d * q rounded once), the products accumulate
 * in fp32, the bias is added in fp32 and the result rounded once to fp16.
 */
attn_status attn_qkv_pack_q8_0(attn_mat x, const void *w_q8_0, const void *b_q, const void *b_v,
                               int64_t rows, int32_t d_model, attn_mat qkv_out, attn_stream_t stream);

/*
 * attn_forward -- multi-head flash attention with a mask
 *   o_i = sum_{j in A_i} softmax_j(scale * <q_i, k_j>) v_j     per head
 * A_i by mask.kind: FULL -> all t_kv keys; CHUNK -> keys of the same chunk
 * (requires t_q == t_kv); BAND -> keys within the window; SLOTMASK -> keys
 * whose bit is set in row i (window, causal, q_lens and kv_lens must be zero /
 * NULL). The range family's lengths and causal flag are defined above. A row
 * with an empty A_i yields zeros.
 *   q   [batch*t_q,  n_heads*64] fp16   (row_stride >= n_heads*64)
 *   k,v [batch*t_kv, n_heads*64] fp16
 *   out [batch*t_q,  n_heads*64] fp16, must not overlap q, k or v
 * q, k and v may be three views of one packed projection buffer (row_stride
 * 3*d_model, pointers at column offsets 0, d_model and 2*d_model).
 * head_dim must be 64. Scores, the running max and sum and the output
 * accumulate in fp32; the softmax weights are rounded to fp16 for the value
 * product; the output is rounded once to fp16.
 * Short query blocks split their key range over several CTAs. A split into
 * at most 8 parts is merged inside a thread-block cluster (the parts combine
 * through distributed shared memory) and needs no workspace; a longer split
 * keeps its partials in the workspace and merges them in a second kernel.
 * mask.flags = ATTN_FLAG_NO_SPLIT turns every split off (one CTA walks each
 * query tile's whole key range, so the summation order does not depend on
 * the SM count); the result agrees within rounding.
 * workspace: device scratch of at least attn_workspace_size(...) bytes, 16-byte
 * aligned (0 bytes, NULL allowed, when no workspace split is planned).
 * Passing workspace == NULL with workspace_bytes == 0 where a workspace split
 * is planned runs that shape unsplit; a non-NULL workspace smaller than
 * required returns ATTN_ERR_INVALID.
 */
attn_status attn_forward(attn_mat q, attn_mat k, attn_mat v, int32_t batch, int32_t t_q,
                         int32_t t_kv, int32_t n_heads, int32_t head_dim, attn_mask mask,
                         float scale, attn_mat out, void *workspace, size_t workspace_bytes,
                         attn_stream_t stream);

/*
 * attn_forward_sinks -- attn_forward with per-head attention sinks
 * Source: the drafter PR (optional per-head "attn_sinks" tensor passed to the
 * attention). Each head h has one extra logit sinks[h], in the units of the
 * scaled scores, that joins the softmax normalisation and carries no value:
 *   o_i = sum_{j in A_i} e^{s_ij} v_j / (e^{sinks[h]} + sum_{j in A_i} e^{s_ij}),
 *   s_ij = scale * <q_i, k_j>.
 * sinks: device pointer, [n_heads] fp32, 4-byte aligned; -INFINITY means no
 * sink for that head; NULL makes the call identical to attn_forward. Every
 * other argument is as for attn_forward (any mask kind).
 */
attn_status attn_forward_sinks(attn_mat q, attn_mat k, attn_mat v, int32_t batch, int32_t t_q,
                               int32_t t_kv, int32_t n_heads, int32_t head_dim, attn_mask mask,
                               const float *sinks, float scale, attn_mat out, void *workspace,
                               size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_cross -- decoder queries attending to every encoder frame
 * Source: the edda PR description (the drafter's flash cross-attention); the
 * decoder attends over the whole encoded sequence (higgs model card note).
 * Same as attn_forward with a FULL mask and t_kv = t_enc (t_q != t_enc allowed).
 *   q [batch*t_q, n_heads*64], k_enc, v_enc [batch*t_enc, n_heads*64], out like q.
 */
attn_status attn_cross(attn_mat q, attn_mat k_enc, attn_mat v_enc, int32_t batch, int32_t t_q,
                       int32_t t_enc, int32_t n_heads, int32_t head_dim, float scale,
                       attn_mat out, void *workspace, size_t workspace_bytes,
                       attn_stream_t stream);

/*
 * attn_cross_static_scratch -- attn_cross for callers that cannot allocate
 * device memory.
 * The pages describe no such entry point; it exists for hosts that may not
 * call cudaMalloc or hand out device buffers on the hot path: an audio or
 * speech plugin whose host owns every device allocation through its own
 * pool, or a real-time decode loop that must not allocate between frames.
 * Same arguments, result and error behaviour as attn_cross, without the
 * workspace: the partials of a split that needs a workspace (more than 8
 * key splits) live in a fixed 4 MiB array in the library's device memory
 * (one per device, held until the process exits).
 *   - The first call on a device looks up that array's address; make it
 *     before any stream capture on that device.
 *   - A shape whose split needs more than 4 MiB (splits x batch x n_heads x
 *     t_q x 264 bytes; splits only happen when batch*n_heads*ceil(t_q/128)
 *     is at most half the SM count, and need the array only beyond 8 splits)
 *     returns ATTN_ERR_INVALID and launches nothing.
 *   - Every call uses the same array. Calls whose kernels may overlap on the
 *     GPU (different streams, or other devices' threads with this device
 *     current) race on it: order them on one stream.
 *   - Nothing is allocated or freed.
 */
attn_status attn_cross_static_scratch(attn_mat q, attn_mat k_enc, attn_mat v_enc, int32_t batch, int32_t t_q,
                                      int32_t t_enc, int32_t n_heads, int32_t head_dim, float scale,
                                      attn_mat out, attn_stream_t stream);

/*
 * attn_workspace_size -- bytes of workspace attn_forward / attn_cross use for
 * these sizes on the current device (0 when no split, or a split merged in a
 * cluster, is planned).
 */
size_t attn_workspace_size(int32_t batch, int32_t t_q, int32_t t_kv, int32_t n_heads,
                           int32_t head_dim, int32_t mask_kind);

/* Static, human-readable name of a status code. */
const char *attn_status_string(attn_status status);

/*
 * attn_debug_error_word -- synchronises `stream`, then reads and clears the
 * device error word that kernels set when a bounded wait expires. Writes the
 * raw word to *word_out when word_out is not NULL. Returns ATTN_ERR_TIMEOUT if
 * it was set, ATTN_OK otherwise.
 */
attn_status attn_debug_error_word(attn_stream_t stream, uint32_t *word_out);

/*
 * attn_debug_plan -- the host-side launch plan, without a device: what
 * attn_forward / attn_qkv_pack would choose on a GPU with num_sms SMs.
 *   seg_len, tiles_per_seg, q_tiles: the query-tile schedule (CHUNK: segments
 *     of whole chunks; otherwise one segment of t_q rows)
 *   kv_splits, kv_tiles_per_split: the key split (1 = none); units = work units
 *   workspace_bytes: what attn_workspace_size would report for that device
 *   cluster_merge: 1 when the split parts merge inside a cluster (no workspace)
 *   narrow: 1 when query tiles of at most 32 rows are computed in the narrow
 *     layout (the rows in each of the four tensor-memory lane quadrants, each
 *     softmax warp a quarter of every key tile's columns, the four partials
 *     merged per row): range masks, no split, at most one unit per SM
 *   proj_tile_n: the projection's output tile for proj_rows rows of d_model:
 *     256 or 192 (128-row tiles of that width on one SM), 512 (256 x 256
 *     tiles on a pair of SMs), 0 when proj_rows or d_model is 0
 * Pure host arithmetic (no CUDA call). Returns ATTN_ERR_INVALID for
 * non-positive sizes or SM count, an unknown mask kind or CHUNK without a
 * positive chunk_len.
 */
typedef struct {
  int32_t seg_len, tiles_per_seg, q_tiles;
  int32_t kv_splits, kv_tiles_per_split;
  int32_t proj_tile_n;
  int64_t units;
  size_t workspace_bytes;
  int32_t cluster_merge;
  int32_t narrow;
} attn_plan_info;

attn_status attn_debug_plan(int32_t batch, int32_t t_q, int32_t t_kv, int32_t n_heads, int32_t mask_kind,
                            int32_t chunk_len, int32_t num_sms, int64_t proj_rows, int32_t d_model,
                            attn_plan_info *out);

/*
 * attn_debug_timeout_probe -- launches one tiny kernel that waits on a barrier
 * nothing will ever complete, with a limit of limit_ns nanoseconds (1e3..1e9).
 * The kernel gives up, records the timeout in the error word and returns, so
 * the context stays usable. A test of the bounded-wait path, with no fault.
 */
attn_status attn_debug_timeout_probe(int64_t limit_ns, attn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SEA_ATTN_H */
