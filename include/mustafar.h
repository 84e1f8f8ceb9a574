/*
 * mustafar.h - C ABI of the B200 (sm_100a) Mustafar KV-cache library.
 *
 * The method (MUSTAFAR summary, atlas.scime.ai, "Approach"; Mustafar abstract,
 * catalyzex author page): every (token, kv head) vector of the Key and Value
 * caches is pruned by magnitude to an unstructured sparsity, compressed into a
 * bitmap-based sparse format, and decode attention is computed directly over
 * the compressed caches.  New decode tokens are pruned and compressed at run
 * time.  K and V take separate sparsities (Mustafar README, Part II: one
 * sparsity setting for the keys, another for the values).
 *
 * Conventions for every call
 * --------------------------
 * - Every data pointer is a DEVICE pointer unless marked "host".  The caller
 *   owns all memory; the library allocates nothing, never synchronises, and
 *   enqueues its kernels on `stream` (a cudaStream_t; NULL = legacy stream).
 * - fp16 tensors are passed as raw 16-bit storage (IEEE binary16).
 * - head_dim must be 128 for the kernels (the format itself needs a multiple of 32).
 * - Host-side validation failures return an error status and launch nothing.
 *   A failed launch returns MUSTAFAR_ERR_CUDA.  mustafar_last_error() gives a
 *   message for the calling thread's last failure.
 * - Problems only the device can see (a position or length beyond the cache
 *   capacity) never trap: the kernel skips that row and ORs a bit into the
 *   optional device word `d_err` (MUSTAFAR_DEVERR_*).
 *
 * Compressed format (one "stream" per (batch row b, kv head h); s = b*H + h)
 * ---------------------------------------------------------------------------
 *   keep k   = head_dim - floor(sparsity * head_dim), sparsity rounded to float
 *              and the product formed in double; 1 <= k <= head_dim.
 *   selection: the k channels with the largest magnitude key (fp16 bits & 0x7FFF);
 *              on equal keys the lower channel index wins.
 *   bitmap   : uint32 [streams][capacity][head_dim/32]; channel c of token t is
 *              kept iff bit (c % 32) of word (c / 32) is set.  Always popcount k.
 *   values   : fp16 bits [streams][capacity * k]; token t's k kept values, in
 *              ascending channel order, start at element t*k of its stream.
 *   tile_offset: uint32 [streams][capacity/64]; element offset of the first value
 *              of each 64-token tile (the popcount prefix sum, = 64*i*k).
 *   Pruned positions read back as +0.  Bytes per stream:
 *              16*L + 2*k*L + 4*capacity/64 for L stored tokens (head_dim 128).
 *
 * Channel-wise caches (pattern MUSTAFAR_PATTERN_CHANNEL: the channel-wise pruning
 * direction of the README, Part II, K/V [t/c] naming) use the same arrays with the
 * selection turned across tokens: tokens are grouped in windows of 16 from token 0;
 * a full window prunes F = floor(16 * sparsity) tokens of every channel and keeps
 * the 16 - F largest magnitudes (ties: the lower token index wins); a window of
 * n < 16 tokens (the newest ones) prunes floor(n*F/16).  keep is then
 * (head_dim/16) * (16 - F) (mustafar_keep_count_channel): window j of a stream
 * owns the 16*keep elements from j*16*keep, its kept values packed token after
 * token, each token's in ascending channel order, so tokens carry varying counts.
 * A fourth array, window (fp16 [streams][16][head_dim]), holds the dense copy of
 * each stream's newest incomplete window, which an append prunes again.
 */
#ifndef MUSTAFAR_H_
#define MUSTAFAR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MUSTAFAR_ABI_VERSION 5

#if defined(__GNUC__)
#define MUSTAFAR_API __attribute__((visibility("default")))
#else
#define MUSTAFAR_API
#endif

typedef struct CUstream_st *mustafar_stream_t; /* identical to cudaStream_t */

typedef enum {
  MUSTAFAR_OK = 0,
  MUSTAFAR_ERR_INVALID_ARG = 1, /* null pointer, bad shape, bad sparsity, keep mismatch   */
  MUSTAFAR_ERR_UNSUPPORTED = 2, /* valid for the format but not for these kernels (d!=128) */
  MUSTAFAR_ERR_MISALIGNED = 3,  /* a pointer or stride breaks the 16-byte rule            */
  MUSTAFAR_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed            */
  MUSTAFAR_ERR_WORKSPACE = 5    /* workspace missing or smaller than the query returned   */
} mustafar_status;

/* device-side error bits ORed into *d_err (never a trap) */
#define MUSTAFAR_DEVERR_POS_RANGE 0x1u /* append: pos[b] < 0 or >= capacity; row skipped     */
#define MUSTAFAR_DEVERR_LEN_RANGE 0x2u /* decode: seq_len[b] < 0 or > capacity; row clamped  */
#define MUSTAFAR_DEVERR_TIMEOUT 0x4u   /* decode: a staged copy did not land in time; result invalid */

/* One compressed cache (K or V).  The three arrays are caller-owned device
 * memory sized by mustafar_cache_sizes(); bitmap and values 16-byte aligned,
 * tile_offset 4-byte aligned.  capacity is a multiple of 64. */
typedef struct {
  int32_t batch;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t capacity;
  int32_t keep; /* = mustafar_keep_count(head_dim, sparsity); with head_keep: the largest of them */
  uint32_t *bitmap;
  uint16_t *values;
  uint32_t *tile_offset;
  /* HOST array [num_kv_heads] (at most 128 heads), or NULL.  Per-head sparsity (the allocation
   * the MUSTAFAR summary, "Limitations", leaves open): kv head h keeps head_keep[h] channels per
   * token, each in [1, head_dim].  Stream (b, h)'s packed values then start at element
   * capacity * (b * sum_h' head_keep[h'] + sum_{h'<h} head_keep[h']), token t's run at + t*head_keep[h],
   * and its tile offsets are 64*i*head_keep[h].  NULL: every head keeps `keep` (the same layout
   * with all head_keep[h] = keep).  Read at call time only; the library keeps no pointer to it. */
  const int32_t *head_keep;
  /* MUSTAFAR_PATTERN_TOPK: per-token top-keep pruning (the method).  MUSTAFAR_PATTERN_2_4: the
   * 2:4 semi-structured comparison pattern the pages benchmark against (MUSTAFAR summary,
   * "Experimental setup"): every group of 4 consecutive channels keeps its 2 largest magnitudes
   * (ties to the lower channel), so keep must be head_dim/2 and head_keep NULL.  Both are stored in
   * the same bitmap format, and the decode calls read either. */
  int32_t pattern;
  /* MUSTAFAR_PATTERN_CHANNEL caches only (NULL otherwise): fp16 [batch][num_kv_heads][16][head_dim],
   * 16-byte aligned, caller-owned like the other arrays.  Slots 0 .. n-1 hold the n tokens of each
   * stream's newest window when n < 16; mustafar_compress writes them and every append adds one. */
  uint16_t *window;
} mustafar_cache_t;

#define MUSTAFAR_PATTERN_TOPK 0
#define MUSTAFAR_PATTERN_2_4 1
/* channel-wise pruning over 16-token windows; keep = mustafar_keep_count_channel(head_dim, s),
 * head_keep NULL and window non-NULL */
#define MUSTAFAR_PATTERN_CHANNEL 2

/* Keep count for a pruning sparsity s (fraction of channels removed, README
 * Part II: a setting of 0.5 prunes half of them).  Returns head_dim - floor(s*head_dim), or -1
 * when head_dim <= 0, head_dim % 32 != 0 or s is outside [0, 1). */
MUSTAFAR_API int32_t mustafar_keep_count(int32_t head_dim, float sparsity);

/* Values per token slot of a channel-wise cache: (head_dim/16) * (16 - floor(16*s)), s rounded
 * to float and the product formed in double.  -1 when head_dim <= 0, head_dim % 32 != 0 or s is
 * outside [0, 1). */
MUSTAFAR_API int32_t mustafar_keep_count_channel(int32_t head_dim, float sparsity);

/* Bytes of the four arrays of a channel-wise cache (host outputs, any may be NULL): bitmap and
 * tile_offset as mustafar_cache_sizes, values 2*streams*capacity*keep with keep from
 * mustafar_keep_count_channel, window 2*streams*16*head_dim.  Errors: INVALID_ARG. */
MUSTAFAR_API mustafar_status mustafar_cache_sizes_channel(int32_t batch, int32_t num_kv_heads, int32_t head_dim,
                                                          int32_t capacity, float sparsity, size_t *bitmap_bytes,
                                                          size_t *values_bytes, size_t *offset_bytes,
                                                          size_t *window_bytes);

/* Bytes of the three arrays of one cache (host outputs, any may be NULL). */
MUSTAFAR_API mustafar_status mustafar_cache_sizes(int32_t batch, int32_t num_kv_heads, int32_t head_dim,
                                     int32_t capacity, float sparsity, size_t *bitmap_bytes,
                                     size_t *values_bytes, size_t *offset_bytes);

/* As mustafar_cache_sizes for a cache with a keep count per kv head (host array
 * head_keep[num_kv_heads], each in [1, head_dim]): values take 2 * batch * capacity *
 * sum_h head_keep[h] bytes.  Errors: INVALID_ARG. */
MUSTAFAR_API mustafar_status mustafar_cache_sizes_per_head(int32_t batch, int32_t num_kv_heads, int32_t head_dim,
                                                           int32_t capacity, const int32_t *head_keep,
                                                           size_t *bitmap_bytes, size_t *values_bytes,
                                                           size_t *offset_bytes);

/* Prune + compress (prefill).  Per-token magnitude pruning followed by the
 * bitmap compression (MUSTAFAR summary, "Approach"; Mustafar abstract).
 *   x        : fp16 dense cache; element (b, h, t, c) at
 *              x[b*stride_b + h*stride_h + t*stride_t + c] (strides in elements,
 *              channels contiguous; x and every stride a multiple of 8 elements).
 *   L        : tokens [0, L) are compressed into slots [0, L); 0 <= L <= capacity.
 *   sparsity : must satisfy c->keep == mustafar_keep_count(c->head_dim, sparsity) (0.5 for a
 *              2:4 cache; mustafar_keep_count_channel for a channel-wise one); ignored when
 *              c->head_keep is set (each head then keeps c->head_keep[h]).
 * The selection follows c->pattern (per-token top-keep, 2:4, or channel-wise over 16-token
 * windows; a channel-wise compress also copies the tokens of an incomplete last window,
 * [16*floor(L/16), L), into slots 0.. of c->window).
 *   c        : the destination cache; its whole tile_offset array is written.
 *   d_err    : optional device word (unused by this call today; may be NULL).
 * Slots >= L are not touched.  Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, CUDA. */
MUSTAFAR_API mustafar_status mustafar_compress(const void *x, int64_t stride_b, int64_t stride_h,
                                  int64_t stride_t, int32_t L, float sparsity,
                                  const mustafar_cache_t *c, uint32_t *d_err,
                                  mustafar_stream_t stream);

/* Append: prune + compress one new decode token per (b, kv head) into slot
 * pos[b] (the runtime compression the abstract describes).
 *   x     : fp16 [batch][num_kv_heads][head_dim] with element (b, h, c) at
 *           x[b*stride_b + h*stride_h + c] (x and strides multiples of 8 elements).
 *   d_pos : int32 [batch] device array of slots; a slot outside [0, capacity)
 *           skips that row and sets MUSTAFAR_DEVERR_POS_RANGE in *d_err.
 * The caller advances its lengths (e.g. seq_len = pos + 1) itself; the library
 * keeps no state beyond the caches.  A channel-wise cache stores the token in slot
 * pos % 16 of c->window and prunes its window (tokens 16*floor(pos/16) .. pos) again,
 * rewriting those tokens' bitmaps and the window's packed values: appends to a row must
 * come in token order, each after the previous one.
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, CUDA. */
MUSTAFAR_API mustafar_status mustafar_append(const void *x, int64_t stride_b, int64_t stride_h,
                                const int32_t *d_pos, const mustafar_cache_t *c, uint32_t *d_err,
                                mustafar_stream_t stream);

/* Workspace bytes for mustafar_decode_attn / mustafar_decode_step /
 * mustafar_dense_decode_attn with these shapes (enough for any of them).
 * num_splits = 0 asks for the automatic plan; a positive value asks the sparse
 * kernel for about that many CTAs per (b, kv head) stream, and the dense baseline
 * for that many context splits (clamped to the number of 16-token chunks).
 * The workspace holds one ticket counter per (b, kv head) and partial softmax
 * states.  It must be zero-filled once when allocated; every completed call
 * leaves the counters at zero again.  Calls that share a workspace must not overlap. */
MUSTAFAR_API mustafar_status mustafar_decode_workspace_bytes(int32_t batch, int32_t num_q_heads,
                                                int32_t num_kv_heads, int32_t head_dim,
                                                int32_t max_len, int32_t num_splits,
                                                size_t *bytes);

/* Sparse decode attention computed straight from the compressed caches (Mustafar
 * abstract: the method's attention kernel reads the compressed caches directly).
 * For q head hq (kv head g = hq / (Hq/Hkv)) of batch row b:
 *   z_t = scale * q[b,hq] . K~[b,g,t]   for t < seq_len[b]
 *   out[b,hq] = sum_t softmax(z)_t V~[b,g,t]          (fp16, fp32 accumulation)
 *   lse[b,hq] = log sum_t exp(z_t)                    (fp32, natural log; optional)
 *   q, out    : fp16 [batch][num_q_heads][head_dim], 16-byte aligned.
 *   k, v      : compressed caches with equal batch, num_kv_heads, head_dim; their
 *               keep counts (sparsities) may differ.
 *   d_seq_len : int32 [batch]; each in [1, capacity] (longer rows are clamped
 *               and flagged in d_err; 0 gives out = 0 and lse = -inf).
 *   max_len   : the longest row the caller expects; it sizes the work split and the
 *               workspace.  A row longer than it is still attended in full.
 *   workspace : see mustafar_decode_workspace_bytes (same max_len and num_splits).
 *   d_err     : optional device error word.
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA. */
MUSTAFAR_API mustafar_status mustafar_decode_attn(const void *q, int32_t num_q_heads, const mustafar_cache_t *k,
                                     const mustafar_cache_t *v, const int32_t *d_seq_len,
                                     int32_t max_len, float scale, void *out, float *lse,
                                     void *workspace, size_t workspace_bytes, int32_t num_splits,
                                     uint32_t *d_err, mustafar_stream_t stream);

/* One decode step in a single launch: append + attend.  For every (b, kv head) the new
 * token's K and V vectors are pruned and compressed into slot pos[b] of both caches (exactly
 * what mustafar_append writes), then the attention of mustafar_decode_attn runs over the
 * pos[b] + 1 tokens [0, pos[b]] - the new token included (the pages prune and compress at
 * run time: Mustafar abstract).  The CTA that will read the new token's 16-token chunk
 * compresses it first, so no separate append launch is needed; a channel-wise cache is the
 * exception: its append (which prunes the token's whole window again) runs as a launch of its
 * own on the same stream just before the attention (if the attention launch then fails, with
 * MUSTAFAR_ERR_CUDA, that cache already holds the new token).
 *   k_new, v_new : fp16 [batch][num_kv_heads][head_dim], element (b, h, c) at
 *                  k_new[b*k_stride_b + h*k_stride_h + c]; 16-byte aligned, strides multiples of 8.
 *   d_pos        : int32 [batch]; a slot outside [0, capacity) skips the append, sets
 *                  MUSTAFAR_DEVERR_POS_RANGE and clamps the row.
 *   max_len      : the longest pos[b] + 1 the caller expects (sizes the work split and the
 *                  workspace, as in mustafar_decode_attn).
 * Other arguments as in mustafar_decode_attn (same workspace query).
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA. */
MUSTAFAR_API mustafar_status mustafar_decode_step(const void *q, int32_t num_q_heads, const void *k_new,
                                                  int64_t k_stride_b, int64_t k_stride_h, const void *v_new,
                                                  int64_t v_stride_b, int64_t v_stride_h, const int32_t *d_pos,
                                                  const mustafar_cache_t *k, const mustafar_cache_t *v,
                                                  int32_t max_len, float scale, void *out, float *lse,
                                                  void *workspace, size_t workspace_bytes, int32_t num_splits,
                                                  uint32_t *d_err, mustafar_stream_t stream);

/* Dense fp16 decode attention over uncompressed caches, the baseline the pages
 * compare against (dense FlashAttention-style and cuBLAS attention: MUSTAFAR
 * summary, "Experimental setup").  Same math and kernel skeleton as mustafar_decode_attn.
 *   k_dense, v_dense : fp16 [batch][num_kv_heads][capacity][head_dim], 16-byte aligned.
 * Other arguments as in mustafar_decode_attn. */
MUSTAFAR_API mustafar_status mustafar_dense_decode_attn(const void *q, int32_t num_q_heads, const void *k_dense,
                                           const void *v_dense, int32_t batch, int32_t num_kv_heads,
                                           int32_t head_dim, int32_t capacity,
                                           const int32_t *d_seq_len, int32_t max_len, float scale,
                                           void *out, float *lse, void *workspace,
                                           size_t workspace_bytes, int32_t num_splits,
                                           uint32_t *d_err, mustafar_stream_t stream);

/* Bytes of device memory the library reserves (on every GPU that loads it, until the
 * process exits) for mustafar_decode_attn_noalloc's split-K scratch. */
#define MUSTAFAR_NOALLOC_SCRATCH_BYTES (16u << 20)

/* Sparse decode attention that allocates nothing and takes no workspace.
 * The paper has no counterpart to this call: it exists for callers that cannot hand the
 * library a workspace - serving engines that reserve all device memory at start-up and pass
 * kernels only their inputs and outputs, plugin interfaces whose host framework owns the
 * allocator, or code that must not trigger a device allocation.  It computes exactly what
 * mustafar_decode_attn computes (same arguments, minus workspace and workspace_bytes), with
 * the split-K partial states and ticket counters kept in a fixed array of
 * MUSTAFAR_NOALLOC_SCRATCH_BYTES inside the library instead.
 *   - A call whose split plan needs more scratch than that (a very large batch x heads x
 *     num_splits) is rejected with MUSTAFAR_ERR_WORKSPACE and a message.  The automatic plan
 *     (num_splits = 0) needs at most one wave of CTAs (SMs x 4) x 2 partial slots x
 *     (32 + 128 G) x 4 bytes, plus 4 bytes per (batch row, kv head) for the ticket counters:
 *     9.9 MB on a 148-SM B200 at G = 16 q heads per kv head, so it always fits there.
 *   - Every call looks up the array's device address in the current device's context (a host
 *     query; the first one on a device also loads the library's device code there), so make
 *     the first call on each device before any stream capture.
 *   - Every call shares the one array, on every stream: calls that overlap on the GPU race
 *     and corrupt each other's results.  Each call first clears the ticket counters it uses.
 *   - No cudaMalloc, cudaFree or allocating library routine is called.
 * Errors: as mustafar_decode_attn, plus WORKSPACE when the scratch is too small. */
MUSTAFAR_API mustafar_status mustafar_decode_attn_noalloc(const void *q, int32_t num_q_heads,
                                                          const mustafar_cache_t *k,
                                                          const mustafar_cache_t *v,
                                                          const int32_t *d_seq_len, int32_t max_len,
                                                          float scale, void *out, float *lse,
                                                          int32_t num_splits, uint32_t *d_err,
                                                          mustafar_stream_t stream);

/* The split count the automatic plan would use for this call (host query, for
 * benchmarks and tests).  Returns a value >= 1, or -1 on invalid shapes. */
MUSTAFAR_API int32_t mustafar_decode_plan_splits(int32_t batch, int32_t num_kv_heads, int32_t head_dim,
                                    int32_t max_len, int32_t keep_k, int32_t keep_v, int32_t dense);

/* How the automatic plan of mustafar_decode_attn merges the split-K partials of a pair of
 * uniform token-wise caches (host query, for benchmarks and tests; num_splits = 0).  When the
 * plan gives every (batch row, kv head) stream the same number C of CTAs and all B * Hkv
 * clusters of C CTAs fit on the device at once, each stream's CTAs run as one thread-block
 * cluster and merge in distributed shared memory: the call returns C (2..16).  It returns 0 when
 * the partials go through the workspace and a per-stream ticket instead (one CTA per stream, or
 * CTAs per stream not whole, above 16 or not all resident), and -1 on invalid shapes.  Both
 * merges compute the same log-sum-exp combination of the same partials. */
MUSTAFAR_API int32_t mustafar_decode_plan_cluster(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                                  int32_t head_dim, int32_t max_len, int32_t keep_k,
                                                  int32_t keep_v);

MUSTAFAR_API const char *mustafar_status_string(mustafar_status s);
MUSTAFAR_API const char *mustafar_last_error(void);
MUSTAFAR_API int32_t mustafar_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MUSTAFAR_H_ */
