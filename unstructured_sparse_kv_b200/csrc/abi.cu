// abi.cu - the extern "C" entry points declared in include/mustafar.h: argument
// validation, split planning and kernel launches.  No allocation, no synchronisation.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "common.cuh"
#include "internal.h"

namespace mustafar {
namespace {

thread_local std::string g_last_error;

mustafar_status fail(mustafar_status s, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
mustafar_status fail(mustafar_status s, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

mustafar_status cuda_fail(cudaError_t e, const char *where) {
  return fail(MUSTAFAR_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int32_t keep_count(int32_t d, float s) {
  if (d <= 0 || d % 32 != 0) return -1;
  if (!(s >= 0.0f && s < 1.0f)) return -1;  // also rejects NaN
  const double pruned = std::floor(static_cast<double>(s) * static_cast<double>(d));
  return d - static_cast<int32_t>(pruned);
}

// Values per token slot of a channel-wise cache: (d/16) * (16 - floor(16 s)).
int32_t keep_count_channel(int32_t d, float s) {
  if (d <= 0 || d % 32 != 0) return -1;
  if (!(s >= 0.0f && s < 1.0f)) return -1;
  const int32_t F = static_cast<int32_t>(std::floor(static_cast<double>(s) * kWindowTokens));
  return (d / kWindowTokens) * (kWindowTokens - F);
}

// The prune count F of a full window of a checked channel-wise cache (keep = (d/16) * (16 - F)).
int channel_prune_count(const mustafar_cache_t *c) { return kWindowTokens - c->keep / (c->head_dim / kWindowTokens); }

mustafar_status check_cache(const mustafar_cache_t *c, const char *name) {
  if (c == nullptr) return fail(MUSTAFAR_ERR_INVALID_ARG, "%s: cache descriptor is NULL", name);
  if (c->batch <= 0 || c->num_kv_heads <= 0 || c->capacity <= 0)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "%s: batch, num_kv_heads and capacity must be positive", name);
  if (c->head_dim <= 0 || c->head_dim % 32 != 0)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "%s: head_dim must be a positive multiple of 32", name);
  if (c->head_dim != kHeadDim)
    return fail(MUSTAFAR_ERR_UNSUPPORTED, "%s: kernels are built for head_dim 128 (got %d)", name, c->head_dim);
  if (c->capacity % kTileTokens != 0)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "%s: capacity must be a multiple of 64 (got %d)", name, c->capacity);
  if (c->keep < 1 || c->keep > c->head_dim)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "%s: keep must lie in [1, head_dim] (got %d)", name, c->keep);
  if (c->pattern != MUSTAFAR_PATTERN_TOPK && c->pattern != MUSTAFAR_PATTERN_2_4 &&
      c->pattern != MUSTAFAR_PATTERN_CHANNEL)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "%s: pattern must be MUSTAFAR_PATTERN_TOPK, _2_4 or _CHANNEL (got %d)", name,
                c->pattern);
  if (c->pattern == MUSTAFAR_PATTERN_CHANNEL) {
    if (c->keep % (c->head_dim / kWindowTokens) != 0 || c->head_keep != nullptr)
      return fail(MUSTAFAR_ERR_INVALID_ARG,
                  "%s: a channel-wise cache keeps a multiple of head_dim/16 values per token and has no head_keep",
                  name);
    if (c->window == nullptr) return fail(MUSTAFAR_ERR_INVALID_ARG, "%s: a channel-wise cache needs its window array", name);
    if (!aligned(c->window, 16)) return fail(MUSTAFAR_ERR_MISALIGNED, "%s: window needs 16-byte alignment", name);
  }
  if (c->pattern == MUSTAFAR_PATTERN_2_4 && (c->keep != c->head_dim / 2 || c->head_keep != nullptr))
    return fail(MUSTAFAR_ERR_INVALID_ARG, "%s: a 2:4 cache keeps head_dim/2 channels and has no head_keep", name);
  if (c->head_keep != nullptr) {
    if (c->num_kv_heads > kMaxKvHeads)
      return fail(MUSTAFAR_ERR_UNSUPPORTED, "%s: per-head keep supports at most %d kv heads", name, kMaxKvHeads);
    int32_t kmax = 0;
    for (int h = 0; h < c->num_kv_heads; ++h) {
      if (c->head_keep[h] < 1 || c->head_keep[h] > c->head_dim)
        return fail(MUSTAFAR_ERR_INVALID_ARG, "%s: head_keep[%d] = %d outside [1, head_dim]", name, h, c->head_keep[h]);
      kmax = c->head_keep[h] > kmax ? c->head_keep[h] : kmax;
    }
    if (kmax != c->keep)
      return fail(MUSTAFAR_ERR_INVALID_ARG, "%s: keep must be the largest head_keep (%d), got %d", name, kmax, c->keep);
  } else if (c->num_kv_heads > kMaxKvHeads) {
    return fail(MUSTAFAR_ERR_UNSUPPORTED, "%s: at most %d kv heads", name, kMaxKvHeads);
  }
  if (static_cast<int64_t>(c->capacity) * c->keep >= (int64_t(1) << 32))
    return fail(MUSTAFAR_ERR_INVALID_ARG, "%s: capacity*keep must stay below 2^32 (32-bit tile offsets)", name);
  if (c->bitmap == nullptr || c->values == nullptr || c->tile_offset == nullptr)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "%s: bitmap, values and tile_offset must be non-NULL", name);
  if (!aligned(c->bitmap, 16) || !aligned(c->values, 16) || !aligned(c->tile_offset, 4))
    return fail(MUSTAFAR_ERR_MISALIGNED, "%s: bitmap/values need 16-byte, tile_offset 4-byte alignment", name);
  return MUSTAFAR_OK;
}

}  // namespace

void set_last_error(const char *msg) { g_last_error = msg; }

cudaError_t ensure_smem_limit(const void *kernel, int slot, int bytes) {
  static int done[64][kKernelSlots];  // bytes already granted per (device, kernel slot)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || slot < 0 || slot >= kKernelSlots)
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (done[dev][slot] >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done[dev][slot] = bytes;
  return e;
}

}  // namespace mustafar

using namespace mustafar;

extern "C" {

int32_t mustafar_abi_version(void) { return MUSTAFAR_ABI_VERSION; }

const char *mustafar_status_string(mustafar_status s) {
  switch (s) {
    case MUSTAFAR_OK: return "ok";
    case MUSTAFAR_ERR_INVALID_ARG: return "invalid argument";
    case MUSTAFAR_ERR_UNSUPPORTED: return "unsupported";
    case MUSTAFAR_ERR_MISALIGNED: return "misaligned pointer or stride";
    case MUSTAFAR_ERR_CUDA: return "CUDA error";
    case MUSTAFAR_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

const char *mustafar_last_error(void) { return g_last_error.c_str(); }

// Keep counts and value placement of every head of a checked cache.
static HeadKeep head_keep_of(const mustafar_cache_t *c) {
  HeadKeep hk;
  hk.pre[0] = 0;
  for (int h = 0; h < c->num_kv_heads; ++h) {
    hk.k[h] = c->head_keep != nullptr ? c->head_keep[h] : c->keep;
    hk.pre[h + 1] = hk.pre[h] + hk.k[h];
  }
  for (int h = c->num_kv_heads; h < kMaxKvHeads; ++h) {
    hk.k[h] = 0;
    hk.pre[h + 1] = hk.pre[h];
  }
  return hk;
}

int32_t mustafar_keep_count(int32_t head_dim, float sparsity) { return keep_count(head_dim, sparsity); }

int32_t mustafar_keep_count_channel(int32_t head_dim, float sparsity) { return keep_count_channel(head_dim, sparsity); }

mustafar_status mustafar_cache_sizes_channel(int32_t batch, int32_t num_kv_heads, int32_t head_dim, int32_t capacity,
                                             float sparsity, size_t *bitmap_bytes, size_t *values_bytes,
                                             size_t *offset_bytes, size_t *window_bytes) {
  const int32_t k = keep_count_channel(head_dim, sparsity);
  if (k < 0)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "cache_sizes_channel: head_dim %% 32 != 0 or sparsity outside [0,1)");
  if (batch <= 0 || num_kv_heads <= 0 || capacity <= 0 || capacity % kTileTokens != 0)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "cache_sizes_channel: positive shapes and capacity %% 64 == 0 required");
  const size_t streams = static_cast<size_t>(batch) * num_kv_heads;
  if (bitmap_bytes) *bitmap_bytes = streams * capacity * (head_dim / 8);
  if (values_bytes) *values_bytes = streams * capacity * static_cast<size_t>(k) * 2;
  if (offset_bytes) *offset_bytes = streams * (capacity / kTileTokens) * 4;
  if (window_bytes) *window_bytes = streams * kWindowTokens * static_cast<size_t>(head_dim) * 2;
  return MUSTAFAR_OK;
}

mustafar_status mustafar_cache_sizes(int32_t batch, int32_t num_kv_heads, int32_t head_dim, int32_t capacity,
                                     float sparsity, size_t *bitmap_bytes, size_t *values_bytes,
                                     size_t *offset_bytes) {
  const int32_t k = keep_count(head_dim, sparsity);
  if (k < 0) return fail(MUSTAFAR_ERR_INVALID_ARG, "cache_sizes: head_dim %% 32 != 0 or sparsity outside [0,1)");
  if (batch <= 0 || num_kv_heads <= 0 || capacity <= 0 || capacity % kTileTokens != 0)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "cache_sizes: positive shapes and capacity %% 64 == 0 required");
  const size_t streams = static_cast<size_t>(batch) * num_kv_heads;
  if (bitmap_bytes) *bitmap_bytes = streams * capacity * (head_dim / 8);
  if (values_bytes) *values_bytes = streams * capacity * static_cast<size_t>(k) * 2;
  if (offset_bytes) *offset_bytes = streams * (capacity / kTileTokens) * 4;
  return MUSTAFAR_OK;
}

mustafar_status mustafar_cache_sizes_per_head(int32_t batch, int32_t num_kv_heads, int32_t head_dim,
                                              int32_t capacity, const int32_t *head_keep, size_t *bitmap_bytes,
                                              size_t *values_bytes, size_t *offset_bytes) {
  if (head_keep == nullptr) return fail(MUSTAFAR_ERR_INVALID_ARG, "cache_sizes_per_head: head_keep is NULL");
  if (head_dim <= 0 || head_dim % 32 != 0)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "cache_sizes_per_head: head_dim must be a positive multiple of 32");
  if (batch <= 0 || num_kv_heads <= 0 || capacity <= 0 || capacity % kTileTokens != 0)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "cache_sizes_per_head: positive shapes and capacity %% 64 == 0 required");
  size_t ksum = 0;
  for (int h = 0; h < num_kv_heads; ++h) {
    if (head_keep[h] < 1 || head_keep[h] > head_dim)
      return fail(MUSTAFAR_ERR_INVALID_ARG, "cache_sizes_per_head: head_keep[%d] = %d outside [1, head_dim]", h,
                  head_keep[h]);
    ksum += static_cast<size_t>(head_keep[h]);
  }
  const size_t streams = static_cast<size_t>(batch) * num_kv_heads;
  if (bitmap_bytes) *bitmap_bytes = streams * capacity * (head_dim / 8);
  if (values_bytes) *values_bytes = static_cast<size_t>(batch) * capacity * ksum * 2;
  if (offset_bytes) *offset_bytes = streams * (capacity / kTileTokens) * 4;
  return MUSTAFAR_OK;
}

mustafar_status mustafar_compress(const void *x, int64_t stride_b, int64_t stride_h, int64_t stride_t, int32_t L,
                                  float sparsity, const mustafar_cache_t *c, uint32_t *d_err,
                                  mustafar_stream_t stream) {
  (void)d_err;
  mustafar_status s = check_cache(c, "compress");
  if (s != MUSTAFAR_OK) return s;
  if (c->head_keep == nullptr) {
    const bool chan = c->pattern == MUSTAFAR_PATTERN_CHANNEL;
    const int32_t k = chan ? keep_count_channel(c->head_dim, sparsity) : keep_count(c->head_dim, sparsity);
    if (k < 0) return fail(MUSTAFAR_ERR_INVALID_ARG, "compress: sparsity must lie in [0, 1)");
    if (k != c->keep)
      return fail(MUSTAFAR_ERR_INVALID_ARG, "compress: cache keep %d != %s(%d, %g) = %d", c->keep,
                  chan ? "keep_count_channel" : "keep_count", c->head_dim, static_cast<double>(sparsity), k);
  }
  if (L < 0 || L > c->capacity) return fail(MUSTAFAR_ERR_INVALID_ARG, "compress: L must lie in [0, capacity]");
  if (x == nullptr && L > 0) return fail(MUSTAFAR_ERR_INVALID_ARG, "compress: x is NULL");
  if (L > 0) {
    if (!aligned(x, 16) || stride_b % 8 != 0 || stride_h % 8 != 0 || stride_t % 8 != 0)
      return fail(MUSTAFAR_ERR_MISALIGNED, "compress: x and its strides must be multiples of 8 elements");
    if (stride_b < 0 || stride_h < 0 || stride_t < 0)
      return fail(MUSTAFAR_ERR_INVALID_ARG, "compress: negative strides are not supported");
  }
  cudaError_t e = launch_compress(static_cast<const uint16_t *>(x), stride_b, stride_h, stride_t, L, c->batch,
                                  c->num_kv_heads, head_keep_of(c), c->keep, c->capacity, c->bitmap, c->values,
                                  c->tile_offset, static_cast<Pattern>(c->pattern), c->window,
                                  c->pattern == MUSTAFAR_PATTERN_CHANNEL ? channel_prune_count(c) : 0,
                                  reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MUSTAFAR_OK : cuda_fail(e, "compress launch");
}

mustafar_status mustafar_append(const void *x, int64_t stride_b, int64_t stride_h, const int32_t *d_pos,
                                const mustafar_cache_t *c, uint32_t *d_err, mustafar_stream_t stream) {
  mustafar_status s = check_cache(c, "append");
  if (s != MUSTAFAR_OK) return s;
  if (x == nullptr || d_pos == nullptr) return fail(MUSTAFAR_ERR_INVALID_ARG, "append: x and pos must be non-NULL");
  if (!aligned(x, 16) || stride_b % 8 != 0 || stride_h % 8 != 0)
    return fail(MUSTAFAR_ERR_MISALIGNED, "append: x and its strides must be multiples of 8 elements");
  if (stride_b < 0 || stride_h < 0) return fail(MUSTAFAR_ERR_INVALID_ARG, "append: negative strides");
  if (!aligned(d_pos, 4)) return fail(MUSTAFAR_ERR_MISALIGNED, "append: pos must be 4-byte aligned");
  cudaError_t e = launch_append(static_cast<const uint16_t *>(x), stride_b, stride_h, d_pos, c->batch,
                                c->num_kv_heads, head_keep_of(c), c->capacity, c->bitmap, c->values, d_err,
                                static_cast<Pattern>(c->pattern), c->window,
                                c->pattern == MUSTAFAR_PATTERN_CHANNEL ? channel_prune_count(c) : 0,
                                reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MUSTAFAR_OK : cuda_fail(e, "append launch");
}

mustafar_status mustafar_decode_workspace_bytes(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                                int32_t head_dim, int32_t max_len, int32_t num_splits,
                                                size_t *bytes) {
  if (bytes == nullptr) return fail(MUSTAFAR_ERR_INVALID_ARG, "workspace_bytes: bytes is NULL");
  if (batch <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_len <= 0 || num_splits < 0)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "workspace_bytes: shapes must be positive, num_splits >= 0");
  if (num_q_heads % num_kv_heads != 0) return fail(MUSTAFAR_ERR_INVALID_ARG, "workspace_bytes: Hq %% Hkv != 0");
  if (head_dim != kHeadDim) return fail(MUSTAFAR_ERR_UNSUPPORTED, "workspace_bytes: head_dim must be 128");
  const int nch = (max_len + kChunk - 1) / kChunk;
  int splits = num_splits > 0 ? (num_splits < nch ? num_splits : nch) : decode_split_bound(batch, num_kv_heads, max_len);
  // enough for the dense baseline's split-K and for the sparse kernel's partial slots
  const size_t dense = decode_workspace_bytes(batch, num_q_heads, num_kv_heads, splits);
  const size_t sparse =
      sparse_workspace_bound(batch, num_kv_heads, num_q_heads / num_kv_heads, max_len, num_splits);
  *bytes = dense > sparse ? dense : sparse;
  return MUSTAFAR_OK;
}

int32_t mustafar_decode_plan_splits(int32_t batch, int32_t num_kv_heads, int32_t head_dim, int32_t max_len,
                                    int32_t keep_k, int32_t keep_v, int32_t dense) {
  if (batch <= 0 || num_kv_heads <= 0 || head_dim != kHeadDim || max_len <= 0) return -1;
  if (!dense && (keep_k < 1 || keep_k > kHeadDim || keep_v < 1 || keep_v > kHeadDim)) return -1;
  DecodePlan plan;
  if (dense) {
    if (plan_dense(batch, num_kv_heads, 4, max_len, 0, &plan) != cudaSuccess) return -1;
    return plan.splits;
  }
  // the sparse kernel cuts the end-to-end chunk sequence into CTA ranges; report the CTAs per stream
  if (plan_sparse(batch, num_kv_heads, 4, max_len, keep_k, keep_v, 0, 0, &plan) != cudaSuccess) return -1;
  const int streams = batch * num_kv_heads;
  return (plan.splits + streams - 1) / streams;
}

int32_t mustafar_decode_plan_cluster(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                     int32_t max_len, int32_t keep_k, int32_t keep_v) {
  if (batch <= 0 || num_kv_heads <= 0 || num_q_heads <= 0 || num_q_heads % num_kv_heads != 0 ||
      head_dim != kHeadDim || max_len <= 0 || keep_k < 1 || keep_k > kHeadDim || keep_v < 1 || keep_v > kHeadDim)
    return -1;
  const int G = num_q_heads / num_kv_heads;
  if (G > 16 || (G & (G - 1)) != 0) return -1;
  DecodePlan plan;
  if (plan_sparse(batch, num_kv_heads, G, max_len, keep_k, keep_v, 0, 0, &plan) != cudaSuccess) return -1;
  return plan.clu;
}

namespace {

mustafar_status run_sparse(DecodeParams &p, int max_len, int num_splits, void *workspace, size_t workspace_bytes,
                           const char *name, cudaStream_t stream) {
  DecodePlan plan;
  const bool chan = p.kwin != nullptr || p.vwin != nullptr;
  if (chan && p.perhead)
    return fail(MUSTAFAR_ERR_UNSUPPORTED, "%s: a channel-wise cache cannot be paired with a per-head cache", name);
  const int variant = chan ? 3 : p.perhead ? 1 : (p.p24_k && p.p24_v ? 2 : 0);
  cudaError_t e = plan_sparse(p.B, p.Hkv, p.G, max_len, p.keep_k, p.keep_v, num_splits, variant, &plan);
  if (e != cudaSuccess) return cuda_fail(e, name);
  p.stage_bytes = plan.stage_bytes;
  p.warp_bytes = plan.warp_bytes;
  p.lg_k = plan.lg_k;
  p.lg_v = plan.lg_v;
  p.skew_k = plan.skew_k;
  p.skew_v = plan.skew_v;
  p.clu = plan.clu;
  const size_t need = sparse_workspace_bytes(p.B, p.Hkv, p.G, plan.splits);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(MUSTAFAR_ERR_WORKSPACE, "%s: workspace of %zu bytes needed (%d CTAs), got %zu", name, need,
                plan.splits, workspace == nullptr ? size_t(0) : workspace_bytes);
  if (!aligned(workspace, 256)) return fail(MUSTAFAR_ERR_MISALIGNED, "%s: workspace must be 256-byte aligned", name);
  uint8_t *w = static_cast<uint8_t *>(workspace);
  const size_t cnt = ((static_cast<size_t>(p.B) * p.Hkv * 4 + 255) / 256) * 256;
  p.ws_cnt = reinterpret_cast<uint32_t *>(w);
  p.ws_part = reinterpret_cast<float *>(w + cnt);
  if (p.pos != nullptr && (p.kwin != nullptr || p.vwin != nullptr)) {
    // a decode step: the channel-wise caches take their new token in one launch of their own before
    // the attention (each newest window is pruned again); the attention kernel appends the rest
    ChannelAppend c[2];
    int n = 0;
    if (p.kwin != nullptr)
      c[n++] = ChannelAppend{p.kn, p.kn_sb, p.kn_sh, p.keep_k, p.chF_k, p.cap_k, const_cast<uint32_t *>(p.kbm),
                             const_cast<uint16_t *>(p.kval), p.kwin};
    if (p.vwin != nullptr)
      c[n++] = ChannelAppend{p.vn, p.vn_sb, p.vn_sh, p.keep_v, p.chF_v, p.cap_v, const_cast<uint32_t *>(p.vbm),
                             const_cast<uint16_t *>(p.vval), p.vwin};
    e = launch_append_channel(c, n, p.pos, p.B, p.Hkv, p.err, stream);
    if (e != cudaSuccess) return cuda_fail(e, name);
  }
  e = launch_sparse(p, plan, stream);
  return e == cudaSuccess ? MUSTAFAR_OK : cuda_fail(e, name);
}

mustafar_status run_decode(bool sparse, DecodeParams &p, int max_len, int num_splits, void *workspace,
                           size_t workspace_bytes, const char *name, cudaStream_t stream) {
  if (sparse) return run_sparse(p, max_len, num_splits, workspace, workspace_bytes, name, stream);
  DecodePlan plan;
  cudaError_t e = plan_dense(p.B, p.Hkv, p.G, max_len, num_splits, &plan);
  if (e != cudaSuccess) return cuda_fail(e, name);
  p.num_splits = plan.splits;
  p.chunks_per_split = plan.chunks_per_split;
  p.stage_bytes = plan.stage_bytes;
  p.warp_bytes = plan.warp_bytes;
  if (plan.splits > 1) {
    const size_t need = decode_workspace_bytes(p.B, p.Hq, p.Hkv, plan.splits);
    if (workspace == nullptr || workspace_bytes < need)
      return fail(MUSTAFAR_ERR_WORKSPACE, "%s: workspace of %zu bytes needed (%d splits), got %zu", name, need,
                  plan.splits, workspace == nullptr ? size_t(0) : workspace_bytes);
    if (!aligned(workspace, 256)) return fail(MUSTAFAR_ERR_MISALIGNED, "%s: workspace must be 256-byte aligned", name);
    uint8_t *w = static_cast<uint8_t *>(workspace);
    const size_t cnt = ((static_cast<size_t>(p.B) * p.Hkv * 4 + 255) / 256) * 256;
    const size_t ml = ((static_cast<size_t>(p.B) * p.Hq * plan.splits * 2 * 4 + 255) / 256) * 256;
    p.ws_cnt = reinterpret_cast<uint32_t *>(w);
    p.ws_ml = reinterpret_cast<float *>(w + cnt);
    p.ws_o = reinterpret_cast<float *>(w + cnt + ml);
  }
  e = launch_dense(p, plan, stream);
  return e == cudaSuccess ? MUSTAFAR_OK : cuda_fail(e, name);
}

// Channel-wise caches of a decode call: their window copies and full-window prune counts.
void set_channel(DecodeParams &p, const mustafar_cache_t *k, const mustafar_cache_t *v) {
  const bool ck = k->pattern == MUSTAFAR_PATTERN_CHANNEL, cv = v->pattern == MUSTAFAR_PATTERN_CHANNEL;
  p.kwin = ck ? k->window : nullptr;
  p.vwin = cv ? v->window : nullptr;
  p.chF_k = ck ? channel_prune_count(k) : 0;
  p.chF_v = cv ? channel_prune_count(v) : 0;
}

mustafar_status check_decode_common(const void *q, int32_t Hq, int32_t B, int32_t Hkv, const int32_t *d_seq_len,
                                    int32_t max_len, float scale, const void *out, const float *lse,
                                    const char *name, const char *len_name = "seq_len") {
  if (q == nullptr || out == nullptr || d_seq_len == nullptr)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "%s: q, out and %s must be non-NULL", name, len_name);
  if (Hq <= 0 || Hq % Hkv != 0) return fail(MUSTAFAR_ERR_INVALID_ARG, "%s: num_q_heads must be a multiple of num_kv_heads", name);
  if (Hq / Hkv > 16) return fail(MUSTAFAR_ERR_UNSUPPORTED, "%s: at most 16 q heads per kv head", name);
  if (max_len <= 0) return fail(MUSTAFAR_ERR_INVALID_ARG, "%s: max_len must be positive", name);
  if (!std::isfinite(scale)) return fail(MUSTAFAR_ERR_INVALID_ARG, "%s: scale must be finite", name);
  if (!aligned(q, 16) || !aligned(out, 16)) return fail(MUSTAFAR_ERR_MISALIGNED, "%s: q and out need 16-byte alignment", name);
  if (lse != nullptr && !aligned(lse, 4)) return fail(MUSTAFAR_ERR_MISALIGNED, "%s: lse needs 4-byte alignment", name);
  if (!aligned(d_seq_len, 4)) return fail(MUSTAFAR_ERR_MISALIGNED, "%s: %s needs 4-byte alignment", name, len_name);
  (void)B;
  return MUSTAFAR_OK;
}

}  // namespace

mustafar_status mustafar_decode_attn(const void *q, int32_t num_q_heads, const mustafar_cache_t *k,
                                     const mustafar_cache_t *v, const int32_t *d_seq_len, int32_t max_len,
                                     float scale, void *out, float *lse, void *workspace, size_t workspace_bytes,
                                     int32_t num_splits, uint32_t *d_err, mustafar_stream_t stream) {
  mustafar_status s = check_cache(k, "decode_attn(k)");
  if (s != MUSTAFAR_OK) return s;
  s = check_cache(v, "decode_attn(v)");
  if (s != MUSTAFAR_OK) return s;
  if (k->batch != v->batch || k->num_kv_heads != v->num_kv_heads || k->head_dim != v->head_dim)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "decode_attn: K and V caches disagree on batch/heads/head_dim");
  s = check_decode_common(q, num_q_heads, k->batch, k->num_kv_heads, d_seq_len, max_len, scale, out, lse,
                          "decode_attn");
  if (s != MUSTAFAR_OK) return s;
  if (num_splits < 0) return fail(MUSTAFAR_ERR_INVALID_ARG, "decode_attn: num_splits must be >= 0");
  DecodeParams p{};
  p.q = static_cast<const uint16_t *>(q);
  p.kbm = k->bitmap;
  p.kval = k->values;
  p.vbm = v->bitmap;
  p.vval = v->values;
  p.keep_k = k->keep;
  p.keep_v = v->keep;
  p.hk_k = head_keep_of(k);
  p.hk_v = head_keep_of(v);
  p.perhead = k->head_keep != nullptr || v->head_keep != nullptr;
  p.p24_k = k->pattern == MUSTAFAR_PATTERN_2_4;
  p.p24_v = v->pattern == MUSTAFAR_PATTERN_2_4;
  set_channel(p, k, v);
  p.cap_k = k->capacity;
  p.cap_v = v->capacity;
  p.seq_len = d_seq_len;
  p.B = k->batch;
  p.Hq = num_q_heads;
  p.Hkv = k->num_kv_heads;
  p.G = num_q_heads / k->num_kv_heads;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.out = static_cast<uint16_t *>(out);
  p.lse = lse;
  p.err = d_err;
  return run_decode(true, p, max_len, num_splits, workspace, workspace_bytes, "decode_attn",
                    reinterpret_cast<cudaStream_t>(stream));
}

mustafar_status mustafar_decode_step(const void *q, int32_t num_q_heads, const void *k_new, int64_t k_stride_b,
                                     int64_t k_stride_h, const void *v_new, int64_t v_stride_b, int64_t v_stride_h,
                                     const int32_t *d_pos, const mustafar_cache_t *k, const mustafar_cache_t *v,
                                     int32_t max_len, float scale, void *out, float *lse, void *workspace,
                                     size_t workspace_bytes, int32_t num_splits, uint32_t *d_err,
                                     mustafar_stream_t stream) {
  mustafar_status s = check_cache(k, "decode_step(k)");
  if (s != MUSTAFAR_OK) return s;
  s = check_cache(v, "decode_step(v)");
  if (s != MUSTAFAR_OK) return s;
  if (k->batch != v->batch || k->num_kv_heads != v->num_kv_heads || k->head_dim != v->head_dim)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "decode_step: K and V caches disagree on batch/heads/head_dim");
  s = check_decode_common(q, num_q_heads, k->batch, k->num_kv_heads, d_pos, max_len, scale, out, lse,
                          "decode_step", "pos");
  if (s != MUSTAFAR_OK) return s;
  if (num_splits < 0) return fail(MUSTAFAR_ERR_INVALID_ARG, "decode_step: num_splits must be >= 0");
  if (k_new == nullptr || v_new == nullptr)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "decode_step: k_new and v_new must be non-NULL");
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || k_stride_b % 8 != 0 || k_stride_h % 8 != 0 ||
      v_stride_b % 8 != 0 || v_stride_h % 8 != 0)
    return fail(MUSTAFAR_ERR_MISALIGNED, "decode_step: k_new, v_new and their strides must be multiples of 8 elements");
  if (k_stride_b < 0 || k_stride_h < 0 || v_stride_b < 0 || v_stride_h < 0)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "decode_step: negative strides are not supported");
  DecodeParams p{};
  p.q = static_cast<const uint16_t *>(q);
  p.kbm = k->bitmap;
  p.kval = k->values;
  p.vbm = v->bitmap;
  p.vval = v->values;
  p.keep_k = k->keep;
  p.keep_v = v->keep;
  p.hk_k = head_keep_of(k);
  p.hk_v = head_keep_of(v);
  p.perhead = k->head_keep != nullptr || v->head_keep != nullptr;
  p.p24_k = k->pattern == MUSTAFAR_PATTERN_2_4;
  p.p24_v = v->pattern == MUSTAFAR_PATTERN_2_4;
  set_channel(p, k, v);
  p.cap_k = k->capacity;
  p.cap_v = v->capacity;
  p.B = k->batch;
  p.Hq = num_q_heads;
  p.Hkv = k->num_kv_heads;
  p.G = num_q_heads / k->num_kv_heads;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.out = static_cast<uint16_t *>(out);
  p.lse = lse;
  p.err = d_err;
  p.pos = d_pos;
  p.kn = static_cast<const uint16_t *>(k_new);
  p.vn = static_cast<const uint16_t *>(v_new);
  p.kn_sb = k_stride_b;
  p.kn_sh = k_stride_h;
  p.vn_sb = v_stride_b;
  p.vn_sh = v_stride_h;
  return run_decode(true, p, max_len, num_splits, workspace, workspace_bytes, "decode_step",
                    reinterpret_cast<cudaStream_t>(stream));
}

mustafar_status mustafar_dense_decode_attn(const void *q, int32_t num_q_heads, const void *k_dense,
                                           const void *v_dense, int32_t batch, int32_t num_kv_heads,
                                           int32_t head_dim, int32_t capacity, const int32_t *d_seq_len,
                                           int32_t max_len, float scale, void *out, float *lse, void *workspace,
                                           size_t workspace_bytes, int32_t num_splits, uint32_t *d_err,
                                           mustafar_stream_t stream) {
  if (k_dense == nullptr || v_dense == nullptr)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "dense_decode_attn: k_dense and v_dense must be non-NULL");
  if (batch <= 0 || num_kv_heads <= 0 || capacity <= 0)
    return fail(MUSTAFAR_ERR_INVALID_ARG, "dense_decode_attn: shapes must be positive");
  if (head_dim != kHeadDim) return fail(MUSTAFAR_ERR_UNSUPPORTED, "dense_decode_attn: head_dim must be 128");
  if (capacity % kChunk != 0) return fail(MUSTAFAR_ERR_INVALID_ARG, "dense_decode_attn: capacity must be a multiple of 16");
  if (!aligned(k_dense, 16) || !aligned(v_dense, 16))
    return fail(MUSTAFAR_ERR_MISALIGNED, "dense_decode_attn: caches need 16-byte alignment");
  mustafar_status s = check_decode_common(q, num_q_heads, batch, num_kv_heads, d_seq_len, max_len, scale, out, lse,
                                          "dense_decode_attn");
  if (s != MUSTAFAR_OK) return s;
  if (num_splits < 0) return fail(MUSTAFAR_ERR_INVALID_ARG, "dense_decode_attn: num_splits must be >= 0");
  DecodeParams p{};
  p.q = static_cast<const uint16_t *>(q);
  p.kd = static_cast<const uint16_t *>(k_dense);
  p.vd = static_cast<const uint16_t *>(v_dense);
  p.cap_k = p.cap_v = capacity;
  p.keep_k = p.keep_v = kHeadDim;
  p.seq_len = d_seq_len;
  p.B = batch;
  p.Hq = num_q_heads;
  p.Hkv = num_kv_heads;
  p.G = num_q_heads / num_kv_heads;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.out = static_cast<uint16_t *>(out);
  p.lse = lse;
  p.err = d_err;
  return run_decode(false, p, max_len, num_splits, workspace, workspace_bytes, "dense_decode_attn",
                    reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
