// internal.h - declarations shared by the library's translation units (not part of the ABI).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "mustafar.h"

namespace mustafar {

// Record the message mustafar_last_error() returns on this thread.
void set_last_error(const char *msg);

// Set a kernel's dynamic shared-memory limit once per device; `slot` (< kKernelSlots) names the
// kernel in the per-device caches.
constexpr int kKernelSlots = 48;
cudaError_t ensure_smem_limit(const void *kernel, int slot, int bytes);

// Keep count of every kv head of one cache, and where each stream's packed values start: stream
// (b, h) keeps k[h] values per token, and its values begin at element cap*(b*pre[H] + pre[h]),
// pre being the prefix sums of k.  A uniform cache has k[h] = keep for every head.  Passed to the
// kernels by value.
constexpr int kMaxKvHeads = 128;
struct HeadKeep {
  int32_t k[kMaxKvHeads];
  int32_t pre[kMaxKvHeads + 1];
  __host__ __device__ __forceinline__ int64_t value_base(int b, int h, int H, int cap) const {
    return static_cast<int64_t>(cap) * (static_cast<int64_t>(b) * pre[H] + pre[h]);
  }
};

// Selection rule of a cache (mustafar_cache_t::pattern).
enum class Pattern { kTopK = 0, k24 = 1, kChannel = 2 };

// Tokens a window of n tokens keeps in every channel of a channel-wise cache, F being the prune
// count of a full 16-token window.
__host__ __device__ __forceinline__ int window_keep(int n, int F) { return n - (n * F) / 16; }

// window (channel-wise caches): fp16 [B][H][16][128] dense copy of each stream's newest window;
// chF: the prune count F of a full window.
cudaError_t launch_compress(const uint16_t *x, int64_t sb, int64_t sh, int64_t st, int L, int B, int H,
                            const HeadKeep &hk, int kmax, int cap, uint32_t *bitmap, uint16_t *values,
                            uint32_t *tile_offset, Pattern pat, uint16_t *window, int chF, cudaStream_t stream);
cudaError_t launch_append(const uint16_t *x, int64_t sb, int64_t sh, const int32_t *pos, int B, int H,
                          const HeadKeep &hk, int cap, uint32_t *bitmap, uint16_t *values, uint32_t *err,
                          Pattern pat, uint16_t *window, int chF, cudaStream_t stream);

// One channel-wise cache's share of an append launch: the new tokens (x, strided [B][H][128]) and
// the cache arrays; F is the prune count of a full window.
struct ChannelAppend {
  const uint16_t *x;
  int64_t sb, sh;
  int keep, F, cap;
  uint32_t *bitmap;
  uint16_t *values;
  uint16_t *window;
};
// Append one token per (b, kv head) to each of `ncaches` (1 or 2) channel-wise caches in one launch.
cudaError_t launch_append_channel(const ChannelAppend *c, int ncaches, const int32_t *pos, int B, int H,
                                  uint32_t *err, cudaStream_t stream);

struct DecodeParams {
  const uint16_t *q;  // [B][Hq][128]
  // compressed caches (sparse kernel)
  const uint32_t *kbm;
  const uint16_t *kval;
  const uint32_t *vbm;
  const uint16_t *vval;
  int keep_k, keep_v;  // the largest keep of each cache (sizes the staging buffers)
  HeadKeep hk_k, hk_v;  // per kv head keep counts and value placement
  int perhead;          // either cache has a keep count per kv head
  int p24_k, p24_v;     // the cache is 2:4-pruned (the fused step appends with that rule)
  uint16_t *kwin, *vwin;  // channel-wise caches: the dense newest-window copies (else nullptr)
  int chF_k, chF_v;       // channel-wise caches: the prune count F of a full 16-token window
  // dense caches (baseline kernel), [B][Hkv][cap][128]
  const uint16_t *kd;
  const uint16_t *vd;
  int cap_k, cap_v;
  const int32_t *seq_len;
  int B, Hq, Hkv, G;
  float scale_log2;
  int num_splits, chunks_per_split;
  int stage_bytes, warp_bytes;
  int lg_k, lg_v;      // sparse kernel: a cache is staged in groups of 2^lg tokens, 16 B apart (4: one copy)
  int skew_k, skew_v;  // sparse kernel: bytes those gaps add to the cache's staged region
  uint16_t *out;
  float *lse;
  int clu;            // sparse kernel: 0, or the CTAs of one thread-block cluster per stream (each takes an
                      // equal share of its stream's chunks; partials merge in distributed shared memory)
  float *ws_part;     // sparse kernel: [2 * ctas][32 + G*128] partial (m, l, o) slots
  float *ws_o;        // [B*Hq][splits][128]
  float *ws_ml;       // [B*Hq][splits][2]
  uint32_t *ws_cnt;   // [B*Hkv]
  uint32_t *err;
  // fused decode step (sparse kernel, pos != nullptr): append the new token of every (b, kv head)
  // at slot pos[b] of both caches, then attend over pos[b] + 1 tokens
  const int32_t *pos;
  const uint16_t *kn;  // [B][Hkv][128] strided
  const uint16_t *vn;
  int64_t kn_sb, kn_sh, vn_sb, vn_sh;
};

struct DecodePlan {
  int splits;
  int chunks_per_split;
  int nstage;
  int stage_bytes;
  int warp_bytes;
  int smem_bytes;
  int lg_k, lg_v, skew_k, skew_v;  // sparse kernel: staging groups of a keep that is a multiple of 32
  int variant;  // sparse kernel: 0 uniform caches, 1 a keep count per kv head, 2 both caches 2:4,
                // 3 token runs located by popcount prefixes (a channel-wise cache)
  int clu;      // sparse kernel: CTAs per thread-block cluster, one cluster per stream (0: no clusters)
};

// Dense fp16 baseline: plan (split count, pipeline depth, shared memory) and launch.
cudaError_t plan_dense(int B, int Hkv, int G, int max_len, int forced_splits, DecodePlan *plan);
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int splits);
int decode_split_bound(int B, int Hkv, int max_len);
cudaError_t launch_dense(const DecodeParams &p, const DecodePlan &plan, cudaStream_t stream);

// Sparse decode over the compressed caches (one wave of CTAs over the end-to-end chunk sequence):
// plan->splits holds the CTA count.
// variant: as DecodePlan::variant
cudaError_t plan_sparse(int B, int Hkv, int G, int max_len, int keep_k, int keep_v, int forced_splits, int variant,
                        DecodePlan *plan);
cudaError_t launch_sparse(const DecodeParams &p, const DecodePlan &plan, cudaStream_t stream);
int sparse_decode_ctas(int B, int Hkv, int max_len, int forced_splits, int per_sm);
size_t sparse_workspace_bytes(int B, int Hkv, int G, int ctas);
// workspace that suffices for any plan of these shapes (assumes the most resident CTAs per SM)
size_t sparse_workspace_bound(int B, int Hkv, int G, int max_len, int forced_splits);

}  // namespace mustafar
