// compress.cu - prune + compress (prefill) and append (decode) kernels.
//
// Per-token magnitude pruning and the bitmap-based sparse format (MUSTAFAR summary,
// atlas.scime.ai, "Approach"; Mustafar abstract, catalyzex author page).  Layout of
// the format: see include/mustafar.h.
//
// compress: one CTA = 128 consecutive tokens of one (b, kv head) stream, one thread per
//   token.  The CTA stages its 32 KB of dense rows in shared memory with coalesced
//   16-byte cp.async (16 threads per 256-byte row), each thread runs the top-k on its
//   own row, writes its 16-byte bitmap and packs its kept values into a shared staging run
//   (one predicated 16-bit store per channel); then the CTA writes the 128*k packed values
//   with coalesced 16-byte stores.
// append: one warp per (b, kv head) vector of the new token.
// channel-wise caches: one warp per 16-token window (compress) or per stream's newest window
//   (append), through warp_compress_window.
#include "internal.h"
#include "select.cuh"

namespace mustafar {

constexpr int kCompressThreads = 128;
constexpr int kRowBytesDense = kHeadDim * 2;  // 256

// byte offset of 16-byte chunk j of staged row `tok` (XOR swizzle: conflict-free row reads)
__device__ __forceinline__ int stage_off(int tok, int j) { return tok * kRowBytesDense + ((j ^ (tok & 15)) << 4); }

// Channels I and I+1 of a chunk (the halves of x): each whose bit is set in `bits` is stored at the
// shared address dst, which then steps by one value.
template <int I>
__device__ __forceinline__ void pack_pair(uint32_t &dst, uint32_t bits, uint32_t x) {
  asm volatile(
      "{\n .reg .pred p, q;\n .reg .b32 t, h;\n"
      " and.b32 t, %1, %3;\n setp.ne.u32 p, t, 0;\n @p st.shared.u16 [%0], %2;\n @p add.u32 %0, %0, 2;\n"
      " and.b32 t, %1, %4;\n setp.ne.u32 q, t, 0;\n shr.u32 h, %2, 16;\n @q st.shared.u16 [%0], h;\n"
      " @q add.u32 %0, %0, 2;\n}\n"
      : "+r"(dst)
      : "r"(bits), "r"(x), "n"(1u << I), "n"(2u << I)
      : "memory");
}

template <bool P24>
__global__ void __launch_bounds__(kCompressThreads)
compress_kernel(const uint16_t *__restrict__ x, int64_t sb, int64_t sh, int64_t st, int L, int H, const HeadKeep hk,
                int cap, uint32_t *__restrict__ bitmap, uint16_t *__restrict__ values,
                uint32_t *__restrict__ tile_offset) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t *in_stage = smem;
  uint16_t *out_stage = reinterpret_cast<uint16_t *>(smem + kCompressThreads * kRowBytesDense);

  const int tid = threadIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t stream = static_cast<int64_t>(b) * H + h;
  const int k = hk.k[h];

  // tile offsets of the whole stream: the closed form 64*i*k (= popcount prefix sums, every
  // token keeps exactly k channels)
  const int ntiles = cap / kTileTokens;
  for (int i = blockIdx.x * kCompressThreads + tid; i < ntiles; i += gridDim.x * kCompressThreads)
    tile_offset[stream * ntiles + i] = static_cast<uint32_t>(i) * kTileTokens * static_cast<uint32_t>(k);

  const int t0 = blockIdx.x * kCompressThreads;
  const int ntok = min(kCompressThreads, L - t0);
  if (ntok <= 0) return;

  const uint16_t *xs = x + static_cast<int64_t>(b) * sb + static_cast<int64_t>(h) * sh;
  for (int idx = tid; idx < ntok * 16; idx += kCompressThreads) {
    const int tok = idx >> 4, j = idx & 15;
    cp_async16(smem_addr(in_stage + stage_off(tok, j)), xs + static_cast<int64_t>(t0 + tok) * st + j * 8);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  if (tid < ntok) {
    uint32_t T = 0;
    if constexpr (!P24) {
      // the threshold's high bits from the row's high bytes, before the full keys take registers
      uint32_t hb[32];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint4 v = *reinterpret_cast<const uint4 *>(in_stage + stage_off(tid, j));
        hb[2 * j] = __byte_perm(v.x, v.y, 0x7531u) & 0x7F7F7F7Fu;
        hb[2 * j + 1] = __byte_perm(v.z, v.w, 0x7531u) & 0x7F7F7F7Fu;
      }
      T = high_threshold(hb, k);
      asm volatile("" ::: "memory");  // the full row is loaded only now, after the high bytes are dead
    }
    uint32_t raw[64];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint4 v = *reinterpret_cast<const uint4 *>(in_stage + stage_off(tid, j));
      raw[4 * j + 0] = v.x;
      raw[4 * j + 1] = v.y;
      raw[4 * j + 2] = v.z;
      raw[4 * j + 3] = v.w;
    }
    uint32_t bm[kWords];
    if constexpr (P24) {
      bitmap_24(raw, bm);
    } else {
      topk_bitmap(raw, k, T, bm);
    }
    const uint4 row = make_uint4(bm[0], bm[1], bm[2], bm[3]);
    reinterpret_cast<uint4 *>(bitmap)[stream * cap + t0 + tid] = row;
    if (popc4(bm) == k) {  // (the bitmap holds k bits by construction; the check keeps the run in bounds)
      // the thread packs its own row: one predicated 16-bit store per channel (bit set: store and step
      // the run pointer), reading the staged row 16 bytes at a time, so the cost does not grow with k
      // (a walk over the set bits costs about 25 instructions per kept value, and a CTA-wide pass with
      // one thread per 8-channel slice of a row measured slower than this at every keep)
      uint32_t dst = smem_addr(out_stage + tid * k);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint4 v = *reinterpret_cast<const uint4 *>(in_stage + stage_off(tid, j));
        const uint32_t bits = bm[j >> 2] >> (8 * (j & 3));  // channels 8j .. 8j+7
        pack_pair<0>(dst, bits, v.x);
        pack_pair<2>(dst, bits, v.y);
        pack_pair<4>(dst, bits, v.z);
        pack_pair<6>(dst, bits, v.w);
      }
    }
  }
  __syncthreads();

  // coalesced write-out of the CTA's packed run; its start (value base + t0*k)*2 bytes is
  // 16-byte aligned because the value base is a multiple of cap, cap % 64 == 0 and t0 % 128 == 0
  uint16_t *vdst = values + hk.value_base(b, h, H, cap) + static_cast<int64_t>(t0) * k;
  const int n = ntok * k;
  const int nvec = n >> 3;
  for (int i = tid; i < nvec; i += kCompressThreads)
    reinterpret_cast<uint4 *>(vdst)[i] = reinterpret_cast<const uint4 *>(out_stage)[i];
  for (int i = (nvec << 3) + tid; i < n; i += kCompressThreads) vdst[i] = out_stage[i];
}

// append: one warp per (b, kv head) vector, for latency (a decode step appends only B*Hkv
// vectors).  Lane l holds channels l, l+32, l+64, l+96, so a ballot over one of its four keys
// is directly one bitmap word.  The same selection as topk_bitmap: binary search for the k-th
// largest key T, then the keys equal to T are taken lowest channel first.
template <bool P24>
__global__ void __launch_bounds__(128)
append_kernel(const uint16_t *__restrict__ x, int64_t sb, int64_t sh, const int32_t *__restrict__ pos, int B,
              int H, const HeadKeep hk, int cap, uint32_t *__restrict__ bitmap, uint16_t *__restrict__ values,
              uint32_t *__restrict__ err) {
  const int lane = threadIdx.x & 31;
  const int v = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (v >= B * H) return;
  const int b = v / H, h = v - b * H;
  const int p = pos[b];
  if (p < 0 || p >= cap) {
    if (lane == 0 && err != nullptr) atomicOr(err, MUSTAFAR_DEVERR_POS_RANGE);
    return;
  }
  const uint16_t *src = x + static_cast<int64_t>(b) * sb + static_cast<int64_t>(h) * sh;
  const int64_t stream = static_cast<int64_t>(b) * H + h;
  const int k = hk.k[h];
  uint32_t *bm_dst = bitmap + (stream * cap + p) * kWords;
  uint16_t *val_dst = values + hk.value_base(b, h, H, cap) + static_cast<int64_t>(p) * k;
  if constexpr (P24) {
    warp_compress_vector_24(src, bm_dst, val_dst, lane);
  } else {
    warp_compress_vector(src, k, bm_dst, val_dst, lane);
  }
}

// Channel-wise compress: warp w of CTA x takes window 4x + w of stream (b = z, h = y), and the
// warp of an incomplete last window also keeps its tokens in the stream's dense window copy.  The
// CTA first stages its 64 dense rows in shared memory with coalesced 16-byte copies, so that the
// selection reads its keys with plain shared loads.
__global__ void __launch_bounds__(128)
compress_channel_kernel(const uint16_t *__restrict__ x, int64_t sb, int64_t sh, int64_t st, int L, int H, int keep,
                        int F, int cap, uint32_t *__restrict__ bitmap, uint16_t *__restrict__ values,
                        uint32_t *__restrict__ tile_offset, uint16_t *__restrict__ window) {
  __shared__ uint32_t scratch[4][128];
  __shared__ __align__(16) uint16_t rows[4 * kWindowTokens][kHeadDim];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t stream = static_cast<int64_t>(b) * H + h;
  // tile i starts at 64*i*keep: window j owns the 16*keep elements from j*16*keep
  const int ntiles = cap / kTileTokens;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < ntiles; i += gridDim.x * blockDim.x)
    tile_offset[stream * ntiles + i] = static_cast<uint32_t>(i) * kTileTokens * static_cast<uint32_t>(keep);
  const int tb = blockIdx.x * 4 * kWindowTokens;
  const int ntok = min(4 * kWindowTokens, L - tb);
  if (ntok <= 0) return;
  const uint16_t *xs = x + static_cast<int64_t>(b) * sb + static_cast<int64_t>(h) * sh;
  for (int idx = threadIdx.x; idx < ntok * 16; idx += blockDim.x) {
    const int tok = idx >> 4, j = idx & 15;
    cp_async16(smem_addr(&rows[tok][8 * j]), xs + static_cast<int64_t>(tb + tok) * st + 8 * j);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  const int t0 = tb + warp * kWindowTokens;
  if (t0 >= L) return;
  const int n = min(kWindowTokens, L - t0);
  const uint16_t *ws = &rows[warp * kWindowTokens][0];
  uint16_t *win = n < kWindowTokens ? window + stream * kWindowTokens * kHeadDim : nullptr;
  warp_compress_window<false>([=](int t) { return ws + t * kHeadDim; }, n, F, bitmap + (stream * cap + t0) * kWords,
                       values + (stream * cap + t0) * keep, win, 0, scratch[warp], lane);
}

// Channel-wise append: one warp per (cache, b, kv head), for one or two caches (a decode step's K
// and V) in one launch.  The new token goes to slot pos % 16 of the stream's window copy, and the
// window (tokens 16*floor(pos/16) .. pos) is pruned again.
__global__ void __launch_bounds__(128)
append_channel_kernel(const ChannelAppend c0, const ChannelAppend c1, const int32_t *__restrict__ pos, int B, int H,
                      int ncaches, uint32_t *__restrict__ err) {
  __shared__ uint32_t scratch[4][128];
  const int lane = threadIdx.x & 31;
  int v = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (v >= ncaches * B * H) return;
  const bool second = v >= B * H;
  const ChannelAppend &c = second ? c1 : c0;
  v -= second ? B * H : 0;
  const int b = v / H, h = v - b * H;
  const int p = pos[b];
  if (p < 0 || p >= c.cap) {
    if (lane == 0 && err != nullptr) atomicOr(err, MUSTAFAR_DEVERR_POS_RANGE);
    return;
  }
  const int r = p % kWindowTokens, t0 = p - r;
  const int64_t stream = static_cast<int64_t>(b) * H + h;
  const uint16_t *xn = c.x + static_cast<int64_t>(b) * c.sb + static_cast<int64_t>(h) * c.sh;
  uint16_t *win = c.window + stream * kWindowTokens * kHeadDim;
  warp_compress_window<true>([=](int t) -> const uint16_t * { return t < r ? win + t * kHeadDim : xn; }, r + 1, c.F,
                       c.bitmap + (stream * c.cap + t0) * kWords, c.values + (stream * c.cap + t0) * c.keep, win, r,
                       scratch[threadIdx.x >> 5], lane);
}

cudaError_t launch_append_channel(const ChannelAppend *c, int ncaches, const int32_t *pos, int B, int H,
                                  uint32_t *err, cudaStream_t stream) {
  const int threads = 128;  // 4 windows per CTA
  const int warps = ncaches * B * H;
  append_channel_kernel<<<(warps * 32 + threads - 1) / threads, threads, 0, stream>>>(
      c[0], ncaches > 1 ? c[1] : c[0], pos, B, H, ncaches, err);
  return cudaGetLastError();
}

cudaError_t launch_compress(const uint16_t *x, int64_t sb, int64_t sh, int64_t st, int L, int B, int H,
                            const HeadKeep &hk, int kmax, int cap, uint32_t *bitmap, uint16_t *values,
                            uint32_t *tile_offset, Pattern pat, uint16_t *window, int chF, cudaStream_t stream) {
  if (pat == Pattern::kChannel) {
    const int windows = (L + kWindowTokens - 1) / kWindowTokens;
    dim3 grid(windows > 0 ? (windows + 3) / 4 : 1, H, B);
    compress_channel_kernel<<<grid, 128, 0, stream>>>(x, sb, sh, st, L, H, kmax, chF, cap, bitmap, values,
                                                      tile_offset, window);
    return cudaGetLastError();
  }
  const bool p24 = pat == Pattern::k24;
  auto kernel = p24 ? compress_kernel<true> : compress_kernel<false>;
  const size_t smem = kCompressThreads * kRowBytesDense + static_cast<size_t>(kCompressThreads) * kmax * 2;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(kernel), p24 ? 9 : 0,
                                    kCompressThreads * kRowBytesDense + kCompressThreads * kHeadDim * 2);
  if (e != cudaSuccess) return e;
  const int nbx = L > 0 ? (L + kCompressThreads - 1) / kCompressThreads : 1;
  dim3 grid(nbx, H, B);
  kernel<<<grid, kCompressThreads, smem, stream>>>(x, sb, sh, st, L, H, hk, cap, bitmap, values, tile_offset);
  return cudaGetLastError();
}

cudaError_t launch_append(const uint16_t *x, int64_t sb, int64_t sh, const int32_t *pos, int B, int H,
                          const HeadKeep &hk, int cap, uint32_t *bitmap, uint16_t *values, uint32_t *err,
                          Pattern pat, uint16_t *window, int chF, cudaStream_t stream) {
  const int warps = B * H;
  const int threads = 128;  // 4 vectors per CTA
  if (pat == Pattern::kChannel) {
    const ChannelAppend c{x, sb, sh, hk.k[0], chF, cap, bitmap, values, window};
    return launch_append_channel(&c, 1, pos, B, H, err, stream);
  }
  auto kernel = pat == Pattern::k24 ? append_kernel<true> : append_kernel<false>;
  kernel<<<(warps * 32 + threads - 1) / threads, threads, 0, stream>>>(x, sb, sh, pos, B, H, hk, cap, bitmap,
                                                                       values, err);
  return cudaGetLastError();
}

}  // namespace mustafar
