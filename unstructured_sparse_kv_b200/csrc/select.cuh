// select.cuh - deterministic per-token top-k by magnitude, one thread per 128-channel vector.
//
// Per-token magnitude pruning (MUSTAFAR summary, atlas.scime.ai, "Approach"; Mustafar
// abstract, catalyzex author page): keep the k channels with the largest |x|.  The
// library fixes the two points the pages leave open: the magnitude key is the fp16
// bit pattern with the sign cleared (so the order is |x| for finite values and +0 == -0),
// and on equal keys the lower channel index is kept.
//
// Method: a 15-step binary search for the k-th largest key T (the largest T with
// #{key >= T} >= k).  Each count is SIMD-within-a-register: for the top 7 bits four key high
// bytes share a word, for the low 8 two 15-bit keys do, and key + (0x8000 - T) sets bit 15 of
// its half exactly when key >= T (no carry leaves a half).  Keys are paired as (channel i, channel i+16) of a 32-channel
// group so that shifting the sum right by 15-i drops both indicator bits onto bits i and
// 16+i: OR-ing the 16 pairs of a group yields that group's bitmap word directly.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace mustafar {

// raw[r] holds channels (2r, 2r+1) as two fp16 values (low half = even channel).
// Produces p[16w + i] = key(32w + i) | key(32w + i + 16) << 16.
__device__ __forceinline__ void make_keys(const uint32_t (&raw)[64], uint32_t (&p)[64]) {
#pragma unroll
  for (int w = 0; w < kWords; ++w) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t a = raw[16 * w + (i >> 1)];
      const uint32_t b = raw[16 * w + 8 + (i >> 1)];
      p[16 * w + i] = __byte_perm(a, b, (i & 1) ? 0x7632u : 0x5410u) & 0x7FFF7FFFu;
    }
  }
}

// Bitmap of {channel : key >= T}, 0 <= T <= 0x8000.
__device__ __forceinline__ void ge_bitmap(const uint32_t (&p)[64], uint32_t T, uint32_t (&g)[kWords]) {
  uint32_t c = 0x8000u - T;
  c |= c << 16;
#pragma unroll
  for (int w = 0; w < kWords; ++w) {
    uint32_t acc = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      // bits 15 and 31 of t -> bits i and 16+i: t >> (15-i) as a multiply-high, so that the integer
      // multiply-add unit takes the shift and the accumulation off the logic pipe (the positions
      // never overlap, so adding is OR-ing)
      const uint32_t t = (p[16 * w + i] + c) & 0x80008000u;
      acc += i == 15 ? t : __umulhi(t, 1u << (17 + i));
    }
    g[w] = acc;
  }
}

__device__ __forceinline__ int popc4(const uint32_t (&g)[kWords]) {
  return __popc(g[0]) + __popc(g[1]) + __popc(g[2]) + __popc(g[3]);
}

// Bits 14..8 of the top-k threshold (the largest T with #{key >= T} >= k), from the keys' high
// bytes packed four to a word (any channel order: only counts are needed).  For a candidate with a
// zero low byte, key >= cand exactly when (key >> 8) >= (cand >> 8), and byte + (0x80 - h) sets
// the byte's bit 7 exactly when byte >= h (no carry leaves a byte).
__device__ __forceinline__ uint32_t high_threshold(const uint32_t (&hb)[32], int k) {
  uint32_t T = 0;
#pragma unroll 1
  for (int bit = 6; bit >= 0; --bit) {
    const uint32_t h = (T >> 8) | (1u << bit);
    const uint32_t c = (0x80u - h) * 0x01010101u;
    uint32_t acc[4] = {0u, 0u, 0u, 0u};  // four per-byte counts each (at most 8): four independent chains
#pragma unroll
    for (int r = 0; r < 32; ++r) acc[r & 3] += __umulhi((hb[r] + c) & 0x80808080u, 1u << 25);
    const uint32_t sum = (acc[0] + acc[1]) + (acc[2] + acc[3]);  // each byte at most 32
    if (static_cast<int>((sum * 0x01010101u) >> 24) >= k) T = h << 8;
  }
  return T;
}

// #{key >= T} over the 128 keys packed two per register, by fp16x2 compares: valid when T is a finite
// fp16 pattern (T < 0x7C00) and only for keys that are not NaN.  set.ge gives 1.0 or 0.0 per half; the
// sums (at most 16 per half in each of four accumulators) are exact in fp16.
__device__ __forceinline__ uint32_t count_f16_ge(const uint32_t (&p)[64], uint32_t T) {
  const uint32_t t2 = T | (T << 16);
  uint32_t acc[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    uint32_t s;
    asm("set.ge.f16x2.f16x2 %0, %1, %2;" : "=r"(s) : "r"(p[i]), "r"(t2));
    asm("add.rn.f16x2 %0, %0, %1;" : "+r"(acc[i & 3]) : "r"(s));
  }
  uint32_t a01, a23, a;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(a01) : "r"(acc[0]), "r"(acc[1]));
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(a23) : "r"(acc[2]), "r"(acc[3]));
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(a) : "r"(a01), "r"(a23));
  const __half2 h = *reinterpret_cast<const __half2 *>(&a);
  return static_cast<uint32_t>(__half2float(__low2half(h)) + __half2float(__high2half(h)));
}

// #{key that is a NaN pattern (key > 0x7C00)} over the 128 packed keys (an unordered self-compare).
__device__ __forceinline__ uint32_t count_f16_nan(const uint32_t (&p)[64]) {
  uint32_t acc[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    uint32_t s;
    asm("set.nan.f16x2.f16x2 %0, %1, %1;" : "=r"(s) : "r"(p[i]));
    asm("add.rn.f16x2 %0, %0, %1;" : "+r"(acc[i & 1]) : "r"(s));
  }
  uint32_t a;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(a) : "r"(acc[0]), "r"(acc[1]));
  const __half2 h = *reinterpret_cast<const __half2 *>(&a);
  return static_cast<uint32_t>(__half2float(__low2half(h)) + __half2float(__high2half(h)));
}

// Kept-channel bitmap of the k largest keys, ties toward the lower channel index, given bits
// 14..8 of the threshold (high_threshold).
__device__ __forceinline__ void topk_bitmap(const uint32_t (&raw)[64], int k, uint32_t T, uint32_t (&bm)[kWords]) {
  uint32_t p[64];
  make_keys(raw, p);
  // bits 7..0 on the full keys, two per register
  uint32_t g[kWords];
  if (T < 0x7C00u) {
    // a finite threshold: a key is a non-negative fp16 bit pattern, and for two such patterns that are
    // not NaN the integer order is the fp16 order, so the counts can use fp16x2 compares (one logic-pipe
    // op per two keys instead of two); NaN keys rank above every finite candidate but compare false,
    // so they are counted once and added
    const uint32_t nan = count_f16_nan(p);
#pragma unroll 1
    for (int bit = 7; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      if (count_f16_ge(p, cand) + nan >= static_cast<uint32_t>(k)) T = cand;
    }
  } else {
#pragma unroll 1
    for (int bit = 7; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      ge_bitmap(p, cand, g);
      if (popc4(g) >= k) T = cand;
    }
  }
  ge_bitmap(p, T, g);  // #{key >= T} >= k, and #{key > T} < k
  if (popc4(g) == k) {
#pragma unroll
    for (int w = 0; w < kWords; ++w) bm[w] = g[w];
    return;
  }
  uint32_t gt[kWords];
  ge_bitmap(p, T + 1, gt);
  int need = k - popc4(gt);  // how many of the keys equal to T survive, lowest channels first
#pragma unroll
  for (int w = 0; w < kWords; ++w) {
    uint32_t e = g[w] & ~gt[w];
    uint32_t take = 0;
    while (e != 0u && need > 0) {
      const uint32_t low = e & (0u - e);
      take |= low;
      e ^= low;
      --need;
    }
    bm[w] = gt[w] | take;
  }
}

// One warp prunes and compresses one 128-channel vector (fp16 at src, device memory):
// writes its 4 bitmap words to bm_dst and its k kept values, ascending channel, to val_dst.
// Lane l holds channels l, l+32, l+64, l+96, so a ballot over one of its four keys is one bitmap
// word.  Same selection as topk_bitmap: binary search for the k-th largest key T, then the keys
// equal to T are taken lowest channel first.  All 32 lanes must call it.
__device__ __forceinline__ void warp_compress_vector(const uint16_t *src, int k, uint32_t *bm_dst, uint16_t *val_dst,
                                                     int lane) {
  uint32_t raw[kWords], key[kWords];
#pragma unroll
  for (int w = 0; w < kWords; ++w) {
    raw[w] = src[32 * w + lane];
    key[w] = raw[w] & 0x7FFFu;
  }
  uint32_t T = 0;
#pragma unroll 1
  for (int bit = 14; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    int n = 0;
#pragma unroll
    for (int w = 0; w < kWords; ++w) n += __popc(__ballot_sync(0xffffffffu, key[w] >= cand));
    if (n >= k) T = cand;
  }
  uint32_t bm[kWords];
  int n_gt = 0;
#pragma unroll
  for (int w = 0; w < kWords; ++w) {
    bm[w] = __ballot_sync(0xffffffffu, key[w] > T);
    n_gt += __popc(bm[w]);
  }
  int need = k - n_gt;  // keys equal to T that survive, lowest channels first
#pragma unroll
  for (int w = 0; w < kWords; ++w) {
    uint32_t e = __ballot_sync(0xffffffffu, key[w] == T);
    while (e != 0u && need > 0) {
      const uint32_t low = e & (0u - e);
      bm[w] |= low;
      e ^= low;
      --need;
    }
  }
  if (lane < kWords) bm_dst[lane] = lane == 0 ? bm[0] : lane == 1 ? bm[1] : lane == 2 ? bm[2] : bm[3];
  const uint32_t below = (1u << lane) - 1u;
  int prefix = 0;
#pragma unroll
  for (int w = 0; w < kWords; ++w) {
    if ((bm[w] >> lane) & 1u) val_dst[prefix + __popc(bm[w] & below)] = static_cast<uint16_t>(raw[w]);
    prefix += __popc(bm[w]);
  }
}

// ---- 2:4 semi-structured pruning (the comparison pattern of the pages' baselines): in every group
// of 4 consecutive channels keep the 2 largest keys, ties to the lower channel.  An element is kept
// when fewer than 2 group mates beat it (a mate beats it with a larger key, or an equal key at a
// lower channel).

// Bitmap of the 2:4 selection of one vector (raw as in topk_bitmap).
__device__ __forceinline__ void bitmap_24(const uint32_t (&raw)[64], uint32_t (&bm)[kWords]) {
#pragma unroll
  for (int w = 0; w < kWords; ++w) bm[w] = 0u;
#pragma unroll
  for (int j = 0; j < 32; ++j) {  // group j: channels 4j..4j+3 = raw[2j] (lo, hi), raw[2j+1] (lo, hi)
    const uint32_t a = raw[2 * j] & 0x7FFFu, b = (raw[2 * j] >> 16) & 0x7FFFu;
    const uint32_t c = raw[2 * j + 1] & 0x7FFFu, d = (raw[2 * j + 1] >> 16) & 0x7FFFu;
    const int ra = (b > a) + (c > a) + (d > a);
    const int rb = (a >= b) + (c > b) + (d > b);
    const int rc = (a >= c) + (b >= c) + (d > c);
    const int rd = (a >= d) + (b >= d) + (c >= d);
    const uint32_t nib = (ra < 2 ? 1u : 0u) | (rb < 2 ? 2u : 0u) | (rc < 2 ? 4u : 0u) | (rd < 2 ? 8u : 0u);
    bm[j >> 3] |= nib << (4 * (j & 7));
  }
}

// One warp 2:4-prunes and compresses one 128-channel vector (layout as warp_compress_vector:
// lane l holds channels l, l+32, l+64, l+96; a group's four channels sit in lanes 4m..4m+3).
__device__ __forceinline__ void warp_compress_vector_24(const uint16_t *src, uint32_t *bm_dst, uint16_t *val_dst,
                                                        int lane) {
  uint32_t raw[kWords], bm[kWords];
  const int i = lane & 3, g0 = lane & ~3;
#pragma unroll
  for (int w = 0; w < kWords; ++w) {
    raw[w] = src[32 * w + lane];
    const uint32_t key = raw[w] & 0x7FFFu;
    int rank = 0;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const uint32_t km = __shfl_sync(0xffffffffu, key, g0 + m);
      rank += (m != i) && (km > key || (km == key && m < i));
    }
    bm[w] = __ballot_sync(0xffffffffu, rank < 2);
  }
  if (lane < kWords) bm_dst[lane] = lane == 0 ? bm[0] : lane == 1 ? bm[1] : lane == 2 ? bm[2] : bm[3];
  const uint32_t below = (1u << lane) - 1u;
  int prefix = 0;
#pragma unroll
  for (int w = 0; w < kWords; ++w) {
    if ((bm[w] >> lane) & 1u) val_dst[prefix + __popc(bm[w] & below)] = static_cast<uint16_t>(raw[w]);
    prefix += __popc(bm[w]);
  }
}

// ---- channel-wise pruning (the channel direction of the README's K/V [t/c] naming): each channel
// of a stream is pruned across the tokens of a 16-token window.  A window of n tokens keeps, in
// every channel, its window_keep(n, F) largest keys, the lower token index first on ties.

// Descending bitonic sort of 16 keys (every index is a compile-time constant once unrolled).
__device__ __forceinline__ void sort16_desc(uint32_t (&a)[16]) {
#pragma unroll
  for (int k = 2; k <= 16; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int l = i ^ j;
        if (l > i) {
          const uint32_t hi = max(a[i], a[l]), lo = min(a[i], a[l]);
          a[i] = (i & k) == 0 ? hi : lo;
          a[l] = (i & k) == 0 ? lo : hi;
        }
      }
    }
  }
}

// The same network on two 16-bit keys per word (independent sorts of the two halves).
__device__ __forceinline__ void sort16_desc_x2(uint32_t (&a)[16]) {
#pragma unroll
  for (int k = 2; k <= 16; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int l = i ^ j;
        if (l > i) {
          const uint32_t hi = __vmaxu2(a[i], a[l]), lo = __vminu2(a[i], a[l]);
          a[i] = (i & k) == 0 ? hi : lo;
          a[l] = (i & k) == 0 ? lo : hi;
        }
      }
    }
  }
}

// One warp prunes and compresses one window of n (1..16) tokens of a stream, channel-wise.
// src(t) points at token t's 128 fp16 channels (device memory when GLOBAL_SRC, else shared).  Writes the n tokens' bitmap rows
// from bm_dst (4 words a token) and the window's packed values from val_dst, token after token,
// each token's kept channels in ascending order.  When win_dst is not null, tokens win_from .. n-1
// are also copied, dense, to win_dst + 128 t.  `scratch` is 128 words of this warp's shared
// memory.  Lane l holds channels l, l+32, l+64, l+96 of every token, so a ballot over one of them
// is one bitmap word.  All 32 lanes must call it.
// The loops over words and tokens stay rolled: the routine often runs once per warp (an append),
// where a long unrolled body would be fetched from a cold instruction cache.
template <bool GLOBAL_SRC, class Src>
__device__ __forceinline__ void warp_compress_window(Src src, int n, int F, uint32_t *bm_dst, uint16_t *val_dst,
                                                     uint16_t *win_dst, int win_from, uint32_t *scratch, int lane) {
  const int kc = window_keep(n, F);
  const uint32_t valid = n >= 16 ? 0xFFFFu : (1u << n) - 1u;
  // rows in device memory (two 128-byte lines each) are requested up front
  if (GLOBAL_SRC && lane < 2 * n) {
    const uint16_t *line = src(lane >> 1) + 64 * (lane & 1);
    asm volatile("prefetch.global.L1 [%0];\n" ::"l"(line));
  }
  // 1. per channel: sort the window's keys, keep the kc largest (lower token on ties).  Two channels
  //    (words 2p and 2p+1) are sorted together, their keys (at most 0x8000) packed in the two halves of
  //    a word and compared with SIMD 16-bit min/max.  Bit 16w + t of `kept`: token t of channel
  //    32w + lane is kept.
  uint64_t kept = 0u;
#pragma unroll 1
  for (int pw = 0; pw < kWords / 2; ++pw) {
    uint32_t key[16], a[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      const uint16_t *row = src(min(t, n - 1));
      key[t] = row[64 * pw + lane] | (static_cast<uint32_t>(row[64 * pw + 32 + lane]) << 16);  // all in flight
    }
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      if (win_dst != nullptr && t >= win_from && t < n) {
        win_dst[kHeadDim * t + 64 * pw + lane] = static_cast<uint16_t>(key[t]);
        win_dst[kHeadDim * t + 64 * pw + 32 + lane] = static_cast<uint16_t>(key[t] >> 16);
      }
      // keys are shifted up by one so that the missing tokens of a short window (0) sort last
      key[t] = t < n ? (key[t] & 0x7FFF7FFFu) + 0x00010001u : 0u;
      a[t] = key[t];
    }
    sort16_desc_x2(a);
    uint32_t T2 = a[0];  // the kc-th largest key of each half
#pragma unroll
    for (int i = 1; i < 16; ++i) T2 = i == kc - 1 ? a[i] : T2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t T = (T2 >> (16 * h)) & 0xFFFFu;
      uint32_t gt = 0u, eq = 0u;
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const uint32_t kk = (key[t] >> (16 * h)) & 0xFFFFu;
        gt |= (kk > T ? 1u : 0u) << t;
        eq |= (kk == T ? 1u : 0u) << t;
      }
      gt &= valid;
      eq &= valid;
      int need = kc - __popc(gt);  // keys equal to T that survive, lowest tokens first
      uint32_t take = gt;
      while (eq != 0u && need > 0) {
        const uint32_t low = eq & (0u - eq);
        take |= low;
        eq ^= low;
        --need;
      }
      kept |= static_cast<uint64_t>(take) << (16 * (2 * pw + h));
    }
  }
  // 2. bitmap words by ballot, and where each (token, word) run starts: scratch[4t + w] holds the
  //    word, scratch[64 + 4t + w] the run start within the window
  uint32_t pre = 0u;
#pragma unroll 1
  for (int t = 0; t < n; ++t) {  // n is the same in every lane
    uint32_t bm[kWords];
#pragma unroll
    for (int w = 0; w < kWords; ++w) bm[w] = __ballot_sync(0xffffffffu, (kept >> (16 * w + t)) & 1u);
    if (lane < kWords) {
      const uint32_t mine = lane == 0 ? bm[0] : lane == 1 ? bm[1] : lane == 2 ? bm[2] : bm[3];
      const uint32_t before = lane == 0 ? 0u
                              : lane == 1 ? __popc(bm[0])
                              : lane == 2 ? __popc(bm[0]) + __popc(bm[1])
                                          : __popc(bm[0]) + __popc(bm[1]) + __popc(bm[2]);
      bm_dst[kWords * t + lane] = mine;
      scratch[kWords * t + lane] = mine;
      scratch[64 + kWords * t + lane] = pre + before;
    }
    pre += __popc(bm[0]) + __popc(bm[1]) + __popc(bm[2]) + __popc(bm[3]);
  }
  __syncwarp();
  // 3. the kept values, one word (32 channels) of every token at a time
  const uint32_t below = (1u << lane) - 1u;
#pragma unroll 1
  for (int w = 0; w < kWords; ++w) {
    uint16_t xs[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) xs[t] = src(min(t, n - 1))[32 * w + lane];  // all in flight at once
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      if (t < n) {
        const uint32_t word = scratch[kWords * t + w];
        if ((word >> lane) & 1u) val_dst[scratch[64 + kWords * t + w] + __popc(word & below)] = xs[t];
      }
    }
  }
  __syncwarp();  // the scratch may be reused by the caller's next window
}

}  // namespace mustafar
