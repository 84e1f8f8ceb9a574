// decode_sparse.cu - decode attention computed directly over the bitmap-compressed caches.
//
// For each batch row b and q head hq (kv head g = hq / G):
//   out = softmax(scale * q K~^T) V~  over the pruned caches K~, V~,
// read in their compressed form (Mustafar abstract, catalyzex author page: a custom attention
// kernel that works on the compressed caches; MUSTAFAR summary, atlas.scime.ai, "Approach": an
// SpMV-style attention kernel over the bitmap format).  The fused decode step (pos != nullptr)
// first prunes and compresses each stream's new token into slot pos[b] (the runtime pruning of
// the Mustafar abstract), then attends over pos[b] + 1 tokens.
//
// Work decomposition (B200-first, not the pages' design):
// * a stream is one (b, kv head); its context is cut into 16-token chunks.  The chunks of all
//   streams are laid end to end (stream-major) and the sequence is cut into one contiguous,
//   equal range per CTA, for one wave of CTAs.  Warp w of a CTA takes chunks w, w+4, ... of the
//   range, so every warp of the grid gets the same number of chunks to within one, whatever the
//   mix of row lengths.
// * a range may cross streams.  Its pieces are taken in order; at the end of each piece the four
//   warps merge (m, l, o) in shared memory.  A stream whose chunks all lie in one range is
//   finished by that CTA; a stream cut by range edges leaves one partial per CTA in the
//   workspace and the last of those CTAs to finish (atomic ticket, no waiting) merges them.
//   When the plan gives every stream the same whole number C of CTAs and all the streams' C-CTA
//   thread-block clusters are resident at once, each stream's CTAs run as one cluster instead
//   and merge through distributed shared memory between two cluster barriers.
// * every warp reads the row lengths and computes its CTA's range itself, so that it can start
//   its copies before the CTA-wide barrier.
// * each warp stages its chunks through its own ring of NSTAGE buffers.  One lane issues, per
//   chunk, four bulk copies of contiguous bytes (K bitmap rows, V bitmap rows, K packed values,
//   V packed values) that complete on the buffer's mbarrier; every wait is bounded in time.
// * per chunk, S = Q K~^T and O^T += V~^T P^T run as mma.sync m16n8k16 (fp16 in, fp32
//   accumulate) on fragments that each lane expands straight from the compressed bytes: one
//   predicated 16-bit shared load per channel, the bitmap bit as the predicate, pruned channels
//   reading a shared zero.  The contraction index is permuted so that a lane's channels are one
//   bitmap word (K) or half word (V); q's fragments use the same permutation and the output
//   channels are put back in order at the merge.  Online softmax per head in the log2 domain.
//
// Template variants (chosen on the host per call): PERHEAD reads a keep count and value base per
// kv head; P24 expands 2:4 caches with byte permutes instead of the per-channel walk; SCAN finds
// each token's run from popcount prefix sums (channel-wise caches, whose tokens keep varying
// counts); SKEW stages a cache whose keep is a multiple of 32 in 16-byte-skewed token groups so
// that the runs do not all start on one shared-memory bank.
#include <cfloat>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace mustafar {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr float kNegInf = -INFINITY;
constexpr long long kWaitCycles = 4000000000LL;   // a bulk copy not landed after ~2 s is an error
constexpr long long kWaitCyclesAfter = 2000000LL;  // later waits of a warp that already timed out

__device__ __forceinline__ int n_chunks(int L) { return (L + kChunk - 1) / kChunk; }

// Tokens of batch row b that the attention covers (clamped to [0, cap]); `bits` collects the
// device error flags of the row.
__device__ __forceinline__ int row_len(const DecodeParams &P, int b, int cap, uint32_t &bits) {
  if (P.pos != nullptr) {
    const int p = P.pos[b];
    if (p < 0 || p >= cap) {
      bits |= MUSTAFAR_DEVERR_POS_RANGE;
      return p < 0 ? 0 : cap;
    }
    return p + 1;
  }
  const int L = P.seq_len[b];
  if (L < 0 || L > cap) {
    bits |= MUSTAFAR_DEVERR_LEN_RANGE;
    return L < 0 ? 0 : cap;
  }
  return L;
}

__device__ __forceinline__ int row_len(const DecodeParams &P, int b, int cap) {
  uint32_t ignored = 0;
  return row_len(P, b, cap, ignored);
}

// Lengths of the batch rows below kRowCache, read once per CTA at the start (one round of
// independent loads by warp 0) and kept in shared memory: the later look-ups of a row's length
// (the plan, the rows a CTA reports, every stream step) then cost no global round trip.
constexpr int kRowCache = 128;
__device__ __forceinline__ int len_of(const DecodeParams &P, const int *sh_len, int b, int cap) {
  return b < kRowCache ? sh_len[b] : row_len(P, b, cap);
}

// The chunk units of one stream in the end-to-end sequence: [start, start + n).
struct Stream {
  int b, g;   // batch row, kv head
  int n;      // its chunks
  int start;  // its first unit
  __device__ __forceinline__ int end() const { return start + n; }
};

// Step to the next stream in (b, g) order; false past the last one.
__device__ __forceinline__ bool next_stream(const DecodeParams &P, const int *sh_len, int cap, Stream &s) {
  s.start += s.n;
  if (++s.g == P.Hkv) {
    s.g = 0;
    if (++s.b >= P.B) return false;
    s.n = n_chunks(len_of(P, sh_len, s.b, cap));
  }
  return true;
}

// floor(p / d) for 0 <= p, 0 < d: a 32-bit division whenever p fits (every shape up to about 2^31
// chunk-CTA products), which is several times shorter than the 64-bit routine on this latency path
__device__ __forceinline__ long long div_floor(long long p, long long d) {
  if (p <= 0xFFFFFFFFLL && d <= 0xFFFFFFFFLL)
    return static_cast<long long>(static_cast<uint32_t>(p) / static_cast<uint32_t>(d));
  return p / d;
}

// The CTA whose range holds unit u: ranges are [floor(c U / n), floor((c+1) U / n)).
__device__ __forceinline__ int cta_of(long long u, long long U, long long n) {
  return static_cast<int>(div_floor((u + 1) * n - 1, U));
}
__device__ __forceinline__ int range_start(long long c, long long U, long long n) {
  return static_cast<int>(div_floor(c * U, n));
}

// x = (bits & MASK) ? the fp16 at shared address ra : 0 (read from the CTA's zero slot `za`);
// ra advances past a taken value.  No branch and no register zeroing: pruned channels load the
// zero slot, which every pruned lane of a warp reads at the same address (a broadcast).
template <uint32_t MASK>
__device__ __forceinline__ uint32_t take(uint32_t bits, uint32_t &ra, uint32_t za) {
  uint32_t x;
  asm volatile(
      "{\n .reg .pred p;\n .reg .b32 t, a;\n and.b32 t, %2, %3;\n setp.ne.u32 p, t, 0;\n"
      " selp.u32 a, %1, %4, p;\n ld.shared.u16 %0, [a];\n @p add.u32 %1, %1, 2;\n}\n"
      : "=r"(x), "+r"(ra)
      : "r"(bits), "n"(MASK), "r"(za)
      : "memory");
  return x;
}

// The 32 channels of one bitmap word as 16 packed fp16 pairs (channels 2i, 2i+1); the low and
// high half words walk two independent value pointers (ra, rb), interleaved.
template <int I = 0>
__device__ __forceinline__ void expand_word(uint32_t bits, uint32_t ra, uint32_t rb, uint32_t za,
                                            uint32_t (&out)[16]) {
  if constexpr (I < 8) {
    const uint32_t a0 = take<(1u << (2 * I))>(bits, ra, za);
    const uint32_t b0 = take<(1u << (2 * I + 16))>(bits, rb, za);
    const uint32_t a1 = take<(1u << (2 * I + 1))>(bits, ra, za);
    const uint32_t b1 = take<(1u << (2 * I + 17))>(bits, rb, za);
    out[I] = __byte_perm(a0, a1, 0x5410);
    out[I + 8] = __byte_perm(b0, b1, 0x5410);
    expand_word<I + 1>(bits, ra, rb, za, out);
  }
}

// The 16 channels of a half word (bits 0..15 of `bits`) as 16 separate fp16 values.
template <int I = 0>
__device__ __forceinline__ void expand_half(uint32_t bits, uint32_t ra, uint32_t za, uint32_t (&out)[16]) {
  if constexpr (I < 16) {
    out[I] = take<(1u << I)>(bits, ra, za);
    expand_half<I + 1>(bits, ra, za, out);
  }
}

// Running state of one warp over one stream piece: online softmax (m, l) per q-head row and the
// O^T accumulators.  Sparse layout: accumulator rows g / g+8 of m-tile mt are channels
// 16g+2mt / 16g+2mt+1; columns 2q, 2q+1 are heads (oh: heads 8+2q, 8+2q+1).
template <bool HIROWS>
struct Acc {
  float ot[8][4];
  float oh[HIROWS ? 8 : 1][4];
  float m_run[2], l_run[2];
  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int i = 0; i < 8; ++i) ot[i][0] = ot[i][1] = ot[i][2] = ot[i][3] = 0.f;
#pragma unroll
    for (int i = 0; i < (HIROWS ? 8 : 1); ++i) oh[i][0] = oh[i][1] = oh[i][2] = oh[i][3] = 0.f;
    m_run[0] = m_run[1] = kNegInf;
    l_run[0] = l_run[1] = 0.f;
  }
};

// q's A fragments for stream (b, g): rows = the G q heads (zero beyond G), 8 k-steps; k-step ks,
// fragment column 2q+e is channel 32q+4ks+e and column 2q+8+e is 32q+4ks+2+e (the permutation
// that gives lane q the 32 channels of bitmap word q).
template <bool HIROWS>
__device__ __forceinline__ void load_q(const DecodeParams &P, int b, int g, int lane, uint32_t (&qa)[8][4]) {
  const int G = P.G, gq = lane >> 2, qq = lane & 3;
  const uint16_t *qb = P.q + (static_cast<int64_t>(b) * P.Hq + static_cast<int64_t>(g) * G) * kHeadDim;
  const bool r0 = gq < G, r1 = HIROWS && (gq + 8 < G);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int c0 = 32 * qq + 4 * ks, c1 = c0 + 2;
    qa[ks][0] = r0 ? *reinterpret_cast<const uint32_t *>(qb + gq * kHeadDim + c0) : 0u;
    qa[ks][1] = r1 ? *reinterpret_cast<const uint32_t *>(qb + (gq + 8) * kHeadDim + c0) : 0u;
    qa[ks][2] = r0 ? *reinterpret_cast<const uint32_t *>(qb + gq * kHeadDim + c1) : 0u;
    qa[ks][3] = r1 ? *reinterpret_cast<const uint32_t *>(qb + (gq + 8) * kHeadDim + c1) : 0u;
  }
}

// One 16-token chunk staged at `stage` ([K bitmap rows 16x16 B][V bitmap rows][K values 16*kK]
// [V values 16*kV]); tokens t0 .. t0+15 of a row of length L.  `htab` is the warp's 512-byte
// per-row half-word prefix table.  SCAN: token runs of varying length (a channel-wise cache), each
// found by the kept counts of the tokens before it in the chunk; otherwise token T's run starts at
// T*keep.
template <bool HIROWS, bool PERHEAD, bool P24, bool SCAN, bool SKEW>
__device__ __forceinline__ void consume_chunk(const DecodeParams &P, uint8_t *stage, uint8_t *htab, uint32_t za,
                                              int t0, int L, int kKh, int kVh, int lane, const uint32_t (&qa)[8][4],
                                              Acc<HIROWS> &acc, const uint2 *lut24) {
  // keep counts of this stream; a uniform cache reads them from the kernel parameters here, so that
  // they hold no register across the chunk loop
  const int kK = PERHEAD ? kKh : P.keep_k, kV = PERHEAD ? kVh : P.keep_v;
  const int gq = lane >> 2, qq = lane & 3;
  const bool full = t0 + kChunk <= L;
  // lane r (K rows 0-15, V rows 16-31) zeroes the bitmap of a token >= L in place and stores the
  // kept-value count before each of its row's 8 half words (u16 each)
  {
    uint4 *row = reinterpret_cast<uint4 *>(stage + lane * 16);
    uint4 w = *row;
    if (!full && t0 + (lane & 15) >= L) {
      w = make_uint4(0u, 0u, 0u, 0u);
      *row = w;
    }
    if constexpr (!P24) {  // 2:4 runs need no prefixes: every word holds 16 values, every nibble 2
      const uint32_t h0 = __popc(w.x & 0xFFFFu), c0 = __popc(w.x);
      const uint32_t h1 = c0 + __popc(w.y & 0xFFFFu), c1 = c0 + __popc(w.y);
      const uint32_t h2 = c1 + __popc(w.z & 0xFFFFu), c2 = c1 + __popc(w.z);
      const uint32_t h3 = c2 + __popc(w.w & 0xFFFFu);
      uint32_t base = 0u;
      if constexpr (SCAN) {
        // the row's run start: an exclusive prefix sum of the kept counts over the chunk's 16 rows
        // of its cache (lanes 0-15 K, 16-31 V), capped at the staged run length so that a row never
        // reads outside the staging buffers, whatever its bitmap holds
        const uint32_t tot = c2 + __popc(w.w);
        uint32_t inc = tot;
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o, 16);
          if ((lane & 15) >= o) inc += y;
        }
        base = min(inc - tot, static_cast<uint32_t>(kChunk * (lane < 16 ? kK : kV)));
        base |= base << 16;
      }
      *reinterpret_cast<uint4 *>(htab + lane * 16) =
          make_uint4((h0 << 16) + base, (c0 | (h1 << 16)) + base, (c1 | (h2 << 16)) + base, (c2 | (h3 << 16)) + base);
    }
  }
  __syncwarp();

  // ---- S = Q K~^T for the 16 tokens (two n-tiles of 8)
  float s[2][4];
  const uint32_t kvals = smem_addr(stage + 512);
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    const int T = gq + 8 * nt;  // this lane's token (the fragment's n index) in n-tile nt
    const uint32_t word = *reinterpret_cast<const uint32_t *>(stage + T * 16 + qq * 4);
    uint32_t kb[16];
    if constexpr (P24) {
      // word qq's 16 values: 32 contiguous bytes of the token's 128-byte run, nibble j's two in value
      // pair j; placed into channel pairs (4j, 4j+1), (4j+2, 4j+3) by the nibble's two selectors
      const uint8_t *run = stage + 512 + T * 128 + (SKEW ? (T >> P.lg_k) << 4 : 0);
      const uint4 va = *reinterpret_cast<const uint4 *>(run + qq * 32);
      const uint4 vb = *reinterpret_cast<const uint4 *>(run + qq * 32 + 16);
      const uint32_t x[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint2 sel = lut24[(word >> (4 * j)) & 15u];
        kb[2 * j] = __byte_perm(x[j], 0u, sel.x);
        kb[2 * j + 1] = __byte_perm(x[j], 0u, sel.y);
      }
    } else {
      const uint32_t pre = *reinterpret_cast<const uint32_t *>(htab + T * 16 + qq * 4);  // halves 2q, 2q+1
      const uint32_t rbase = SCAN ? kvals : kvals + 2 * T * kK + (SKEW ? (T >> P.lg_k) << 4 : 0);
      expand_word(word, rbase + 2 * (pre & 0xFFFFu), rbase + 2 * (pre >> 16), za, kb);
    }
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) mma_f16_16816(s[nt], qa[ks], kb[2 * ks], kb[2 * ks + 1]);
  }

  // ---- scale into the log2 domain, mask tokens >= L, online softmax per row (= q head)
  float mx[2] = {kNegInf, kNegInf};
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
    for (int e = 0; e < (HIROWS ? 4 : 2); ++e) {
      const int tok = t0 + nt * 8 + 2 * qq + (e & 1);
      const float x = (full || tok < L) ? s[nt][e] * P.scale_log2 : kNegInf;
      s[nt][e] = x;
      mx[e >> 1] = fmaxf(mx[e >> 1], x);
    }
  }
  float alpha[2] = {1.f, 1.f};
#pragma unroll
  for (int h = 0; h < (HIROWS ? 2 : 1); ++h) {
    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
    const float m_new = fmaxf(acc.m_run[h], mx[h]);
    const float base = m_new == kNegInf ? 0.f : m_new;
    alpha[h] = fast_exp2(acc.m_run[h] - base);
    acc.m_run[h] = m_new;
    mx[h] = base;
  }
  float psum[2] = {0.f, 0.f};
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
    for (int e = 0; e < (HIROWS ? 4 : 2); ++e) {
      const float p = fast_exp2(s[nt][e] - mx[e >> 1]);
      s[nt][e] = p;
      psum[e >> 1] += p;
    }
  }
  acc.l_run[0] = acc.l_run[0] * alpha[0] + psum[0];
  if constexpr (HIROWS) acc.l_run[1] = acc.l_run[1] * alpha[1] + psum[1];
  if (__any_sync(0xffffffffu, alpha[0] != 1.f || (HIROWS && alpha[1] != 1.f))) {
    // the O^T columns this lane holds are heads 2q and 2q+1, whose factors live in lanes 8q and 8q+4
    const float a_lo = __shfl_sync(0xffffffffu, alpha[0], 8 * qq);
    const float a_hi = __shfl_sync(0xffffffffu, alpha[0], 8 * qq + 4);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      acc.ot[mt][0] *= a_lo;
      acc.ot[mt][1] *= a_hi;
      acc.ot[mt][2] *= a_lo;
      acc.ot[mt][3] *= a_hi;
    }
    if constexpr (HIROWS) {
      const float b_lo = __shfl_sync(0xffffffffu, alpha[1], 8 * qq);
      const float b_hi = __shfl_sync(0xffffffffu, alpha[1], 8 * qq + 4);
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        acc.oh[mt][0] *= b_lo;
        acc.oh[mt][1] *= b_hi;
        acc.oh[mt][2] *= b_lo;
        acc.oh[mt][3] *= b_hi;
      }
    }
  }
  // P^T as the B operand: the S accumulator layout (row = head, columns = tokens) is exactly the
  // m16n8k16 B layout for K = tokens, N = heads
  const uint32_t pb0 = pack_half2(s[0][0], s[0][1]);
  const uint32_t pb1 = pack_half2(s[1][0], s[1][1]);
  const uint32_t pc0 = HIROWS ? pack_half2(s[0][2], s[0][3]) : 0u;
  const uint32_t pc1 = HIROWS ? pack_half2(s[1][2], s[1][3]) : 0u;

  // ---- O^T += V~^T P^T : 8 m-tiles of 16 channels.  This lane's A fragments cover channels
  // 16g..16g+15 (half word g of the bitmap) of tokens 2q, 2q+1 and 2q+8, 2q+9.
  const uint32_t vvals = smem_addr(stage + 512 + 32 * kK + (SKEW ? P.skew_k : 0));
  uint32_t va[8][4];
  if constexpr (P24) {
    // half word gq of each token: 8 values, 16 contiguous bytes at 16*gq in the token's run
#pragma unroll
    for (int pair = 0; pair < 2; ++pair) {
      uint32_t y[2][8];  // [token of the pair][channel pair 16g + 2i, +1]
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int T = 2 * qq + 8 * pair + e;
        const uint32_t bits = *reinterpret_cast<const uint16_t *>(stage + 256 + T * 16 + gq * 2);
        const uint4 v = *reinterpret_cast<const uint4 *>(stage + 512 + 2048 + (SKEW ? P.skew_k : 0) + T * 128 +
                                                         (SKEW ? (T >> P.lg_v) << 4 : 0) + gq * 16);
        const uint32_t x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint2 sel = lut24[(bits >> (4 * m)) & 15u];
          y[e][2 * m] = __byte_perm(x[m], 0u, sel.x);
          y[e][2 * m + 1] = __byte_perm(x[m], 0u, sel.y);
        }
      }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        va[mt][2 * pair] = __byte_perm(y[0][mt], y[1][mt], 0x5410);
        va[mt][2 * pair + 1] = __byte_perm(y[0][mt], y[1][mt], 0x7632);
      }
    }
  } else {
#pragma unroll
    for (int pair = 0; pair < 2; ++pair) {
      uint32_t x0[16], x1[16];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int T = 2 * qq + 8 * pair + e;
        const uint32_t bits = *reinterpret_cast<const uint16_t *>(stage + 256 + T * 16 + gq * 2);
        const uint32_t pre = *reinterpret_cast<const uint16_t *>(htab + (16 + T) * 16 + gq * 2);
        expand_half(bits, vvals + (SCAN ? 0 : 2 * T * kV + (SKEW ? (T >> P.lg_v) << 4 : 0)) + 2 * pre, za,
                    e ? x1 : x0);
      }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        va[mt][2 * pair] = __byte_perm(x0[2 * mt], x1[2 * mt], 0x5410);
        va[mt][2 * pair + 1] = __byte_perm(x0[2 * mt + 1], x1[2 * mt + 1], 0x5410);
      }
    }
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const uint32_t a[4] = {va[mt][0], va[mt][1], va[mt][2], va[mt][3]};
    mma_f16_16816(acc.ot[mt], a, pb0, pb1);
    if constexpr (HIROWS) mma_f16_16816(acc.oh[mt], a, pc0, pc1);
  }
}

// Write the merged row r (out, lse) of q head hq from its (m, l, o[c]) sums.
__device__ __forceinline__ void write_row(const DecodeParams &P, int64_t hq, int c, float M, float lsum, float acc) {
  P.out[hq * kHeadDim + c] = __half_as_ushort(__float2half_rn(lsum > 0.f ? __fdividef(acc, lsum) : 0.f));
  if (c == 0 && P.lse != nullptr) P.lse[hq] = lsum > 0.f ? (M + __log2f(lsum)) * 0.69314718055994531f : kNegInf;
}

// A piece of a stream that other CTAs share: this CTA's partial is in the workspace, and the
// ticket is taken when the CTA has finished its whole range.
struct Pending {
  int b, g;        // the stream
  int ca, cb;      // the CTAs holding part of it
  int first_slot;  // workspace slot of CTA ca's partial (CTA ca + j > ca uses slot 2 (ca + j))
};

// ---- thread-block clusters: barrier over all threads of the cluster (release / acquire), and loads
// from another CTA's shared memory
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t local_addr, uint32_t cta_rank) {
  uint32_t remote;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(remote) : "r"(local_addr), "r"(cta_rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];\n" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// Per-warp output rows in the merge area: channel c of (warp, head) row i at i * kMerStride +
// mer_pos(c), 16-channel groups 18 floats apart.  A lane's accumulator pair (channels 16g + 2m,
// +1 of one head) goes in with one 8-byte store, and the 16 lanes of a half warp (groups g, heads
// 2q) then hit 16 different bank pairs; unpadded rows put them on two bank pairs (8-way conflicts).
constexpr int kMerStride = 148;
__device__ __forceinline__ int mer_pos(int c) { return c + 2 * (c >> 4); }

// End of one piece [seg_a, ...) of stream st: the four warps merge their (m, l, o) in shared
// memory (`mer`: m[4][16], l[4][16], o[4][G][kMerStride] fp32).  A stream held by this CTA alone is
// written out; otherwise the CTA's partial goes to its workspace slot and the piece is queued in
// `pend`.  Called by every thread of the CTA.
template <bool HIROWS>
__device__ void flush_piece(const DecodeParams &P, Acc<HIROWS> &acc, float *mer, int warp, int lane,
                            const Stream &st, int seg_a, int u0, int U, int cta, int nctas, Pending *pend,
                            int *npend) {
  const int G = P.G, gq = lane >> 2, qq = lane & 3;
  float *sm_m = mer, *sm_l = mer + kWarps * 16, *sm_o = mer + 2 * kWarps * 16;
#pragma unroll
  for (int h = 0; h < (HIROWS ? 2 : 1); ++h) {
    acc.l_run[h] += __shfl_xor_sync(0xffffffffu, acc.l_run[h], 1);
    acc.l_run[h] += __shfl_xor_sync(0xffffffffu, acc.l_run[h], 2);
  }
  if (qq == 0) {
    if (gq < G) {
      sm_m[warp * 16 + gq] = acc.m_run[0];
      sm_l[warp * 16 + gq] = acc.l_run[0];
    }
    if (HIROWS && gq + 8 < G) {
      sm_m[warp * 16 + gq + 8] = acc.m_run[1];
      sm_l[warp * 16 + gq + 8] = acc.l_run[1];
    }
  }
  {
    const int h0 = 2 * qq, h1 = 2 * qq + 1;
    auto row = [&](int h) { return reinterpret_cast<float2 *>(sm_o + (warp * G + h) * kMerStride + 18 * gq); };
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      // accumulator rows g and g+8 are channels 16g + 2mt and 16g + 2mt + 1: mer_pos = 18g + 2mt, +1
      if (h0 < G) row(h0)[mt] = make_float2(acc.ot[mt][0], acc.ot[mt][2]);
      if (h1 < G) row(h1)[mt] = make_float2(acc.ot[mt][1], acc.ot[mt][3]);
      if constexpr (HIROWS) {
        if (h0 + 8 < G) row(h0 + 8)[mt] = make_float2(acc.oh[mt][0], acc.oh[mt][2]);
        if (h1 + 8 < G) row(h1 + 8)[mt] = make_float2(acc.oh[mt][1], acc.oh[mt][3]);
      }
    }
  }
  __syncthreads();

  if (P.clu > 0) {
    // one cluster per stream: this CTA's merged (m, l, o) replaces the per-warp states in `mer`, then,
    // after a cluster barrier, CTA rank j merges rows j, j + C, ... of the cluster's C partials through
    // distributed shared memory and writes them out; a second barrier keeps every CTA's partial alive
    // until all reads are done.  Every thread of every CTA of the cluster reaches both barriers.
    static_assert(kThreads == kHeadDim, "one thread per output channel");
    const int c = threadIdx.x;
    float pm[16], pl[16], po[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      pm[r] = kNegInf;
      pl[r] = po[r] = 0.f;
      if (r < G) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w) pm[r] = fmaxf(pm[r], sm_m[w * 16 + r]);
        if (pm[r] != kNegInf) {
#pragma unroll
          for (int w = 0; w < kWarps; ++w) {
            const float wt = fast_exp2(sm_m[w * 16 + r] - pm[r]);
            pl[r] += sm_l[w * 16 + r] * wt;
            po[r] += sm_o[(w * G + r) * kMerStride + mer_pos(c)] * wt;
          }
        }
      }
    }
    __syncthreads();  // every thread has read the per-warp states
    float *cpart = mer;  // m[16], l[16], o[G][128]
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      if (r < G) {
        cpart[32 + r * kHeadDim + c] = po[r];
        if (c == 0) {
          cpart[r] = pm[r];
          cpart[16 + r] = pl[r];
        }
      }
    }
    cluster_sync_all();
    const int C = P.clu, rank = cta % C;
    const uint32_t cbase = smem_addr(cpart);
    const int64_t hq0 = static_cast<int64_t>(st.b) * P.Hq + static_cast<int64_t>(st.g) * G;
    for (int r = rank; r < G; r += C) {
      float M = kNegInf;
      for (int j = 0; j < C; ++j) M = fmaxf(M, ld_cluster_f32(cbase + 4 * r, j));
      float lsum = 0.f, o = 0.f;
      if (M != kNegInf) {
        for (int j = 0; j < C; ++j) {
          const float wt = fast_exp2(ld_cluster_f32(cbase + 4 * r, j) - M);
          lsum += ld_cluster_f32(cbase + 4 * (16 + r), j) * wt;
          o += ld_cluster_f32(cbase + 4 * (32 + r * kHeadDim + c), j) * wt;
        }
      }
      write_row(P, hq0 + r, c, M, lsum, o);
    }
    cluster_sync_all();
    return;
  }
  // the CTAs holding part of this stream: ca .. cb (an empty range that starts exactly where
  // the stream starts belongs to no stream)
  const int ca = cta_of(st.start, U, nctas), cb = cta_of(st.end() - 1, U, nctas);
  if (cta >= ca && cta <= cb) {
    const int slot_floats = 32 + G * kHeadDim;
    const int c = threadIdx.x;  // output channel
    const int64_t hq0 = static_cast<int64_t>(st.b) * P.Hq + static_cast<int64_t>(st.g) * G;
    float *part = P.ws_part + static_cast<int64_t>(2 * cta + (seg_a == u0 ? 0 : 1)) * slot_floats;
    const int pc = mer_pos(c);
    // four rows at a time, all their shared loads issued before any result is used
    for (int r0 = 0; r0 < G; r0 += 4) {
      float M[4], lsum[4], o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = r0 + j;
        M[j] = kNegInf;
        lsum[j] = o[j] = 0.f;
        if (r < G) {
          float mw[kWarps];
#pragma unroll
          for (int w = 0; w < kWarps; ++w) {
            mw[w] = sm_m[w * 16 + r];
            M[j] = fmaxf(M[j], mw[w]);
          }
          if (M[j] != kNegInf) {
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
              const float wt = fast_exp2(mw[w] - M[j]);
              lsum[j] += sm_l[w * 16 + r] * wt;
              o[j] += sm_o[(w * G + r) * kMerStride + pc] * wt;
            }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = r0 + j;
        if (r >= G) continue;
        if (ca == cb) {
          write_row(P, hq0 + r, c, M[j], lsum[j], o[j]);
        } else {
          part[32 + r * kHeadDim + c] = o[j];
          if (c == 0) {
            part[r] = M[j];
            part[16 + r] = lsum[j];
          }
        }
      }
    }
    if (ca != cb && threadIdx.x == 0) {
      Pending &pd = pend[(*npend)++];
      pd.b = st.b;
      pd.g = st.g;
      pd.ca = ca;
      pd.cb = cb;
      pd.first_slot = 2 * ca + (range_start(ca, U, nctas) < st.start ? 1 : 0);
    }
  }
  __syncthreads();  // the merge area is reused by the next piece
}

// The last CTA of a shared stream: merge its n = cb - ca + 1 partials and write out / lse.
// Latency-bound, so every load of a block of 16 partials (their m, l and this thread's float4 of
// o) is issued before any is used; blocks are combined with an online rescale.  Thread t handles
// the (row, 4-channel quad) pairs t, t+128, ... (G <= 16 -> at most 4).
__device__ void merge_stream(const DecodeParams &P, const Pending &pd) {
  const int G = P.G, n = pd.cb - pd.ca + 1;
  const int slot_floats = 32 + G * kHeadDim;
  const int64_t hq0 = static_cast<int64_t>(pd.b) * P.Hq + static_cast<int64_t>(pd.g) * G;
  for (int it = threadIdx.x; it < G * (kHeadDim / 4); it += kThreads) {
    const int r = it >> 5, q4 = it & 31;
    float M = kNegInf, Lsum = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < n; j0 += 16) {
      float mv[16], lv[16];
      float4 ov[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int j = j0 + u;
        if (j < n) {
          const int slot = j == 0 ? pd.first_slot : 2 * (pd.ca + j);
          const float *pp = P.ws_part + static_cast<int64_t>(slot) * slot_floats;
          mv[u] = __ldcg(pp + r);
          lv[u] = __ldcg(pp + 16 + r);
          ov[u] = __ldcg(reinterpret_cast<const float4 *>(pp + 32 + r * kHeadDim) + q4);
        } else {
          mv[u] = kNegInf;
          lv[u] = 0.f;
          ov[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      float mb = M;
#pragma unroll
      for (int u = 0; u < 16; ++u) mb = fmaxf(mb, mv[u]);
      const float base = mb == kNegInf ? 0.f : mb;
      const float a = fast_exp2(M - base);
      Lsum *= a;
      o.x *= a;
      o.y *= a;
      o.z *= a;
      o.w *= a;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float wt = fast_exp2(mv[u] - base);
        Lsum += wt * lv[u];
        o.x += wt * ov[u].x;
        o.y += wt * ov[u].y;
        o.z += wt * ov[u].z;
        o.w += wt * ov[u].w;
      }
      M = mb;
    }
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    *reinterpret_cast<uint2 *>(P.out + (hq0 + r) * kHeadDim + 4 * q4) =
        make_uint2(pack_half2(o.x * inv, o.y * inv), pack_half2(o.z * inv, o.w * inv));
    if (q4 == 0 && P.lse != nullptr) P.lse[hq0 + r] = Lsum > 0.f ? (M + __log2f(Lsum)) * 0.69314718055994531f : kNegInf;
  }
}

// Ticket of a shared stream: acq_rel at gpu scope, so the release covers this CTA's partial
// stores (ordered before it by the CTA barrier) and the acquire covers the other CTAs' ones.
__device__ __forceinline__ uint32_t take_ticket(uint32_t *counter) {
  uint32_t old;
  asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;\n" : "=r"(old) : "l"(counter) : "memory");
  return old;
}

// Keep count and first packed value of stream (b, h) in one cache.  PERHEAD = false is the uniform
// cache: the keep count is the kernel parameter, so it costs no register across the chunk loop.
template <bool PERHEAD>
__device__ __forceinline__ int keep_of(const HeadKeep &hk, int keep, int h) {
  return PERHEAD ? hk.k[h] : keep;
}
template <bool PERHEAD>
__device__ __forceinline__ int64_t base_of(const HeadKeep &hk, int keep, int b, int h, int H, int cap) {
  return PERHEAD ? hk.value_base(b, h, H, cap) : (static_cast<int64_t>(b) * H + h) * cap * static_cast<int64_t>(keep);
}

// PRMT selectors that place a 2:4 nibble's two values (one 32-bit pair, lower channel first) at
// their channels: .x builds channels (0, 1), .y channels (2, 3); bytes 4-7 are the zero operand.
// Index = the nibble's 4 bits; the six 2-of-4 patterns, and 0 (a masked tail token) -> zeros.
__constant__ uint2 kLut24[16] = {
    {0x5454u, 0x5454u}, {0x5454u, 0x5454u}, {0x5454u, 0x5454u}, {0x3210u, 0x5454u},  // 0, 1, 2, 0011
    {0x5454u, 0x5454u}, {0x5410u, 0x5432u}, {0x1054u, 0x5432u}, {0x5454u, 0x5454u},  // 4, 0101, 0110, 7
    {0x5454u, 0x5454u}, {0x5410u, 0x3254u}, {0x1054u, 0x3254u}, {0x5454u, 0x5454u},  // 8, 1001, 1010, 11
    {0x5454u, 0x3210u}, {0x5454u, 0x5454u}, {0x5454u, 0x5454u}, {0x5454u, 0x5454u}};  // 1100, 13, 14, 15

template <int NSTAGE, bool HIROWS, bool PERHEAD, bool P24, bool SCAN, bool SKEW>
__global__ void __launch_bounds__(kThreads, HIROWS ? 3 : 4) sparse_decode_kernel(const DecodeParams P) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(16) uint32_t zero_slot[4];
  __shared__ int sh_len[kWarps][kRowCache];  // each warp's copy of the row-length cache
  __shared__ int sh_pos[kRowCache];  // fused step: the new token's position in each row
  __shared__ uint32_t sh_bits;       // device error flags of the cached rows this CTA reports
  __shared__ Pending sh_pend[2];
  __shared__ int sh_npend, sh_last[2];
  __shared__ uint2 lut24[16];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x, nctas = gridDim.x;
  const int cap = min(P.cap_k, P.cap_v);

  uint8_t *wbase = smem + warp * P.warp_bytes;
  uint8_t *htab = wbase + NSTAGE * P.stage_bytes;  // [32 rows][8 half words] u16 prefixes
  const uint32_t bars = smem_addr(htab + 512);     // NSTAGE mbarriers of this warp
  float *mer = reinterpret_cast<float *>(smem + kWarps * P.warp_bytes);
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < NSTAGE; ++i) mbar_init(bars + 8 * i, 1);
    mbar_init_fence();
  }

  // ---- the end-to-end chunk sequence: its length U and where this CTA's range starts.  Every warp
  // computes them itself (the same values), so that it can fill its copy ring without waiting for the
  // others: it reads the lengths of rows below kRowCache in one round of independent loads into its
  // own copy of the row cache (warp 0 also collects the error flags of the rows this CTA reports);
  // longer batches read the rest from global memory.  With one cluster per stream, the cluster's C
  // CTAs split that stream's chunks evenly and nothing else.
  int *const my_len = sh_len[warp];
  int U, u0, u1, row, row_start;  // row: batch row of the CTA's first unit (-1: none); row_start: its first unit
  {
    int nrow[kRowCache / 32];
    int tot = 0;
    uint32_t bits = 0;
#pragma unroll
    for (int i = 0; i < kRowCache / 32; ++i) {
      const int b = lane + 32 * i;
      int L = 0;
      if (b < P.B) {
        uint32_t rb = 0;
        L = row_len(P, b, cap, rb);
        my_len[b] = L;
        if (warp == 0) {
          if (P.pos != nullptr) sh_pos[b] = P.pos[b];
          if (b % nctas == cta) bits |= rb;
        }
      }
      nrow[i] = P.Hkv * n_chunks(L);
      tot += nrow[i];
    }
    if (warp == 0) {
      bits = __reduce_or_sync(0xffffffffu, bits);
      if (lane == 0) sh_bits = bits;
    }
    __syncwarp();  // this warp's row cache is complete
    if (P.clu > 0) {
      // units are counted from the stream's first chunk; row_start holds the stream's kv head
      const int s = cta / P.clu, r = cta % P.clu;
      row = s / P.Hkv;
      row_start = s % P.Hkv;
      const int n = n_chunks(len_of(P, my_len, row, cap));
      U = 0;
      u0 = r * n / P.clu;
      u1 = (r + 1) * n / P.clu;
    } else {
      for (int b = kRowCache + lane; b < P.B; b += 32) tot += P.Hkv * n_chunks(row_len(P, b, cap));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
      U = tot;
      u0 = range_start(cta, tot, nctas);
      u1 = range_start(cta + 1, tot, nctas);
      row = -1;
      row_start = 0;
      int before = 0;
      for (int b0 = 0; b0 < P.B && u0 < tot; b0 += 32) {
        const int b = b0 + lane;
        int n;
        if (b0 < kRowCache) {
          const int i = b0 >> 5;
          n = i == 0 ? nrow[0] : i == 1 ? nrow[1] : i == 2 ? nrow[2] : nrow[3];
        } else {
          n = b < P.B ? P.Hkv * n_chunks(row_len(P, b, cap)) : 0;
        }
        int incl = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, before + incl > u0);
        if (hit != 0u) {
          const int f = __ffs(hit) - 1;
          row = b0 + f;
          row_start = before + __shfl_sync(0xffffffffu, incl - n, f);
          break;
        }
        before += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
  }

  Stream first;
  first.b = row;
  first.n = row >= 0 ? n_chunks(len_of(P, my_len, row, cap)) : 0;
  if (P.clu > 0) {
    first.g = row_start;
    first.start = 0;
  } else {
    first.g = row >= 0 ? (u0 - row_start) / first.n : 0;
    first.start = row_start + first.g * first.n;
  }

  // ---- the warp's chunks: units u0 + warp + 4j of the range, through a ring of NSTAGE buffers
  const uint32_t za = smem_addr(zero_slot);
  // producer state of each warp in shared memory (only lane 0 walks it), to keep registers for
  // the chunk math: the stream of the next unit to copy in, and that unit
  __shared__ Stream sh_ps[kWarps];
  __shared__ int sh_punit[kWarps];
  if (lane == 0) {
    sh_ps[warp] = first;
    sh_punit[warp] = u0 + warp;
  }
  __syncwarp();
  // the four copies of unit punit of stream ps into ring buffer `slot` (lane 0; not the SKEW staging)
  auto issue = [&](const Stream &ps, int punit, int slot) {
    const uint32_t dst = smem_addr(wbase + slot * P.stage_bytes);
    const uint32_t bar = bars + 8 * slot;
    const int64_t sid = static_cast<int64_t>(ps.b) * P.Hkv + ps.g;
    const int64_t t0 = static_cast<int64_t>(punit - ps.start) * kChunk;
    const int64_t tk = sid * P.cap_k + t0, tv = sid * P.cap_v + t0;
    if constexpr (PERHEAD) {
      const int kK = P.hk_k.k[ps.g], kV = P.hk_v.k[ps.g];
      mbar_expect_tx(bar, 512 + 32 * (kK + kV));
      bulk_g2s(dst, P.kbm + tk * kWords, 256, bar);
      bulk_g2s(dst + 256, P.vbm + tv * kWords, 256, bar);
      bulk_g2s(dst + 512, P.kval + P.hk_k.value_base(ps.b, ps.g, P.Hkv, P.cap_k) + t0 * kK, 32 * kK, bar);
      bulk_g2s(dst + 512 + 32 * kK, P.vval + P.hk_v.value_base(ps.b, ps.g, P.Hkv, P.cap_v) + t0 * kV, 32 * kV, bar);
    } else {  // stream (b, h) of a uniform cache starts at (b*H + h) * cap * keep
      mbar_expect_tx(bar, 512 + 32 * (P.keep_k + P.keep_v));
      bulk_g2s(dst, P.kbm + tk * kWords, 256, bar);
      bulk_g2s(dst + 256, P.vbm + tv * kWords, 256, bar);
      bulk_g2s(dst + 512, P.kval + tk * P.keep_k, 32 * P.keep_k, bar);
      bulk_g2s(dst + 512 + 32 * P.keep_k, P.vval + tv * P.keep_v, 32 * P.keep_v, bar);
    }
  };
  auto produce = [&](int item) {
    if constexpr (SKEW) {
      // a cache whose keep is a multiple of 32 is staged in groups of 2^lg tokens (about 256 bytes),
      // each group 16 bytes after the previous one ends: otherwise every token's run starts on the
      // same bank and the lanes that read one word position of eight tokens collide.  Lanes 0-15
      // copy K groups, 16-31 V groups; a cache without skew (lg = 4) arrives in one copy.
      const int punit = sh_punit[warp];
      if (punit >= u1) return;  // the same in every lane
      Stream ps = sh_ps[warp];
      while (punit >= ps.end()) next_stream(P, my_len, cap, ps);
      const int slot = item % NSTAGE;
      const uint32_t dst = smem_addr(wbase + slot * P.stage_bytes);
      const uint32_t bar = bars + 8 * slot;
      const int64_t sid = static_cast<int64_t>(ps.b) * P.Hkv + ps.g;
      const int64_t t0 = static_cast<int64_t>(punit - ps.start) * kChunk;
      const int64_t tk = sid * P.cap_k + t0, tv = sid * P.cap_v + t0;
      if (lane == 0) {
        mbar_expect_tx(bar, 512 + 32 * (P.keep_k + P.keep_v));
        bulk_g2s(dst, P.kbm + tk * kWords, 256, bar);
        bulk_g2s(dst + 256, P.vbm + tv * kWords, 256, bar);
      }
      __syncwarp();
      const bool kside = lane < 16;
      const int g = lane & 15, keep = kside ? P.keep_k : P.keep_v, lg = kside ? P.lg_k : P.lg_v;
      const uint32_t base = dst + 512 + (kside ? 0 : 32 * P.keep_k + P.skew_k);
      const uint16_t *src = kside ? P.kval + tk * P.keep_k : P.vval + tv * P.keep_v;
      if (g < (kChunk >> lg))  // group g: tokens g*2^lg .. (g+1)*2^lg - 1
        bulk_g2s(base + ((2 * keep) << lg) * g + 16 * g, src + (keep << lg) * g, (2 * keep) << lg, bar);
      __syncwarp();  // every lane has read the producer state before lane 0 moves it on
      if (lane == 0) {
        sh_ps[warp] = ps;
        sh_punit[warp] = punit + kWarps;
      }
      return;
    }
    if (lane != 0) return;
    int punit = sh_punit[warp];
    if (punit >= u1) return;
    Stream ps = sh_ps[warp];
    while (punit >= ps.end()) next_stream(P, my_len, cap, ps);
    issue(ps, punit, item % NSTAGE);
    sh_ps[warp] = ps;
    sh_punit[warp] = punit + kWarps;
  };
  // fill the copy ring with the warp's first NSTAGE units
  auto fill = [&]() {
    if constexpr (SKEW) {
#pragma unroll 1
      for (int i = 0; i < NSTAGE; ++i) produce(i);
    } else {
      // lane 0 walks the streams in registers and issues every item in one pass (the chunk loop's
      // producer keeps its state in shared memory to spare registers)
      if (lane == 0) {
        Stream ps = first;
        int punit = u0 + warp;
#pragma unroll 1
        for (int i = 0; i < NSTAGE && punit < u1; ++i, punit += kWarps) {
          while (punit >= ps.end()) next_stream(P, my_len, cap, ps);
          issue(ps, punit, i);
        }
        sh_ps[warp] = ps;
        sh_punit[warp] = punit;
      }
      __syncwarp();
    }
  };
  // attention alone: fill the ring before waiting for the other warps (a fused step fills it after
  // the new tokens are in the caches, below)
  if (P.pos == nullptr && row >= 0) fill();

  if (threadIdx.x < 4) zero_slot[threadIdx.x] = 0u;
  if (threadIdx.x == 0) sh_npend = 0;
  if (P24 && threadIdx.x < 16) lut24[threadIdx.x] = kLut24[threadIdx.x];
  __syncthreads();

  // ---- rows this CTA reports on: device error flags, and the output of rows with no tokens
  uint32_t bits = sh_bits;
  for (int b = cta; b < P.B; b += nctas) {
    const int L = b < kRowCache ? my_len[b] : row_len(P, b, cap, bits);
    if (L == 0) {
      uint16_t *o = P.out + static_cast<int64_t>(b) * P.Hq * kHeadDim;
      for (int i = threadIdx.x; i < P.Hq * kHeadDim; i += kThreads) o[i] = 0;
      if (P.lse != nullptr)
        for (int i = threadIdx.x; i < P.Hq; i += kThreads) P.lse[static_cast<int64_t>(b) * P.Hq + i] = kNegInf;
    }
  }
  if (threadIdx.x == 0 && bits != 0u && P.err != nullptr) atomicOr(P.err, bits);
  if (row < 0) return;  // an empty range at the end of the sequence (never with clusters)

  // ---- fused decode step: compress the new token of every stream whose new-token chunk lies in
  // this range (warp 0: K, warp 1: V) before any chunk is copied in
  if (P.pos != nullptr) {
    Stream st = first;
    bool any = false;
    while (st.start < u1) {
      const int p = st.b < kRowCache ? sh_pos[st.b] : P.pos[st.b];
      if (st.n > 0 && p >= 0 && p < cap) {
        const int unit = st.start + p / kChunk;
        if (unit >= u0 && unit < u1) {
          any = true;
          if (warp < 2) {
            const bool kside = warp == 0;
            const uint16_t *src =
                kside ? P.kn + st.b * P.kn_sb + st.g * P.kn_sh : P.vn + st.b * P.vn_sb + st.g * P.vn_sh;
            const int capx = kside ? P.cap_k : P.cap_v;
            const int keep = kside ? keep_of<PERHEAD>(P.hk_k, P.keep_k, st.g) : keep_of<PERHEAD>(P.hk_v, P.keep_v, st.g);
            const int64_t base = kside ? base_of<PERHEAD>(P.hk_k, P.keep_k, st.b, st.g, P.Hkv, capx)
                                       : base_of<PERHEAD>(P.hk_v, P.keep_v, st.b, st.g, P.Hkv, capx);
            // a channel-wise cache got its new token from a separate launch before this one (its whole
            // window is pruned again, which would weigh on this kernel's registers)
            if (!SCAN || (kside ? P.kwin : P.vwin) == nullptr) {
              const int64_t sid = static_cast<int64_t>(st.b) * P.Hkv + st.g;
              uint32_t *bm = const_cast<uint32_t *>(kside ? P.kbm : P.vbm) + (sid * capx + p) * kWords;
              uint16_t *vals = const_cast<uint16_t *>(kside ? P.kval : P.vval) + base + static_cast<int64_t>(p) * keep;
              if (kside ? P.p24_k : P.p24_v)
                warp_compress_vector_24(src, bm, vals, lane);
              else
                warp_compress_vector(src, keep, bm, vals, lane);
            }
          }
        }
      }
      if (!next_stream(P, my_len, cap, st)) break;
    }
    if (any) {
      fence_proxy_async_global();  // these stores before the bulk copies that read them
      __syncthreads();
    }
    fill();
  }


  Stream cs = first;
  int cunit = u0 + warp, citem = 0;
  bool timed_out = false;
  Acc<HIROWS> acc;
  uint32_t qa[8][4];
  for (;;) {
    const int seg_a = max(cs.start, u0), seg_e = min(cs.end(), u1);
    const int L = len_of(P, my_len, cs.b, cap);
    const int kK = keep_of<PERHEAD>(P.hk_k, P.keep_k, cs.g), kV = keep_of<PERHEAD>(P.hk_v, P.keep_v, cs.g);
    load_q<HIROWS>(P, cs.b, cs.g, lane, qa);
    acc.reset();
#pragma unroll 1
    for (; cunit < seg_e; cunit += kWarps, ++citem) {
      const int slot = citem % NSTAGE;
      uint8_t *stage = wbase + slot * P.stage_bytes;
      if (!mbar_wait(bars + 8 * slot, (citem / NSTAGE) & 1, timed_out ? kWaitCyclesAfter : kWaitCycles))
        timed_out = true;
      consume_chunk<HIROWS, PERHEAD, P24, SCAN, SKEW>(P, stage, htab, za, (cunit - cs.start) * kChunk, L, kK, kV, lane, qa, acc,
                                          lut24);
      __syncwarp();
      produce(citem + NSTAGE);  // the unit NSTAGE items ahead goes into the buffer just read
    }
    flush_piece<HIROWS>(P, acc, mer, warp, lane, cs, seg_a, u0, U, cta, nctas, sh_pend, &sh_npend);
    if (seg_e >= u1) break;
    bool more;
    do {
      more = next_stream(P, my_len, cap, cs);
    } while (more && cs.n == 0);
    if (!more) break;
  }
  if (timed_out) {
    // a copy that did not land in time may still be in flight into this warp's buffers: before the CTA
    // can exit (and its shared memory be reused), wait once more, again bounded, for the latest copy
    // issued into each buffer of the ring
    if (lane == 0 && P.err != nullptr) atomicOr(P.err, MUSTAFAR_DEVERR_TIMEOUT);
#pragma unroll 1
    for (int s = 0; s < NSTAGE && s < citem; ++s) {
      const int last = s + NSTAGE * ((citem - 1 - s) / NSTAGE);  // the latest item that used buffer s
      mbar_wait(bars + 8 * s, (last / NSTAGE) & 1, kWaitCyclesAfter);
    }
  }

  // ---- tickets for the pieces shared with other CTAs; the last CTA of a stream merges it
  const int np = sh_npend;  // the partial stores are ordered before this by flush_piece's barrier
  if (np > 0) {
    if (threadIdx.x == 0)
      for (int i = 0; i < np; ++i)
        sh_last[i] = take_ticket(P.ws_cnt + sh_pend[i].b * P.Hkv + sh_pend[i].g) ==
                     static_cast<uint32_t>(sh_pend[i].cb - sh_pend[i].ca);
    __syncthreads();
    for (int i = 0; i < np; ++i) {
      if (!sh_last[i]) continue;
      merge_stream(P, sh_pend[i]);
      if (threadIdx.x == 0) P.ws_cnt[sh_pend[i].b * P.Hkv + sh_pend[i].g] = 0u;  // ready for the next call
    }
  }
}

// ------------------------------------------------------------------------------------ host side
using SparseFn = void (*)(const DecodeParams);

template <int NSTAGE, bool PERHEAD, bool P24, bool SCAN, bool SKEW>
SparseFn pick_rows(bool hirows) {
  return hirows ? sparse_decode_kernel<NSTAGE, true, PERHEAD, P24, SCAN, SKEW>
                : sparse_decode_kernel<NSTAGE, false, PERHEAD, P24, SCAN, SKEW>;
}

template <bool PERHEAD, bool P24, bool SCAN, bool SKEW>
SparseFn pick_stages(int nstage, bool hirows) {
  switch (nstage) {
    case 2: return pick_rows<2, PERHEAD, P24, SCAN, SKEW>(hirows);
    case 3: return pick_rows<3, PERHEAD, P24, SCAN, SKEW>(hirows);
    default: return pick_rows<4, PERHEAD, P24, SCAN, SKEW>(hirows);
  }
}

// variant: 0 uniform caches, 1 a keep count per kv head, 2 both caches 2:4, 3 token runs found by
// popcount prefixes (a channel-wise cache; either cache may also be token-wise or 2:4); 4 is 0 with
// a cache staged in skewed token groups (keep a multiple of 32)
SparseFn pick_sparse(int nstage, bool hirows, int variant) {
  switch (variant) {
    case 1: return pick_stages<true, false, false, false>(nstage, hirows);
    case 2: return pick_stages<false, true, false, false>(nstage, hirows);
    case 3: return pick_stages<false, false, true, false>(nstage, hirows);
    case 4: return pick_stages<false, false, false, true>(nstage, hirows);
    default: return pick_stages<false, false, false, false>(nstage, hirows);
  }
}

// ensure_smem_limit / occupancy cache slots 12..41, one per kernel (compress and the dense kernel
// use 0..9)
int sparse_slot(int nstage, bool hirows, int variant) { return 12 + 6 * variant + 2 * (nstage - 2) + (hirows ? 1 : 0); }

constexpr int kMinUnitsPerCta = 2 * kWarps;  // at least two chunks per warp (more CTAs per stream cost more merging)
constexpr int kMaxCtasPerSm = 4;
constexpr int kCtaSmemBudget = 56000;        // four CTAs per SM fit in 228 KB with this much each

int round_up(int x, int m) { return (x + m - 1) / m * m; }

int sms_of_current_device() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) return 148;
  if (dev >= 0 && dev < 64) cached[dev] = sms;
  return sms;
}

// resident CTAs per SM, cached per (device, kernel, smem) so that planning stays capture-safe
cudaError_t resident_ctas(SparseFn fn, int slot, int smem, int *per_sm) {
  static int cache_smem[64][kKernelSlots];
  static int cache_val[64][kKernelSlots];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cacheable = dev >= 0 && dev < 64 && slot >= 0 && slot < kKernelSlots;
  if (cacheable && cache_smem[dev][slot] == smem && cache_val[dev][slot] > 0) {
    *per_sm = cache_val[dev][slot];
    return cudaSuccess;
  }
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, fn, kThreads, smem);
  if (e == cudaSuccess && cacheable) {
    cache_smem[dev][slot] = smem;
    cache_val[dev][slot] = *per_sm;
  }
  return e;
}

// Whether `clusters` clusters of C CTAs of this kernel (one per stream) are resident on the device at
// once, cached per (device, kernel, C) with the shared memory it was asked for, so that planning stays
// capture-safe once warm.  Sizes above 8 need the kernel's non-portable cluster attribute, set here.
bool clusters_fit(SparseFn fn, int slot, int smem, int C, int clusters) {
  constexpr int kDevs = 16, kMaxC = 16;
  static int cache_smem[kDevs][kKernelSlots][kMaxC + 1];
  static int cache_val[kDevs][kKernelSlots][kMaxC + 1];
  int dev = 0;
  if (C < 2 || C > kMaxC || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevs || slot < 0 ||
      slot >= kKernelSlots)
    return false;
  if (cache_smem[dev][slot][C] != smem) {
    int n = 0;
    if (C > 8 && cudaFuncSetAttribute(reinterpret_cast<const void *>(fn), cudaFuncAttributeNonPortableClusterSizeAllowed,
                                      1) != cudaSuccess) {
      (void)cudaGetLastError();
      n = -1;
    }
    if (n == 0) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(static_cast<unsigned>(C));
      cfg.blockDim = dim3(kThreads);
      cfg.dynamicSmemBytes = static_cast<size_t>(smem);
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = static_cast<unsigned>(C);
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = -1;
      }
    }
    cache_smem[dev][slot][C] = smem;
    cache_val[dev][slot][C] = n;
  }
  return cache_val[dev][slot][C] >= clusters;
}

}  // namespace

int sparse_decode_ctas(int B, int Hkv, int max_len, int forced_splits, int per_sm) {
  const long long streams = static_cast<long long>(B) * Hkv;
  const long long units = streams * ((max_len + kChunk - 1) / kChunk);
  long long ctas;
  if (forced_splits > 0) {
    ctas = forced_splits * streams;
  } else {
    // one wave; when a whole number of CTAs per stream fills nearly all of it, take that, so that
    // (for equal row lengths) no range crosses a stream boundary and no piece needs an extra merge
    const long long wave = static_cast<long long>(sms_of_current_device()) * per_sm;
    const long long per_stream = wave / streams;
    ctas = per_stream >= 1 && per_stream * streams * 20 >= wave * 19 ? per_stream * streams : wave;
    // short rows: about two chunks per warp, but never fewer CTAs than streams (up to a wave): the
    // four warps of a CTA step through its stream pieces together, so a CTA holding many one-chunk
    // pieces would run them one after another
    long long by_len = units / kMinUnitsPerCta;
    const long long spread = streams < wave ? streams : wave;
    by_len = by_len > spread ? by_len : spread;
    ctas = by_len < ctas ? by_len : ctas;
  }
  ctas = ctas > units ? units : ctas;
  ctas = ctas > (1 << 20) ? (1 << 20) : ctas;
  return ctas < 1 ? 1 : static_cast<int>(ctas);
}

size_t sparse_workspace_bytes(int B, int Hkv, int G, int ctas) {
  const size_t cnt = ((static_cast<size_t>(B) * Hkv * 4 + 255) / 256) * 256;
  return cnt + static_cast<size_t>(2) * ctas * (32 + static_cast<size_t>(G) * kHeadDim) * 4;
}

size_t sparse_workspace_bound(int B, int Hkv, int G, int max_len, int forced_splits) {
  return sparse_workspace_bytes(B, Hkv, G, sparse_decode_ctas(B, Hkv, max_len, forced_splits, kMaxCtasPerSm));
}

cudaError_t plan_sparse(int B, int Hkv, int G, int max_len, int keep_k, int keep_v, int forced_splits, int variant,
                        DecodePlan *plan) {
  const bool hirows = G > 8;
  // a uniform or 2:4 cache whose keep is a multiple of 32 is staged token by token with a 16-byte
  // skew (see the producer); its staged run then takes 2*keep + 16 bytes per token
  // (not for 2:4: its 128-bit loads see at most 2-way conflicts, and the grouped staging cost more
  // than it saved there, measured)
  const bool can_skew = variant == 0;
  // tokens per staged group, as log2 (4 = the chunk in one copy, no skew).  Keeps of 96 and 128 are
  // staged token by token: there eight tokens' runs share one or two bank offsets (s = 0: 1.2-1.8x).
  // Keep 64 goes in 4-token groups when the other cache's keep is also a multiple of 32 (s = 0.5:
  // 1.05-1.10x); paired with an unskewed cache the grouped copies measured 4 % slower.  Smaller keeps
  // have short runs and stay in one copy.
  auto group_lg = [&](int keep, int other) {
    if (!can_skew || keep % 32 != 0) return 4;
    if (keep >= 96) return 0;
    return keep == 64 && other % 32 == 0 ? 2 : 4;
  };
  plan->lg_k = group_lg(keep_k, keep_v);
  plan->lg_v = group_lg(keep_v, keep_k);
  plan->skew_k = plan->lg_k < 4 ? 16 * (kChunk >> plan->lg_k) : 0;  // skew bytes added to the region
  plan->skew_v = plan->lg_v < 4 ? 16 * (kChunk >> plan->lg_v) : 0;
  if (plan->skew_k || plan->skew_v) variant = 4;
  const int stage_bytes = round_up(512 + 32 * (keep_k + keep_v) + plan->skew_k + plan->skew_v, 128);
  const int merge_bytes = (2 * kWarps * 16 + kWarps * G * kMerStride) * 4;
  auto warp_bytes_of = [&](int ns) { return round_up(ns * stage_bytes + 512 + 8 * ns, 128); };
  int nstage = 2;
  for (int ns = 4; ns > 2; --ns)
    if (kWarps * warp_bytes_of(ns) + merge_bytes <= kCtaSmemBudget) {
      nstage = ns;
      break;
    }
  const int warp_bytes = warp_bytes_of(nstage);
  const int smem = kWarps * warp_bytes + merge_bytes;
  SparseFn fn = pick_sparse(nstage, hirows, variant);
  const int slot = sparse_slot(nstage, hirows, variant);
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(fn), slot, smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = resident_ctas(fn, slot, smem, &per_sm);
  if (e != cudaSuccess) return e;
  per_sm = per_sm < 1 ? 1 : (per_sm > kMaxCtasPerSm ? kMaxCtasPerSm : per_sm);
  plan->splits = sparse_decode_ctas(B, Hkv, max_len, forced_splits, per_sm);
  plan->chunks_per_split = 0;
  // the automatic plan gives every stream the same whole number C of CTAs when that fills the wave;
  // then each stream's CTAs form one thread-block cluster that merges its partials in distributed
  // shared memory (no global partials, no tickets), provided all the clusters are resident at once
  plan->clu = 0;
  const long long streams = static_cast<long long>(B) * Hkv;
  if (forced_splits <= 0 && plan->splits % streams == 0) {
    const int C = static_cast<int>(plan->splits / streams);
    if (C >= 2 && C <= 16 && clusters_fit(fn, slot, smem, C, static_cast<int>(streams))) plan->clu = C;
  }
  plan->nstage = nstage;
  plan->stage_bytes = stage_bytes;
  plan->warp_bytes = warp_bytes;
  plan->smem_bytes = smem;
  plan->variant = variant;
  return cudaSuccess;
}

cudaError_t launch_sparse(const DecodeParams &p, const DecodePlan &plan, cudaStream_t stream) {
  SparseFn fn = pick_sparse(plan.nstage, p.G > 8, plan.variant);
  if (plan.clu > 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(plan.splits));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(plan.smem_bytes);
    cfg.stream = stream;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = static_cast<unsigned>(plan.clu);
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fn, p);
  }
  fn<<<plan.splits, kThreads, plan.smem_bytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mustafar
