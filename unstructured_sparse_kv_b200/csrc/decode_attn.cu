// decode_attn.cu - dense fp16 decode attention: the baseline the pages compare the sparse
// kernel against (MUSTAFAR summary, atlas.scime.ai, "Experimental setup": dense attention over
// uncompressed caches).  Same math as the sparse kernel, over [B][Hkv][cap][128] fp16 caches:
//   out = softmax(scale * q K^T) V
//
// Work decomposition:
// * grid = (splits, Hkv, B); a CTA owns a contiguous range of 16-token chunks of one
//   (b, kv head) stream and the whole GQA group of that kv head.
// * each of the CTA's 4 warps is an independent pipeline over every 4th chunk of the range: a
//   cp.async ring (NSTAGE deep) stages the chunk's 16 K rows and 16 V rows (padded to 272 B)
//   in the warp's own shared memory, so the loop needs no CTA barrier.
// * S = Q K^T and O^T += V^T P^T run as mma.sync m16n8k16 (fp16 in, fp32 accumulate) on
//   ldmatrix (K) / ldmatrix.trans (V) fragments: S has the G q heads (padded to 16) as M and
//   the 16 tokens as N; O^T has the 128 channels as M (8 m-tiles), the heads as N and the
//   tokens as K.  Online softmax per head, log2 domain.
// * warps merge in shared memory; with splits > 1 each CTA writes its (m, l, o) partial to the
//   workspace and the last CTA of the stream (atomic ticket, no spin-wait) merges all splits in
//   a fixed order and writes out / lse.
#include <cfloat>

#include "common.cuh"
#include "internal.h"

namespace mustafar {

constexpr int kDecodeWarps = 4;
constexpr int kDecodeThreads = 32 * kDecodeWarps;
constexpr float kNegInf = -INFINITY;

__device__ __forceinline__ void issue_chunk(const DecodeParams &P, int64_t stream, int c, uint8_t *stage,
                                            int lane) {
  const int64_t row0 = (stream * P.cap_k + static_cast<int64_t>(c) * kChunk) * kHeadDim;
  const uint8_t *src_k = reinterpret_cast<const uint8_t *>(P.kd + row0);
  const uint8_t *src_v = reinterpret_cast<const uint8_t *>(P.vd + row0);
  const uint32_t dst = smem_addr(stage);
#pragma unroll
  for (int i = 0; i < 8; ++i) {  // 256 units of 16 B per tile, 8 per lane
    const int u = lane + 32 * i;
    const int r = u >> 4, j = u & 15;
    cp_async16(dst + r * kRowBytes + j * 16, src_k + u * 16);
    cp_async16(dst + kTileBytes + r * kRowBytes + j * 16, src_v + u * 16);
  }
}

template <int NSTAGE, bool HIROWS>
__global__ void __launch_bounds__(kDecodeThreads, 3) dense_decode_kernel(const DecodeParams P) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int G = P.G;
  const int cap = P.cap_k;
  int L;
  {
    L = P.seq_len[b];
    if (L < 0 || L > cap) {
      if (threadIdx.x == 0 && split == 0 && g == 0 && P.err != nullptr) atomicOr(P.err, MUSTAFAR_DEVERR_LEN_RANGE);
      L = L < 0 ? 0 : cap;
    }
  }
  const int nch = (L + kChunk - 1) / kChunk;
  if (nch > P.num_splits * P.chunks_per_split && threadIdx.x == 0 && split == 0 && P.err != nullptr)
    atomicOr(P.err, MUSTAFAR_DEVERR_LEN_RANGE);  // the row is longer than max_len: its tail is not covered
  const int c_begin = split * P.chunks_per_split;
  const int c_end = min(nch, c_begin + P.chunks_per_split);
  const int my_n = (c_end - c_begin > warp) ? (c_end - c_begin - warp + kDecodeWarps - 1) / kDecodeWarps : 0;
  const int64_t stream = static_cast<int64_t>(b) * P.Hkv + g;

  uint8_t *wbase = smem + warp * P.warp_bytes;

  // Q A-fragments (rows = q heads of the group, zero beyond G), 8 k-steps, natural channel order.
  const int gq = lane >> 2, qq = lane & 3;
  uint32_t qa[8][4];
  {
    const uint16_t *qb = P.q + (static_cast<int64_t>(b) * P.Hq + static_cast<int64_t>(g) * G) * kHeadDim;
    const bool r0 = gq < G, r1 = HIROWS && (gq + 8 < G);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int c0 = ks * 16 + 2 * qq;
      const int c1 = c0 + 8;
      qa[ks][0] = r0 ? *reinterpret_cast<const uint32_t *>(qb + gq * kHeadDim + c0) : 0u;
      qa[ks][1] = r1 ? *reinterpret_cast<const uint32_t *>(qb + (gq + 8) * kHeadDim + c0) : 0u;
      qa[ks][2] = r0 ? *reinterpret_cast<const uint32_t *>(qb + gq * kHeadDim + c1) : 0u;
      qa[ks][3] = r1 ? *reinterpret_cast<const uint32_t *>(qb + (gq + 8) * kHeadDim + c1) : 0u;
    }
  }

  // O^T accumulators, m-tile mt: rows g / g+8 are channels 16mt+g / 16mt+g+8.  Columns 2q, 2q+1
  // are heads; oh holds heads 8+2q, 8+2q+1.
  float ot[8][4];
  float oh[HIROWS ? 8 : 1][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) ot[i][0] = ot[i][1] = ot[i][2] = ot[i][3] = 0.f;
#pragma unroll
  for (int i = 0; i < (HIROWS ? 8 : 1); ++i) oh[i][0] = oh[i][1] = oh[i][2] = oh[i][3] = 0.f;
  float m_run[2] = {kNegInf, kNegInf};
  float l_run[2] = {0.f, 0.f};

#pragma unroll
  for (int i = 0; i < NSTAGE - 1; ++i) {
    if (i < my_n) issue_chunk(P, stream, c_begin + warp + kDecodeWarps * i, wbase + i * P.stage_bytes, lane);
    cp_async_commit();
  }

  // dense path: per-lane ldmatrix row addresses (token rows (mat>>1)*8 + r, channel half mat&1)
  const int mat = lane >> 3, r8 = lane & 7;
  const uint32_t t_off = (((mat >> 1) << 3) + r8) * kRowBytes + ((mat & 1) << 4);

#pragma unroll 1
  for (int i = 0; i < my_n; ++i) {
    {
      const int ni = i + NSTAGE - 1;
      if (ni < my_n)
        issue_chunk(P, stream, c_begin + warp + kDecodeWarps * ni, wbase + (ni % NSTAGE) * P.stage_bytes,
                            lane);
      cp_async_commit();
    }
    cp_async_wait<NSTAGE - 1>();
    __syncwarp();
    uint8_t *stage = wbase + (i % NSTAGE) * P.stage_bytes;
    const int t0 = (c_begin + warp + kDecodeWarps * i) * kChunk;
    const bool full = t0 + kChunk <= L;

    // ---- S = Q K~^T for the chunk's 16 tokens (two n-tiles of 8)
    float s[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    const uint32_t kaddr = smem_addr(stage) + t_off;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(b0, b1, b2, b3, kaddr + ks * 32);
      mma_f16_16816(s[0], qa[ks], b0, b1);
      mma_f16_16816(s[1], qa[ks], b2, b3);
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
      const float m_new = fmaxf(m_run[h], mx[h]);
      const float base = m_new == kNegInf ? 0.f : m_new;
      alpha[h] = fast_exp2(m_run[h] - base);
      m_run[h] = m_new;
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
    l_run[0] = l_run[0] * alpha[0] + psum[0];
    if constexpr (HIROWS) l_run[1] = l_run[1] * alpha[1] + psum[1];
    if (__any_sync(0xffffffffu, alpha[0] != 1.f || (HIROWS && alpha[1] != 1.f))) {
      // the O^T columns this lane holds are heads 2q and 2q+1, whose factors live in lanes 8q and 8q+4
      const float a_lo = __shfl_sync(0xffffffffu, alpha[0], 8 * qq);
      const float a_hi = __shfl_sync(0xffffffffu, alpha[0], 8 * qq + 4);
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        ot[mt][0] *= a_lo;
        ot[mt][1] *= a_hi;
        ot[mt][2] *= a_lo;
        ot[mt][3] *= a_hi;
      }
      if constexpr (HIROWS) {
        const float b_lo = __shfl_sync(0xffffffffu, alpha[1], 8 * qq);
        const float b_hi = __shfl_sync(0xffffffffu, alpha[1], 8 * qq + 4);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          oh[mt][0] *= b_lo;
          oh[mt][1] *= b_hi;
          oh[mt][2] *= b_lo;
          oh[mt][3] *= b_hi;
        }
      }
    }
    // P^T as the B operand: the S accumulator layout (row = head, columns = tokens) is exactly the
    // m16n8k16 B layout for K = tokens, N = heads
    const uint32_t pb0 = pack_half2(s[0][0], s[0][1]);
    const uint32_t pb1 = pack_half2(s[1][0], s[1][1]);
    const uint32_t pc0 = HIROWS ? pack_half2(s[0][2], s[0][3]) : 0u;
    const uint32_t pc1 = HIROWS ? pack_half2(s[1][2], s[1][3]) : 0u;

    // ---- O^T += V~^T P^T : 8 m-tiles of 16 channels
    const uint32_t vaddr = smem_addr(stage + kTileBytes) + t_off;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      uint32_t a[4];
      ldmatrix_x4_trans(a[0], a[1], a[2], a[3], vaddr + mt * 32);
      mma_f16_16816(ot[mt], a, pb0, pb1);
      if constexpr (HIROWS) mma_f16_16816(oh[mt], a, pc0, pc1);
    }
  
    __syncwarp();
  }
  cp_async_wait<0>();

#pragma unroll
  for (int h = 0; h < (HIROWS ? 2 : 1); ++h) {
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
  }

  // ---- merge the 4 warps (shared memory reused after everyone is done)
  __syncthreads();
  float *sm_m = reinterpret_cast<float *>(smem);             // [4][16]
  float *sm_l = sm_m + kDecodeWarps * 16;                     // [4][16]
  float *sm_o = sm_l + kDecodeWarps * 16;                     // [4][G][128]
  if (qq == 0) {
    if (gq < G) {
      sm_m[warp * 16 + gq] = m_run[0];
      sm_l[warp * 16 + gq] = l_run[0];
    }
    if (HIROWS && gq + 8 < G) {
      sm_m[warp * 16 + gq + 8] = m_run[1];
      sm_l[warp * 16 + gq + 8] = l_run[1];
    }
  }
  {
    const int h0 = 2 * qq, h1 = 2 * qq + 1;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      const int ch0 = 16 * mt + gq;  // channel of accumulator rows g
      const int ch1 = ch0 + 8;       // and g+8
      if (h0 < G) {
        sm_o[(warp * G + h0) * kHeadDim + ch0] = ot[mt][0];
        sm_o[(warp * G + h0) * kHeadDim + ch1] = ot[mt][2];
      }
      if (h1 < G) {
        sm_o[(warp * G + h1) * kHeadDim + ch0] = ot[mt][1];
        sm_o[(warp * G + h1) * kHeadDim + ch1] = ot[mt][3];
      }
      if constexpr (HIROWS) {
        if (h0 + 8 < G) {
          sm_o[(warp * G + h0 + 8) * kHeadDim + ch0] = oh[mt][0];
          sm_o[(warp * G + h0 + 8) * kHeadDim + ch1] = oh[mt][2];
        }
        if (h1 + 8 < G) {
          sm_o[(warp * G + h1 + 8) * kHeadDim + ch0] = oh[mt][1];
          sm_o[(warp * G + h1 + 8) * kHeadDim + ch1] = oh[mt][3];
        }
      }
    }
  }
  __syncthreads();

  const int c = threadIdx.x;  // output channel
  const int S = P.num_splits;
  for (int r = 0; r < G; ++r) {
    float M = kNegInf;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, sm_m[w * 16 + r]);
    float lsum = 0.f, acc = 0.f;
    if (M != kNegInf) {
#pragma unroll
      for (int w = 0; w < kDecodeWarps; ++w) {
        const float wt = fast_exp2(sm_m[w * 16 + r] - M);
        lsum += sm_l[w * 16 + r] * wt;
        acc += sm_o[(w * G + r) * kHeadDim + c] * wt;
      }
    }
    const int64_t hq = static_cast<int64_t>(b) * P.Hq + static_cast<int64_t>(g) * G + r;
    if (S == 1) {
      P.out[hq * kHeadDim + c] = __half_as_ushort(__float2half_rn(lsum > 0.f ? acc / lsum : 0.f));
      if (c == 0 && P.lse != nullptr) P.lse[hq] = lsum > 0.f ? (M + __log2f(lsum)) * 0.69314718055994531f : kNegInf;
    } else {
      P.ws_o[(hq * S + split) * kHeadDim + c] = acc;
      if (c == 0) *reinterpret_cast<float2 *>(P.ws_ml + (hq * S + split) * 2) = make_float2(M, lsum);
    }
  }
  if (S == 1) return;

  // ---- last CTA of this stream merges every split (no waiting: an atomic ticket)
  __threadfence();
  __syncthreads();
  __shared__ int is_last;
  if (threadIdx.x == 0) {
    const uint32_t ticket = atomicAdd(P.ws_cnt + stream, 1u);
    is_last = (ticket == static_cast<uint32_t>(S - 1));
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  for (int r = 0; r < G; ++r) {
    const int64_t hq = static_cast<int64_t>(b) * P.Hq + static_cast<int64_t>(g) * G + r;
    const float2 *ml = reinterpret_cast<const float2 *>(P.ws_ml) + hq * S;
    const float *po = P.ws_o + hq * S * kHeadDim + c;
    float M = kNegInf;
    for (int s0 = 0; s0 < S; s0 += 8) {  // 8 loads in flight per step
      float mv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) mv[j] = s0 + j < S ? __ldcg(ml + s0 + j).x : kNegInf;
#pragma unroll
      for (int j = 0; j < 8; ++j) M = fmaxf(M, mv[j]);
    }
    float lsum = 0.f, acc = 0.f;
    if (M != kNegInf) {
      for (int s0 = 0; s0 < S; s0 += 8) {
        float2 mlv[8];
        float ov[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const bool in = s0 + j < S;
          mlv[j] = in ? __ldcg(ml + s0 + j) : make_float2(kNegInf, 0.f);
          ov[j] = in ? __ldcg(po + (s0 + j) * kHeadDim) : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float wt = fast_exp2(mlv[j].x - M);
          lsum += mlv[j].y * wt;
          acc += ov[j] * wt;
        }
      }
    }
    P.out[hq * kHeadDim + c] = __half_as_ushort(__float2half_rn(lsum > 0.f ? acc / lsum : 0.f));
    if (c == 0 && P.lse != nullptr) P.lse[hq] = lsum > 0.f ? (M + __log2f(lsum)) * 0.69314718055994531f : kNegInf;
  }
  if (threadIdx.x == 0) P.ws_cnt[stream] = 0u;  // leave the workspace ready for the next call
}

// ------------------------------------------------------------------------------------ host side
namespace {

using KernelFn = void (*)(const DecodeParams);

template <int NSTAGE>
KernelFn pick_rows(bool hirows) {
  return hirows ? dense_decode_kernel<NSTAGE, true> : dense_decode_kernel<NSTAGE, false>;
}

KernelFn pick_kernel(int nstage, bool hirows) { return nstage == 2 ? pick_rows<2>(hirows) : pick_rows<3>(hirows); }

int kernel_slot(int nstage, bool hirows) { return 1 + 2 * nstage + (hirows ? 1 : 0); }

struct DeviceInfo {
  int sms = 0;
};

cudaError_t device_info(DeviceInfo *info) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static int cached_sms[64] = {0};
  if (dev >= 0 && dev < 64 && cached_sms[dev] > 0) {
    info->sms = cached_sms[dev];
    return cudaSuccess;
  }
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64) cached_sms[dev] = sms;
  info->sms = sms;
  return cudaSuccess;
}

// resident CTAs per SM for a kernel and dynamic smem size, cached per device (the query is
// made once, outside any stream capture, so planning stays capture-safe afterwards)
cudaError_t occupancy(KernelFn fn, int slot, int smem, int *per_sm) {
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
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, fn, kDecodeThreads, smem);
  if (e == cudaSuccess && cacheable) {
    cache_smem[dev][slot] = smem;
    cache_val[dev][slot] = *per_sm;
  }
  return e;
}

constexpr int kMaxSplits = 128;
constexpr int kMinChunksPerCta = 2 * kDecodeWarps;
constexpr int kMaxCtasPerSm = 4;  // the split bound assumes at most this many resident CTAs

}  // namespace

int decode_split_bound(int B, int Hkv, int max_len) {
  DeviceInfo info;
  if (device_info(&info) != cudaSuccess) info.sms = 148;
  const int nch = (max_len + kChunk - 1) / kChunk;
  const int streams = B * Hkv;
  int bound = (info.sms * kMaxCtasPerSm) / (streams > 0 ? streams : 1);
  bound = bound < 1 ? 1 : bound;
  const int by_len = nch / kMinChunksPerCta;
  bound = by_len < bound ? by_len : bound;
  bound = bound < 1 ? 1 : bound;
  return bound > kMaxSplits ? kMaxSplits : bound;
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int splits) {
  if (splits <= 1) return 256;
  const size_t cnt = ((static_cast<size_t>(B) * Hkv * 4 + 255) / 256) * 256;
  const size_t ml = ((static_cast<size_t>(B) * Hq * splits * 2 * 4 + 255) / 256) * 256;
  const size_t o = static_cast<size_t>(B) * Hq * splits * kHeadDim * 4;
  return cnt + ml + o;
}

cudaError_t plan_dense(int B, int Hkv, int G, int max_len, int forced_splits, DecodePlan *plan) {
  DeviceInfo info;
  cudaError_t e = device_info(&info);
  if (e != cudaSuccess) return e;
  const int stage_bytes = 2 * kTileBytes;
  const int nstage = 3;
  const int warp_bytes = nstage * stage_bytes;
  const int merge_bytes = kDecodeWarps * 16 * 2 * 4 + kDecodeWarps * G * kHeadDim * 4;
  int smem = kDecodeWarps * warp_bytes;
  smem = smem < merge_bytes ? merge_bytes : smem;
  const bool hirows = G > 8;
  KernelFn fn = pick_kernel(nstage, hirows);
  e = ensure_smem_limit(reinterpret_cast<const void *>(fn), kernel_slot(nstage, hirows), smem);
  if (e != cudaSuccess) return e;

  const int nch = (max_len + kChunk - 1) / kChunk;
  int splits;
  if (forced_splits > 0) {
    splits = forced_splits;
  } else {
    int per_sm = 0;
    e = occupancy(fn, kernel_slot(nstage, hirows), smem, &per_sm);
    if (e != cudaSuccess) return e;
    per_sm = per_sm < 1 ? 1 : (per_sm > kMaxCtasPerSm ? kMaxCtasPerSm : per_sm);
    const int streams = B * Hkv;
    splits = (info.sms * per_sm) / streams;  // one full wave of CTAs, no partial second wave
    const int by_len = nch / kMinChunksPerCta;
    splits = splits < by_len ? splits : by_len;
    splits = splits < 1 ? 1 : (splits > kMaxSplits ? kMaxSplits : splits);
  }
  splits = splits > nch ? nch : splits;
  splits = splits < 1 ? 1 : splits;
  const int cps = (nch + splits - 1) / splits;
  splits = cps > 0 ? (nch + cps - 1) / cps : 1;
  splits = splits < 1 ? 1 : splits;
  plan->splits = splits;
  plan->chunks_per_split = cps > 0 ? cps : 1;
  plan->nstage = nstage;
  plan->stage_bytes = stage_bytes;
  plan->warp_bytes = warp_bytes;
  plan->smem_bytes = smem;
  return cudaSuccess;
}

cudaError_t launch_dense(const DecodeParams &p, const DecodePlan &plan, cudaStream_t stream) {
  KernelFn fn = pick_kernel(plan.nstage, p.G > 8);
  dim3 grid(plan.splits, p.Hkv, p.B);
  fn<<<grid, kDecodeThreads, plan.smem_bytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mustafar
