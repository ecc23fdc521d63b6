// Exact attention, decode: one new query token per sequence over a ragged,
// packed KV cache (GQA), for sm_100a.
//
// Generating a token re-reads the whole KV cache of its sequence plus the new
// entry, so the cost is linear in the cache length and bound by memory
// bandwidth (first page, the "token generation" case; the zimaspace page's
// "Reduced IO Is Not the Same as Eliminating KV Cache" section: the cache still
// has to be read). The kernel therefore streams each byte of K and V once:
//
//   split pass   grid (nsplit, Hkv * head chunks, B); 4 consumer warps and one
//                producer warp. A CTA takes a contiguous chunk of one
//                sequence's keys for one KV head; the producer copies it into
//                shared memory with bulk asynchronous copies (a ring of 32-key
//                K and V blocks with full/empty mbarriers, so no warp waits for
//                another), and the consumers compute, for the query heads
//                sharing that KV head, the scores (16-byte vector reads, fp32
//                pair FMAs, butterfly shuffle reductions), a running softmax and
//                the weighted sum of V. It writes the chunk's normalised
//                partial output and its log-sum-exp (log2 units).
//   combine      one warp per (b, query head): merges the partials by their
//                log-sum-exp and writes O (input dtype) and LSE (natural log).
//
// Packed cache layout: sequence b starts at token offset sum_{j<b} L_j and is
// stored [Hkv][L_b][d], so one (sequence, KV head) is one contiguous run. The
// offsets come from `seqlens` on the device: for batches above 1024 sequences
// from one prefix sum per call (attn_decode_offsets_kernel below; the
// persistent pass has its own in its plan kernel), else summed by each CTA
// over at most 1024 lengths; negative lengths count as 0; an empty sequence
// gives O = 0 and LSE = -inf.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>

#include "common.cuh"

namespace eta {
namespace decode {

__device__ __forceinline__ bool warp_all_d(bool v) { return __all_sync(0xffffffffu, v); }

constexpr int kWarps = 4;                     // consumer warps
constexpr int kThreads = 32 * (kWarps + 1);   // + one producer warp
constexpr float kRescaleThreshold = 8.0f;

enum : unsigned { kSiteStage = 0x21, kSiteDrain = 0x22 };

// Ring depth in 32-key stages (d = 128; twice as many for d = 64).
#ifndef ETA_DECODE_STAGES
#define ETA_DECODE_STAGES 3
#endif

// GP: query heads per CTA (the group, padded up to 4 or 8).
template <int D, int GP>
struct DCfg {
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(GP == 4 || GP == 8, "group tile");
  static constexpr int LPR = D / 8;          // lanes per cache row (8 elements, 16 B each)
  static constexpr int NGRP = 32 / LPR;      // row groups per warp
  static constexpr int RB = LPR / GP;        // rows per group per batch
  static constexpr int R = NGRP * RB;        // keys per warp batch (= 32 / GP)
  static constexpr int BPS = 32 / (kWarps * R);  // batches per warp per stage
  static constexpr int TK = kWarps * R * BPS;    // keys per stage (32)
  static constexpr int kRowBytes = D * 2;
  static constexpr int kHalfBytes = TK * kRowBytes;  // K (or V) block of one stage
  static constexpr int kStageBytes = 2 * kHalfBytes;
  static constexpr int kStages = (D == 128) ? ETA_DECODE_STAGES : 2 * ETA_DECODE_STAGES;
  static constexpr int kBarOff = kStages * kStageBytes;
  static constexpr int kCtlOff = kBarOff + 2 * kStages * 8;  // full[S], empty[S]
  static constexpr int kXOff = kCtlOff + 32;             // per-warp exchange: 32 p + GP alpha
  static constexpr int kMiscOff = kXOff + kWarps * 64 * 4;
  static constexpr int kSmemBytes = kMiscOff + 32;
  static_assert(RB >= 1 && BPS >= 1 && TK == 32, "tiling");
  static_assert(kWarps * GP * (D + 2) * 4 <= kStages * kStageBytes, "reduction scratch");
};

struct DParams {
  const void* q;
  const void* kc;
  const void* vc;
  const int* seqlens;
  const long long* tok_off;  // [B] token offsets of the sequences, or NULL: summed per CTA
  float* part_o;    // [nsplit][B][Hq][D]
  float* part_lse;  // [nsplit][B][Hq], log2 units
  int B;
  int Hq;
  int Hkv;
  int G;       // Hq / Hkv
  int nsplit;
  int nchunk;  // ceil(G / GP)
  float scale_log2;
  uint64_t wait_ns;
  int window;  // > 0: each new token reads only the last `window` cached tokens
};

template <typename T>
__device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
template <>
__device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// bf16/fp16 x8 (one 16-byte chunk) -> four fp32 pairs.
template <typename T>
__device__ __forceinline__ void unpack8x2(const uint4& v, uint64_t (&f)[4]);

template <>
__device__ __forceinline__ void unpack8x2<__nv_bfloat16>(const uint4& v, uint64_t (&f)[4]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    f[i] = f2_make(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
}

template <>
__device__ __forceinline__ void unpack8x2<__half>(const uint4& v, uint64_t (&f)[4]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    f[i] = f2_make(x.x, x.y);
  }
}

template <int D, int GP, typename T>
__global__ void __launch_bounds__(kThreads) attn_decode_split_kernel(const DParams p) {
  using C = DCfg<D, GP>;
  constexpr int S = C::kStages;
  constexpr int LPR = C::LPR, NGRP = C::NGRP, RB = C::RB, R = C::R, BPS = C::BPS, TK = C::TK;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + S;
  CtaCtl* ctl = reinterpret_cast<CtaCtl*>(smem + C::kCtlOff);
  float* xch = reinterpret_cast<float*>(smem + C::kXOff);
  long long* misc = reinterpret_cast<long long*>(smem + C::kMiscOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int grp = lane / LPR;
  const int li = lane % LPR;
  const int split = blockIdx.x;
  const int g = blockIdx.y / p.nchunk;
  const int hc = blockIdx.y - g * p.nchunk;
  const int b = blockIdx.z;

  if (warp == 0) {
    // The sequence's token offset: computed once for the call by the offsets
    // kernel when the batch is large, else summed here (B <= 1024 lengths).
    long long acc = 0;
    if (p.tok_off == nullptr)
      for (int j = lane; j < b; j += 32) acc += max(p.seqlens[j], 0);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      misc[0] = p.tok_off != nullptr ? p.tok_off[b] : acc;
      misc[1] = max(p.seqlens[b], 0);
    }
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kWarps);
    }
    ctl->abort = 0;
    ctl->wait_ns = p.wait_ns;
    fence_mbar_init();
  }
  __syncthreads();
  const long long tok_off = misc[0];
  const int L = static_cast<int>(misc[1]);
  // Keys read: [tw, L), the whole sequence or its last `window` tokens.
  const int tw = (p.window > 0 && L > p.window) ? L - p.window : 0;
  int per = (L - tw + p.nsplit - 1) / p.nsplit;
  per = (per + TK - 1) / TK * TK;
  const int t_begin = min(L, tw + split * per);
  const int t_end = min(L, t_begin + per);
  const int nkeys = t_end - t_begin;
  const int n_iter = (nkeys + TK - 1) / TK;
  const size_t head_base = (static_cast<size_t>(tok_off) * p.Hkv + static_cast<size_t>(g) * L) * D;
  const T* kbase = reinterpret_cast<const T*>(p.kc) + head_base;
  const T* vbase = reinterpret_cast<const T*>(p.vc) + head_base;

  float m_run = -INFINITY;  // running max for head (li % GP), log2 units
  float l_lane = 0.f;       // this lane's share of the running sum for that head
  uint64_t o2[GP][4];       // output accumulators, fp32 pairs (8 dims per lane)

  if (warp == kWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < n_iter; ++it) {
        const int s = it % S;
        const int use = it / S;
        if (use > 0 && !wait_bar(&empty[s], (use - 1) & 1, ctl, kSiteStage)) break;
        const int t0 = t_begin + it * TK;
        const int nk = min(TK, t_end - t0);
        const uint32_t bytes = static_cast<uint32_t>(nk) * C::kRowBytes;
        uint8_t* dst = stages + s * C::kStageBytes;
        mbar_arrive_expect_tx(&full[s], 2 * bytes);
        bulk_load(dst, kbase + static_cast<size_t>(t0) * D, bytes, &full[s]);
        bulk_load(dst + C::kHalfBytes, vbase + static_cast<size_t>(t0) * D, bytes, &full[s]);
        issued = it + 1;
      }
      // No bulk copy may still be landing when the stages are reused or the CTA exits.
      for (int s = 0; s < S && s < issued; ++s) {
        const int last = s + S * ((issued - 1 - s) / S);
        drain_bar(&full[s], (last / S) & 1, ctl, kSiteDrain);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    // Query rows of this CTA's heads, pre-scaled by scale * log2 e.
    uint64_t qr[GP][4];
#pragma unroll
    for (int hh = 0; hh < GP; ++hh) {
      const int gi = hc * GP + hh;
      if (gi < p.G) {
        const int hq = g * p.G + gi;
        const uint4 raw = *reinterpret_cast<const uint4*>(
            reinterpret_cast<const T*>(p.q) + (static_cast<size_t>(b) * p.Hq + hq) * D + li * 8);
        unpack8x2<T>(raw, qr[hh]);
        const uint64_t sc2 = f2_make(p.scale_log2, p.scale_log2);
#pragma unroll
        for (int c = 0; c < 4; ++c) qr[hh][c] = f2_mul(qr[hh][c], sc2);
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) qr[hh][c] = f2_make(0.f, 0.f);
      }
    }
#pragma unroll
    for (int hh = 0; hh < GP; ++hh)
#pragma unroll
      for (int c = 0; c < 4; ++c) o2[hh][c] = f2_make(0.f, 0.f);
    float* xw = xch + warp * 64;
    for (int it = 0; it < n_iter; ++it) {
      const int s = it % S;
      if (!warp_all_d(wait_bar(&full[s], (it / S) & 1, ctl, kSiteStage))) break;
      const int nk = min(TK, t_end - (t_begin + it * TK));
      const uint8_t* ks = stages + s * C::kStageBytes;
      const uint8_t* vs = ks + C::kHalfBytes;
#pragma unroll
      for (int bb = 0; bb < BPS; ++bb) {
        const int rbase = (warp * BPS + bb) * R;
        // scores: partial dot products over this lane's 8 dims (fp32 pairs),
        // then a butterfly reduce-scatter over the LPR lanes of the row group.
        float v[LPR];
#pragma unroll
        for (int mm = 0; mm < RB; ++mm) {
          const int r = rbase + grp + NGRP * mm;
          const uint4 raw = *reinterpret_cast<const uint4*>(ks + r * C::kRowBytes + li * 16);
          uint64_t kf[4];
          unpack8x2<T>(raw, kf);
#pragma unroll
          for (int hh = 0; hh < GP; ++hh) {
            uint64_t acc = f2_mul(qr[hh][0], kf[0]);
            acc = f2_fma(qr[hh][1], kf[1], acc);
            acc = f2_fma(qr[hh][2], kf[2], acc);
            acc = f2_fma(qr[hh][3], kf[3], acc);
            float a0, a1;
            f2_split(acc, a0, a1);
            v[mm * GP + hh] = a0 + a1;
          }
        }
#pragma unroll
        for (int M = LPR / 2; M >= 1; M >>= 1) {
          const bool up = (li & M) != 0;
#pragma unroll
          for (int j = 0; j < M; ++j) {
            const float send = up ? v[j] : v[j + M];
            const float keep = up ? v[j + M] : v[j];
            v[j] = keep + __shfl_xor_sync(0xffffffffu, send, M);
          }
        }
        // lane li now holds the score of key (grp + NGRP * (li / GP)) for head li % GP
        const int my_row = rbase + grp + NGRP * (li / GP);
        const float sc = (my_row < nk) ? v[0] : -INFINITY;
        float bmax = sc;
#pragma unroll
        for (int M = GP; M < 32; M <<= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, M));
        const float m_new = fmaxf(m_run, bmax);
        const bool need = m_new > m_run + kRescaleThreshold;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_approx(m_run - m_new);
          m_run = m_new;
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        const float pv = ex2_approx(sc - m_use);
        l_lane = fmaf(l_lane, alpha, pv);
        xw[lane] = pv;
        if (grp == 0 && li < GP) xw[32 + li] = alpha;
        __syncwarp();
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int hh = 0; hh < GP; ++hh) {
            const float a = xw[32 + hh];
            const uint64_t a2 = f2_make(a, a);
#pragma unroll
            for (int c = 0; c < 4; ++c) o2[hh][c] = f2_mul(o2[hh][c], a2);
          }
        }
#pragma unroll
        for (int mm = 0; mm < RB; ++mm) {
          const int r = rbase + grp + NGRP * mm;
          uint64_t vf[4];
          if (r < nk) {
            const uint4 raw = *reinterpret_cast<const uint4*>(vs + r * C::kRowBytes + li * 16);
            unpack8x2<T>(raw, vf);
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) vf[c] = f2_make(0.f, 0.f);
          }
          const float* pw = xw + grp * LPR + mm * GP;
#pragma unroll
          for (int hh = 0; hh < GP; ++hh) {
            const float pm = pw[hh];
            const uint64_t p2 = f2_make(pm, pm);
#pragma unroll
            for (int c = 0; c < 4; ++c) o2[hh][c] = f2_fma(p2, vf[c], o2[hh][c]);
          }
        }
        __syncwarp();
      }
      // this warp is done with the stage
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }
  __syncthreads();
  if (ctl->abort) return;

  // Merge the row groups of each warp, then the warps of the CTA.
  float* red_m = reinterpret_cast<float*>(stages);  // [warps][GP]
  float* red_l = red_m + kWarps * GP;               // [warps][GP]
  float* red_o = red_l + kWarps * GP;               // [warps][GP][D]
  if (warp < kWarps) {
    float o[GP][8];
#pragma unroll
    for (int hh = 0; hh < GP; ++hh)
#pragma unroll
      for (int c = 0; c < 4; ++c) f2_split(o2[hh][c], o[hh][2 * c], o[hh][2 * c + 1]);
#pragma unroll
    for (int M = LPR; M < 32; M <<= 1)
#pragma unroll
      for (int hh = 0; hh < GP; ++hh)
#pragma unroll
        for (int c = 0; c < 8; ++c) o[hh][c] += __shfl_xor_sync(0xffffffffu, o[hh][c], M);
    float lt = l_lane;
#pragma unroll
    for (int M = GP; M < 32; M <<= 1) lt += __shfl_xor_sync(0xffffffffu, lt, M);
    if (grp == 0 && li < GP) {
      red_m[warp * GP + li] = m_run;
      red_l[warp * GP + li] = lt;
    }
    if (grp == 0) {
#pragma unroll
      for (int hh = 0; hh < GP; ++hh)
#pragma unroll
        for (int c = 0; c < 8; ++c) red_o[(warp * GP + hh) * D + li * 8 + c] = o[hh][c];
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < GP * D; idx += kThreads) {
    const int hh = idx / D;
    const int dim = idx - hh * D;
    const int gi = hc * GP + hh;
    if (gi >= p.G) continue;
    const int hq = g * p.G + gi;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red_m[w * GP + hh]);
    float Lsum = 0.f, acc = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float sc = ex2_approx(red_m[w * GP + hh] - M);
        Lsum = fmaf(red_l[w * GP + hh], sc, Lsum);
        acc = fmaf(red_o[(w * GP + hh) * D + dim], sc, acc);
      }
    }
    const size_t row = (static_cast<size_t>(split) * p.B + b) * p.Hq + hq;
    p.part_o[row * D + dim] = Lsum > 0.f ? acc / Lsum : 0.f;
    if (dim == 0) p.part_lse[row] = Lsum > 0.f ? M + lg2_approx(Lsum) : -INFINITY;
  }
}

// Token offsets of the packed cache for large batches: tok_off[b] = the sum
// of max(L_j, 0) over j < b, as an exclusive prefix sum in one CTA, 1024
// consecutive sequences per round (coalesced reads of seqlens, a warp scan,
// then a scan of the warp totals; the running total carries over rounds).
constexpr int kOffThreads = 1024;
constexpr int kOffsetsMinBatch = 1024;  // smaller batches sum their offsets per CTA

__global__ void __launch_bounds__(kOffThreads) attn_decode_offsets_kernel(
    const int* __restrict__ seqlens, long long* __restrict__ tok_off, int B) {
  __shared__ long long s_w[kOffThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long carry = 0;
  for (int base = 0; base < B; base += kOffThreads) {
    const int b = base + static_cast<int>(threadIdx.x);
    const long long len = b < B ? max(seqlens[b], 0) : 0;
    long long x = len;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) s_w[warp] = x;
    __syncthreads();
    if (warp == 0) {
      long long w = s_w[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      s_w[lane] = w;
    }
    __syncthreads();
    if (b < B) tok_off[b] = carry + x - len + (warp > 0 ? s_w[warp - 1] : 0);
    carry += s_w[31];
    __syncthreads();  // s_w is rewritten in the next round
  }
}

// One warp per (b, query head): merge the split partials by their LSE.
template <int D, typename T>
__global__ void __launch_bounds__(128) attn_decode_combine_kernel(const float* __restrict__ part_o,
                                                                  const float* __restrict__ part_lse,
                                                                  T* __restrict__ o,
                                                                  float* __restrict__ lse,
                                                                  int rows, int nsplit) {
  constexpr int E = D / 32;  // dims per lane
  const int w = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= rows) return;
  float mx = -INFINITY;
  for (int s = lane; s < nsplit; s += 32) mx = fmaxf(mx, part_lse[static_cast<size_t>(s) * rows + w]);
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
  float tot = 0.f;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  if (mx != -INFINITY) {
    for (int s = 0; s < nsplit; ++s) {
      const size_t row = static_cast<size_t>(s) * rows + w;
      const float wt = ex2_approx(part_lse[row] - mx);
      tot += wt;
      const float* src = part_o + row * D + lane * E;
      if constexpr (E == 4) {
        const float4 x = *reinterpret_cast<const float4*>(src);
        acc[0] = fmaf(wt, x.x, acc[0]);
        acc[1] = fmaf(wt, x.y, acc[1]);
        acc[2] = fmaf(wt, x.z, acc[2]);
        acc[3] = fmaf(wt, x.w, acc[3]);
      } else {
        const float2 x = *reinterpret_cast<const float2*>(src);
        acc[0] = fmaf(wt, x.x, acc[0]);
        acc[1] = fmaf(wt, x.y, acc[1]);
      }
    }
  }
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  T* dst = o + static_cast<size_t>(w) * D + lane * E;
  if constexpr (E == 4) {
    uint2 pk;
    pk.x = pack2<T>(acc[0] * inv, acc[1] * inv);
    pk.y = pack2<T>(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(dst) = pk;
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack2<T>(acc[0] * inv, acc[1] * inv);
  }
  if (lane == 0 && lse != nullptr)
    lse[w] = tot > 0.f ? (mx + lg2_approx(tot)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace decode
}  // namespace eta
