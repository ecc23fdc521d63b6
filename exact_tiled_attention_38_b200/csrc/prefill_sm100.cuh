// Exact tiled attention, prefill: softmax(scale * Q K^T + causal mask) V with
// the log-sum-exp of every row, for sm_100a.
//
// The method is the tiled, running-softmax attention of the aikaboom page
// "11.4d FlashAttention" (sections "Tiling" and "Online Softmax") and of the
// zimaspace page "How Does Flash Attention Reduce Memory Traffic During Local
// Inference?" (sections on tiling, online softmax and kernel fusion): the
// score matrix lives only as one 128x128 fp32 tile in tensor memory, the row
// max and row sum are carried from key tile to key tile, and scaling, masking,
// normalisation and the value product all stay inside one kernel.
//
// One CTA owns two 128-row query tiles of one (batch, query head) and streams
// the key/value tiles of that head's KV head (GQA: kv head = h / (Hq / Hkv)).
// Warp roles (320 threads):
//   warps 0-3  softmax for query tile 0 (one thread per query row)
//   warps 4-7  softmax for query tile 1
//   warp  8    tensor-memory owner and the single thread that issues tcgen05.mma
//   warp  9    TMA producer: Q once, then K_j and V_j through a ring of stages
// Tensor memory (512 columns x 128 lanes): S_0 [0,128), S_1 [128,256),
// O_0 [256, 256+D), O_1 [256+D, 256+2D); the bf16/fp16 probabilities P_t
// overwrite columns [64,128) of S_t once the softmax has read S_t. The MMA
// thread issues, per key tile j: O_t += P_t(j-1) V_{j-1} then S_t = Q_t K_j^T
// for t = 0, 1, so while one softmax group works on its tile the tensor core
// runs the other group's products. tcgen05.mma operations issued by one thread
// execute in issue order, which is what lets S_t(j) reuse the columns that
// P_t(j-1) occupied.
//
// Online softmax per row (fp32, log2 domain, c = scale * log2 e):
//   m' = max over the tile of s * c; if m' > m + 8 the row's running max moves
//   to m' and O and l are multiplied by 2^(m - m'); otherwise the stale max is
//   kept (exact: O and l share the same reference, p <= 2^8).
//   p = 2^(s*c - m), l += sum p (unrounded), P = round(p) -> tensor memory.
// Epilogue: O / l rounded to the input type; LSE = ln 2 * (m + log2 l).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>

#include "common.cuh"

namespace eta {
namespace prefill {

constexpr int BM = 128;   // query rows per tile
constexpr int BN = 128;   // keys per tile
constexpr int NQT = 2;    // query tiles per CTA
constexpr int kThreads = 320;
constexpr int kMmaWarp = 8;
constexpr int kTmaWarp = 9;
constexpr float kRescaleThreshold = 8.0f;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kPCol = 64;  // P_t starts this many columns into S_t

// Wait sites reported in the status word.
enum : unsigned {
  kSiteQFull = 1,
  kSiteKvEmpty = 2,
  kSiteKvFull = 3,
  kSitePReady = 4,
  kSiteSReady = 5,
  kSiteODone = 6,
  kSiteDrain = 7,
};

template <int D>
struct Cfg {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int kBoxes = D / 64;             // 64-element (128-byte) column boxes
  static constexpr int kBoxBytes = 128 * 128;       // 128 rows x 128 bytes
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kStages = (D == 128) ? 4 : 6;
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = NQT * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
  static constexpr int kNumBars = 1 + 2 * kStages + 3 * NQT + 1;
  static constexpr int kCtlOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kCtlOff + 64 + 1024;  // + runtime 1024-byte alignment
  static constexpr uint32_t kOCol = 2 * BN;
};

struct Params {
  void* o;
  float* lse;
  int Hq;
  int Hkv;
  int Nq;
  int Nk;
  int group;       // Hq / Hkv
  int n_pairs;     // ceil(Nq / 256)
  int off;         // Nk - Nq: query i sees keys j <= i + off when causal
  float scale_log2;
  uint64_t wait_ns;
  int debug_flags;  // bit 0: the producer issues no copies (exercises the wait limit)
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

template <typename T>
struct Fmt;
template <>
struct Fmt<__nv_bfloat16> {
  static constexpr uint32_t value = 1;
};
template <>
struct Fmt<__half> {
  static constexpr uint32_t value = 0;
};

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

template <int D, typename T, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = Cfg<D>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);

  uint8_t* sQ = smem + C::kQOff;
  uint8_t* sKV = smem + C::kKVOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + S;
  uint64_t* s_ready = kv_empty + S;
  uint64_t* p_ready = s_ready + NQT;
  uint64_t* o_done = p_ready + NQT;
  uint64_t* drain = o_done + NQT;
  CtaCtl* ctl = reinterpret_cast<CtaCtl*>(smem + C::kCtlOff);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kCtlOff + 32);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x;  // b * Hq + h
  const int b = bh / p.Hq;
  const int h = bh - b * p.Hq;
  const int kvh = h / p.group;
  const int pair = CAUSAL ? (p.n_pairs - 1 - static_cast<int>(blockIdx.y))
                          : static_cast<int>(blockIdx.y);
  const int nkv_all = (p.Nk + BN - 1) / BN;

  // Key tiles each query tile needs (causal: stop at the last visible key).
  int r0[NQT], nt[NQT];
#pragma unroll
  for (int t = 0; t < NQT; ++t) {
    r0[t] = pair * (NQT * BM) + t * BM;
    if (r0[t] >= p.Nq) {
      nt[t] = 0;
    } else if (!CAUSAL) {
      nt[t] = nkv_all;
    } else {
      const int last_row = min(r0[t] + BM - 1, p.Nq - 1);
      const long long kmax = static_cast<long long>(last_row) + p.off;
      const long long ntiles = kmax / BN + 1;
      nt[t] = kmax < 0 ? 0 : static_cast<int>(ntiles < nkv_all ? ntiles : nkv_all);
    }
  }
  const int nmax = max(nt[0], nt[1]);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < NQT; ++t) {
      mbar_init(&s_ready[t], 1);
      mbar_init(&p_ready[t], 4 * 32);
      mbar_init(&o_done[t], 1);
    }
    mbar_init(drain, 1);
    ctl->abort = 0;
    ctl->wait_ns = p.wait_ns;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kTmaWarp && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nmax > 0 && !(p.debug_flags & 1)) {
      const int zkv = b * p.Hkv + kvh;
      uint32_t qbytes = 0;
#pragma unroll
      for (int t = 0; t < NQT; ++t)
        if (r0[t] < p.Nq) qbytes += C::kTileBytes;
      mbar_arrive_expect_tx(q_full, qbytes);
#pragma unroll
      for (int t = 0; t < NQT; ++t) {
        if (r0[t] >= p.Nq) continue;
        for (int bx = 0; bx < C::kBoxes; ++bx)
          tma_load_3d(sQ + t * C::kTileBytes + bx * C::kBoxBytes, &tm_q, q_full, bx * 64, r0[t],
                      bh);
      }
      const int nloads = 2 * nmax;  // K_0, V_0, K_1, V_1, ...
      int issued = 0;
      for (int L = 0; L < nloads; ++L) {
        const int s = L % S;
        const int use = L / S;
        if (use > 0 && !wait_bar(&kv_empty[s], (use - 1) & 1, ctl, kSiteKvEmpty)) break;
        const CUtensorMap* map = (L & 1) ? &tm_v : &tm_k;
        const int j = L >> 1;
        mbar_arrive_expect_tx(&kv_full[s], C::kTileBytes);
        for (int bx = 0; bx < C::kBoxes; ++bx)
          tma_load_3d(sKV + s * C::kTileBytes + bx * C::kBoxBytes, map, &kv_full[s], bx * 64,
                      j * BN, zkv);
        issued = L + 1;
      }
      // No copy may still be landing in shared memory when the CTA exits.
      drain_bar(q_full, 0, ctl, kSiteDrain);
      for (int s = 0; s < S && s < issued; ++s) {
        const int last = s + S * ((issued - 1 - s) / S);
        drain_bar(&kv_full[s], (last / S) & 1, ctl, kSiteDrain);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nmax > 0) {
      constexpr uint32_t fmt = Fmt<T>::value;
      constexpr uint32_t idesc_s = umma_idesc_f16(fmt, BM, BN, 0, 0);
      constexpr uint32_t idesc_pv = umma_idesc_f16(fmt, BM, D, 0, 1);
      const uint32_t sq = smem_u32(sQ);
      const uint32_t skv = smem_u32(sKV);
      bool ok = wait_bar(q_full, 0, ctl, kSiteQFull);
      if (ok) tc_fence_after();
      for (int j = 0; ok && j <= nmax; ++j) {
        const int Lk = 2 * j;
        const int Lv = 2 * j - 1;
        bool have_k = false, have_v = false;
#pragma unroll
        for (int t = 0; t < NQT; ++t) {
          if (!ok) break;
          if (j >= 1 && j - 1 < nt[t]) {
            // O_t += P_t(j-1) V_{j-1}
            if (!have_v) {
              ok = wait_bar(&kv_full[Lv % S], (Lv / S) & 1, ctl, kSiteKvFull);
              if (!ok) break;
              have_v = true;
            }
            ok = wait_bar(&p_ready[t], (j - 1) & 1, ctl, kSitePReady);
            if (!ok) break;
            tc_fence_after();
            const uint32_t vbase = skv + (Lv % S) * C::kTileBytes;
            const uint32_t tP = tmem + t * BN + kPCol;
            const uint32_t tO = tmem + C::kOCol + t * D;
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) {
              const uint64_t bdesc = smem_desc_sw128(vbase + kk * 16 * 128, C::kBoxBytes, 1024);
              umma_ts(tO, tP + kk * 8, bdesc, idesc_pv, (j > 1 || kk > 0) ? 1u : 0u);
            }
            if (j - 1 == nt[t] - 1) umma_commit(&o_done[t]);
          }
          if (j < nt[t]) {
            // S_t = Q_t K_j^T
            if (!have_k) {
              ok = wait_bar(&kv_full[Lk % S], (Lk / S) & 1, ctl, kSiteKvFull);
              if (!ok) break;
              tc_fence_after();
              have_k = true;
            }
            const uint32_t kbase = skv + (Lk % S) * C::kTileBytes;
            const uint32_t qbase = sq + t * C::kTileBytes;
            const uint32_t tS = tmem + t * BN;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t koff = (kk >> 2) * C::kBoxBytes + (kk & 3) * 32;
              umma_ss(tS, smem_desc_sw128(qbase + koff, 16, 1024),
                      smem_desc_sw128(kbase + koff, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
            }
            umma_commit(&s_ready[t]);
          }
        }
        if (have_k) umma_commit(&kv_empty[Lk % S]);
        if (have_v) umma_commit(&kv_empty[Lv % S]);
      }
      // Every MMA must be complete before tensor memory is released.
      umma_commit(drain);
      drain_bar(drain, 0, ctl, kSiteDrain);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int t = warp >> 2;
    const int q4 = warp & 3;
    const int rt = t ? r0[1] : r0[0];
    const int row = rt + q4 * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * BN;
    const uint32_t tP = tS + kPCol;
    const uint32_t tO = tmem + lane_off + C::kOCol + t * D;
    const float sl2 = p.scale_log2;
    const int n = t ? nt[1] : nt[0];
    float m = -INFINITY;  // running max of s * c (log2 units)
    float l = 0.f;        // running sum of p
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      ok = warp_all(wait_bar(&s_ready[t], i & 1, ctl, kSiteSReady));
      if (!ok) break;
      tc_fence_after();
      uint32_t ra[32], rb[32], rc[32], rd[32];
      tmem_ld_x32(tS + 0, ra);
      tmem_ld_x32(tS + 32, rb);
      tmem_ld_x32(tS + 64, rc);
      tmem_ld_x32(tS + 96, rd);
      tmem_wait_ld_x32(ra);
      tmem_wait_ld_x32(rb);
      tmem_wait_ld_x32(rc);
      tmem_wait_ld_x32(rd);
      float s[BN];
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        s[k] = __uint_as_float(ra[k]);
        s[32 + k] = __uint_as_float(rb[k]);
        s[64 + k] = __uint_as_float(rc[k]);
        s[96 + k] = __uint_as_float(rd[k]);
      }
      const int kv0 = i * BN;
      const bool edge = (CAUSAL && kv0 + BN - 1 > rt + p.off) || (kv0 + BN > p.Nk);
      if (edge) {
        const int last = (CAUSAL ? min(row + p.off, p.Nk - 1) : p.Nk - 1) - kv0;
#pragma unroll
        for (int k = 0; k < BN; ++k) s[k] = (k > last) ? -INFINITY : s[k];
      }
      float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
      for (int k = 4; k < BN; k += 4) {
        mx0 = fmaxf(mx0, s[k]);
        mx1 = fmaxf(mx1, s[k + 1]);
        mx2 = fmaxf(mx2, s[k + 2]);
        mx3 = fmaxf(mx3, s[k + 3]);
      }
      const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
      float alpha = 1.f;
      const bool need = m_tile > m + kRescaleThreshold;
      if (need) {
        alpha = ex2_approx(m - m_tile);  // m = -inf gives 0
        m = m_tile;
        l *= alpha;
      }
      const float m_use = (m == -INFINITY) ? 0.f : m;
      float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
      uint32_t pa[32], pb[32];
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const float e0 = ex2_approx(fmaf(s[2 * c], sl2, -m_use));
        const float e1 = ex2_approx(fmaf(s[2 * c + 1], sl2, -m_use));
        const float e2 = ex2_approx(fmaf(s[2 * c + 2], sl2, -m_use));
        const float e3 = ex2_approx(fmaf(s[2 * c + 3], sl2, -m_use));
        l0 += e0;
        l1 += e1;
        l2 += e2;
        l3 += e3;
        pa[c] = pack2<T>(e0, e1);
        pa[c + 1] = pack2<T>(e2, e3);
      }
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const float e0 = ex2_approx(fmaf(s[64 + 2 * c], sl2, -m_use));
        const float e1 = ex2_approx(fmaf(s[64 + 2 * c + 1], sl2, -m_use));
        const float e2 = ex2_approx(fmaf(s[64 + 2 * c + 2], sl2, -m_use));
        const float e3 = ex2_approx(fmaf(s[64 + 2 * c + 3], sl2, -m_use));
        l0 += e0;
        l1 += e1;
        l2 += e2;
        l3 += e3;
        pb[c] = pack2<T>(e0, e1);
        pb[c + 1] = pack2<T>(e2, e3);
      }
      l += (l0 + l1) + (l2 + l3);
      tmem_st_x32(tP, pa);
      tmem_st_x32(tP + 32, pb);
      if (i > 0 && __any_sync(0xffffffffu, need)) {
        // O_t was last written by PV_t(i-1), complete before S_t(i) was signalled.
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld_x32(tO + c * 32, o);
          tmem_wait_ld_x32(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st_x32(tO + c * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_ready[t]);
    }
    if (ok && n > 0) {
      ok = warp_all(wait_bar(&o_done[t], 0, ctl, kSiteODone));
      if (ok) tc_fence_after();
    }
    if (ok) {
      const bool has_row = row < p.Nq;
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      T* orow = reinterpret_cast<T*>(p.o) + (static_cast<size_t>(bh) * p.Nq + row) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (n > 0) {
          tmem_ld_x32(tO + c * 32, o);
          tmem_wait_ld_x32(o);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0u;
        }
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack2<T>(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
        if (has_row) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
          dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
          dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
          dst[2] = make_uint4(w[8], w[9], w[10], w[11]);
          dst[3] = make_uint4(w[12], w[13], w[14], w[15]);
        }
      }
      if (has_row && p.lse != nullptr) {
        p.lse[static_cast<size_t>(bh) * p.Nq + row] =
            l > 0.f ? (m + lg2_approx(l)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace prefill
}  // namespace eta
