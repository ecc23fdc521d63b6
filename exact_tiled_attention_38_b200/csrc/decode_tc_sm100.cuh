// Exact attention, decode, split pass on the tensor cores (sm_100a), for
// head size 128 and query-head groups of up to 32 per KV head.
//
// Same operation, cache layout, split ranges and partial outputs as the
// CUDA-core split pass in decode_sm100.cuh (the combine kernel there merges
// either): a CTA takes a contiguous chunk of one sequence's keys for one KV
// head and computes, for the G query heads sharing that KV head, the running
// softmax and the weighted sum of V (aikaboom page "11.4d FlashAttention",
// "Tiling" and "Online Softmax"; GQA grouping as on the sicorps page). With
// many query heads per KV head the scores are a real contraction (G x 128
// keys x 128 dims per tile), so they go to the tensor core instead of fp32
// shuffle reductions:
//
//   S^T = K_j Q^T      M = 128 keys, N = NP (G padded to 16 or 32), K = d.
//                      A = K tile (K-major), B = Q (K-major), fp32 in tensor
//                      memory: lane = key, column = head.
//   softmax            warp w reads the scores of keys 32w..32w+31; per head
//                      the tile max is reduced by shuffles and across the four
//                      warps through shared memory; p = 2^(s*c - m) with a
//                      lazily moved running max per head, rounded to the
//                      input type and stored as P^T [head][key] in shared
//                      memory; each thread keeps its keys' share of l.
//   O^T += V_j^T P^T   M = 128 dims, N = NP, K = 128 keys. A = V tile read
//                      MN-major, B = P^T (K-major); fp32 in tensor memory.
//
// K and V tiles come in through cp.async (16-byte copies, zero-filled past the
// chunk's last key) written straight into the 128-byte-swizzled layout the
// MMA reads: the packed ragged cache has no per-call extent known on the host,
// so no tensor map can bound it, while every cp.async source row is checked
// against the sequence here. Three producer warps own one ring stage each.
//
// Warp roles (256 threads): warps 0-3 softmax and epilogue, warp 4 tensor
// memory owner and MMA issue (whole warp, one elected lane), warps 5-7
// producers. Every wait is bounded (the CTA gives up and records the site).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>
#include <type_traits>

#include "common.cuh"
#include "decode_sm100.cuh"

namespace eta {
namespace decode_tc {

using decode::DParams;

constexpr int D = 128;
constexpr int TK = 128;  // keys per tile (the M of the score product)
constexpr int kStages = 3;
constexpr int kSoftWarps = 4;
constexpr int kMmaWarp = 4;
constexpr int kProdWarp0 = 5;
constexpr int kThreads = 32 * (kProdWarp0 + kStages);
constexpr float kRescaleThreshold = 8.0f;
constexpr uint32_t kTmemCols = 128;

enum : unsigned {
  kSiteFull = 0x31,
  kSiteEmpty = 0x32,
  kSiteS = 0x33,
  kSiteP = 0x34,
  kSitePv = 0x35,
  kSiteX = 0x36,
  kSiteQ = 0x37,
  kSiteDrain = 0x38,
};

template <int NP>
struct TCfg {
  static_assert(NP == 16 || NP == 32, "padded group");
  static constexpr int kBoxBytes = TK * 128;          // 128 keys x 64 dims
  static constexpr int kTileBytes = 2 * kBoxBytes;    // K or V tile (32 KB)
  static constexpr int kStageBytes = 2 * kTileBytes;  // K tile, then V tile
  static constexpr int kQBox = NP * 128;              // NP rows x 64 dims (or 64 keys)
  static constexpr int kQOff = kStages * kStageBytes;
  static constexpr int kPBuf = 2 * kQBox;             // P^T: 2 boxes of 64 keys
  static constexpr int kPOff = kQOff + 2 * kQBox;
  static constexpr int kRedOff = kPOff + 2 * kPBuf;   // [2][warps][NP] floats
  // full[S], empty[S], s_ready[2], p_ready[2], x_bar[2], q_full, pv_done, drain
  static constexpr int kBarOff = kRedOff + 2 * kSoftWarps * NP * 4;
  static constexpr int kNumBars = 2 * kStages + 6 + 3;
  static constexpr int kCtlOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kCtlOff + 64 + 1024;  // + runtime 1024-byte alignment
  static_assert(kQOff % 1024 == 0 && kPOff % 1024 == 0 && kQBox % 1024 == 0, "swizzle atoms");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

// Byte offset of 16-byte unit u (0..15 along a 256-byte row) of row r in a
// tile of two 128-byte-swizzled boxes (columns 0-63 | 64-127), box_bytes apart.
__device__ __forceinline__ uint32_t sw128_off(int r, int u, int box_bytes) {
  return static_cast<uint32_t>((u >> 3) * box_bytes + r * 128 + (((u & 7) ^ (r & 7)) << 4));
}

template <int NP>
__device__ __forceinline__ void tmem_ld_np(uint32_t taddr, uint32_t (&r)[NP]);
template <>
__device__ __forceinline__ void tmem_ld_np<16>(uint32_t taddr, uint32_t (&r)[16]) {
  tmem_ld_x16(taddr, r);
  tmem_wait_ld_x16(r);
}
template <>
__device__ __forceinline__ void tmem_ld_np<32>(uint32_t taddr, uint32_t (&r)[32]) {
  tmem_ld_x32(taddr, r);
  tmem_wait_ld_x32(r);
}
template <int NP>
__device__ __forceinline__ void tmem_st_np(uint32_t taddr, const uint32_t (&r)[NP]);
template <>
__device__ __forceinline__ void tmem_st_np<16>(uint32_t taddr, const uint32_t (&r)[16]) {
  tmem_st_x16(taddr, r);
}
template <>
__device__ __forceinline__ void tmem_st_np<32>(uint32_t taddr, const uint32_t (&r)[32]) {
  tmem_st_x32(taddr, r);
}

template <typename T>
__device__ __forceinline__ uint16_t to_bits(float x);
template <>
__device__ __forceinline__ uint16_t to_bits<__nv_bfloat16>(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}
template <>
__device__ __forceinline__ uint16_t to_bits<__half>(float x) {
  return __half_as_ushort(__float2half_rn(x));
}

// Value of element h of a register array, taken by lane-uniform selects (a
// variable index into registers would spill the array to local memory).
template <int NP>
__device__ __forceinline__ float pick(const float (&a)[NP], int h) {
  float v = 0.f;
#pragma unroll
  for (int i = 0; i < NP; ++i) v = (i == h) ? a[i] : v;
  return v;
}

template <int NP, typename T>
__global__ void __launch_bounds__(kThreads, 1) attn_decode_tc_kernel(const DParams p) {
  using C = TCfg<NP>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sQ = smem + C::kQOff;
  uint8_t* sP = smem + C::kPOff;
  float* red = reinterpret_cast<float*>(smem + C::kRedOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = full + kStages;
  uint64_t* s_ready = empty + kStages;
  uint64_t* p_ready = s_ready + 2;
  uint64_t* x_bar = p_ready + 2;
  uint64_t* q_full = x_bar + 2;
  uint64_t* pv_done = q_full + 1;
  uint64_t* drain = pv_done + 1;
  CtaCtl* ctl = reinterpret_cast<CtaCtl*>(smem + C::kCtlOff);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kCtlOff + 32);
  long long* misc = reinterpret_cast<long long*>(smem + C::kCtlOff + 40);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int g = blockIdx.y;
  const int b = blockIdx.z;

  if (warp == 0) {
    long long acc = 0;
    for (int j = lane; j < b; j += 32) acc += max(p.seqlens[j], 0);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      misc[0] = acc;
      misc[1] = max(p.seqlens[b], 0);
    }
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 32);  // one cp.async arrival per producer lane
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_ready[i], 1);
      mbar_init(&p_ready[i], 32 * kSoftWarps);
      mbar_init(&x_bar[i], 32 * kSoftWarps);
    }
    mbar_init(q_full, 32 * kSoftWarps);
    mbar_init(pv_done, 1);
    mbar_init(drain, 1);
    ctl->abort = 0;
    ctl->wait_ns = p.wait_ns;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const long long tok_off = misc[0];
  const int L = static_cast<int>(misc[1]);
  // Keys read: [tw, L), the whole sequence or its last `window` tokens.
  const int tw = (p.window > 0 && L > p.window) ? L - p.window : 0;
  int per = (L - tw + p.nsplit - 1) / p.nsplit;
  per = (per + TK - 1) / TK * TK;
  const int t_begin = min(L, tw + split * per);
  const int t_end = min(L, t_begin + per);
  const int ntiles = (t_end - t_begin + TK - 1) / TK;
  const size_t head_base = (static_cast<size_t>(tok_off) * p.Hkv + static_cast<size_t>(g) * L) * D;
  const T* kbase = reinterpret_cast<const T*>(p.kc) + head_base;
  const T* vbase = reinterpret_cast<const T*>(p.vc) + head_base;
  const int G = p.G;
  const uint32_t tS0 = tmem;              // S^T buffers: columns [0, NP), [NP, 2 NP)
  const uint32_t tO = tmem + 2 * NP;      // O^T: columns [2 NP, 3 NP)

  if (warp >= kProdWarp0) {
    // ------------------------------------------------------------ producers
    // Producer pw fills stage pw with tiles pw, pw + 3, ... Lane l copies
    // 16-byte unit (l % 16) of rows 2i + l / 16: each instruction reads two
    // whole 256-byte cache rows.
    const int pw = warp - kProdWarp0;
    bool ok = true;
    const uint32_t kdst = smem_u32(smem + pw * C::kStageBytes);
    const uint32_t vdst = kdst + C::kTileBytes;
    const int u = lane & 15;
    for (int j = pw; ok && j < ntiles; j += kStages) {
      const int use = j / kStages;
      if (use > 0 && !(ok = decode::warp_all_d(wait_bar(&empty[pw], (use - 1) & 1, ctl, kSiteEmpty))))
        break;
      const int t0 = t_begin + j * TK;
#pragma unroll 4
      for (int i = 0; i < TK / 2; ++i) {
        const int r = 2 * i + (lane >> 4);
        const int key = t0 + r;
        const bool valid = key < t_end;
        const size_t row = static_cast<size_t>(valid ? key : t0);  // t0 < t_end: a real row
        const uint32_t nb = valid ? 16u : 0u;                     // 0: zero-fill, no read
        const uint32_t off = sw128_off(r, u, C::kBoxBytes);
        cp_async16(kdst + off, kbase + row * D + u * 8, nb);
        cp_async16(vdst + off, vbase + row * D + u * 8, nb);
      }
      cp_async_mbar_arrive_noinc(&full[pw]);
    }
    cp_async_wait_all();  // no copy may land after the CTA exits
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    constexpr uint32_t fmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
    constexpr uint32_t idesc_s = umma_idesc_f16(fmt, TK, NP, 0, 0);
    constexpr uint32_t idesc_pv = umma_idesc_f16(fmt, D, NP, 1, 0);
    const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
    const uint32_t d_hi = static_cast<uint32_t>(dq >> 32);
    const uint32_t q_lo = static_cast<uint32_t>(dq);
    const uint32_t k_lo = static_cast<uint32_t>(smem_desc_sw128(smem_u32(smem), 16, 1024));
    const uint32_t v_lo = static_cast<uint32_t>(
        smem_desc_sw128(smem_u32(smem + C::kTileBytes), C::kBoxBytes, 1024));
    const uint32_t p_lo = static_cast<uint32_t>(smem_desc_sw128(smem_u32(sP), 16, 1024));
    bool ok = ntiles > 0 && decode::warp_all_d(wait_bar(q_full, 0, ctl, kSiteQ));
    for (int j = 0; ok && j <= ntiles; ++j) {
      if (j < ntiles) {
        // S^T(j) = K_j Q^T into buffer j % 2 (its previous scores, of tile
        // j - 2, were read before p_ready(j - 2), waited for last iteration).
        const int st = j % kStages;
        if (!(ok = decode::warp_all_d(wait_bar(&full[st], (j / kStages) & 1, ctl, kSiteFull)))) break;
        fence_proxy_async_smem();  // the cp.async data is read by the tensor core
        tc_fence_after();
        const uint32_t kd = k_lo + ((st * C::kStageBytes) >> 4);
        const uint32_t tS = tS0 + (j & 1) * NP;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
          const uint32_t qo = ((kk >> 2) * C::kQBox + (kk & 3) * 32) >> 4;
          if (kk == 0)
            umma_ss_w<0>(tS, desc_words(kd + ko, d_hi), desc_words(q_lo + qo, d_hi), idesc_s);
          else
            umma_ss_w<1>(tS, desc_words(kd + ko, d_hi), desc_words(q_lo + qo, d_hi), idesc_s);
        }
        umma_commit_w(&s_ready[j & 1]);
      }
      if (j >= 1) {
        // O^T += V_{j-1}^T P^T(j-1); then stage (j-1) % 3 is free again.
        const int jp = j - 1;
        const int st = jp % kStages;
        if (!(ok = decode::warp_all_d(wait_bar(&p_ready[jp & 1], (jp >> 1) & 1, ctl, kSiteP)))) break;
        fence_proxy_async_smem();
        tc_fence_after();
        const uint32_t vd = v_lo + ((st * C::kStageBytes) >> 4);
        const uint32_t pd = p_lo + (((jp & 1) * C::kPBuf) >> 4);
#pragma unroll
        for (int kk = 0; kk < TK / 16; ++kk) {
          const uint32_t vo = kk * 128;  // 16 keys = 16 rows of 128 bytes
          const uint32_t po = ((kk >> 2) * C::kQBox + (kk & 3) * 32) >> 4;
          if (jp == 0 && kk == 0)
            umma_ss_w<0>(tO, desc_words(vd + vo, d_hi), desc_words(pd + po, d_hi), idesc_pv);
          else
            umma_ss_w<1>(tO, desc_words(vd + vo, d_hi), desc_words(pd + po, d_hi), idesc_pv);
        }
        umma_commit_w(&empty[st]);
        umma_commit_w(pv_done);
      }
    }
    // Every MMA must be complete before tensor memory is released.
    umma_commit_w(drain);
    drain_bar(drain, 0, ctl, kSiteDrain);
  } else {
    // ------------------------------------------------------------ softmax
    // Q rows of the group -> shared memory (K-major, swizzled); rows >= G are 0.
    for (int i = threadIdx.x; i < NP * 16; i += 32 * kSoftWarps) {
      const int h = i >> 4;
      const int uu = i & 15;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (h < G)
        v = *reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.q) +
                                            (static_cast<size_t>(b) * p.Hq + g * G + h) * D +
                                            uu * 8);
      *reinterpret_cast<uint4*>(sQ + sw128_off(h, uu, C::kQBox)) = v;
    }
    fence_proxy_async_smem();
    mbar_arrive(q_full);

    const int krow = warp * 32 + lane;  // this thread's key within a tile (tensor-memory lane)
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = p.scale_log2;
    float m[NP], l[NP];
#pragma unroll
    for (int h = 0; h < NP; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.f;
    }
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      if (!(ok = decode::warp_all_d(wait_bar(&s_ready[j & 1], (j >> 1) & 1, ctl, kSiteS)))) break;
      tc_fence_after();
      uint32_t r[NP];
      tmem_ld_np<NP>(tS0 + lane_off + (j & 1) * NP, r);
      const bool valid = t_begin + j * TK + krow < t_end;
      float s[NP], wm[NP];
#pragma unroll
      for (int h = 0; h < NP; ++h) {
        s[h] = (valid && h < G) ? __uint_as_float(r[h]) * sl2 : -INFINITY;
        wm[h] = s[h];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int h = 0; h < NP; ++h) wm[h] = fmaxf(wm[h], __shfl_xor_sync(0xffffffffu, wm[h], o));
      float* rb = red + (j & 1) * (kSoftWarps * NP);
      if (lane < NP) rb[warp * NP + lane] = pick<NP>(wm, lane);
      mbar_arrive(&x_bar[j & 1]);
      if (!(ok = decode::warp_all_d(wait_bar(&x_bar[j & 1], (j >> 1) & 1, ctl, kSiteX)))) break;
      float alpha[NP];
      bool rescale = false;
#pragma unroll
      for (int h = 0; h < NP; ++h) {
        const float tm = fmaxf(fmaxf(rb[h], rb[NP + h]), fmaxf(rb[2 * NP + h], rb[3 * NP + h]));
        alpha[h] = 1.f;
        if (tm > m[h] + kRescaleThreshold) {
          alpha[h] = ex2_approx(m[h] - tm);  // m = -inf gives 0
          m[h] = tm;
          l[h] *= alpha[h];
          rescale = true;
        }
      }
      if (rescale && j > 0) {
        // O^T was last written by PV(j-1); wait for it, then scale its columns
        // (this warp's 32 dims) by the heads' alpha.
        if (!(ok = decode::warp_all_d(wait_bar(pv_done, (j - 1) & 1, ctl, kSitePv)))) break;
        tc_fence_after();
        uint32_t o[NP];
        tmem_ld_np<NP>(tO + lane_off, o);
#pragma unroll
        for (int h = 0; h < NP; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
        tmem_st_np<NP>(tO + lane_off, o);
        tmem_wait_st();
      }
      // P^T(j): row h, key krow, in buffer j % 2 (read by PV(j - 2), which
      // completed before S(j) was signalled).
      uint8_t* pb = sP + (j & 1) * C::kPBuf + (krow >> 6) * C::kQBox;
      const int kc = krow & 63;
#pragma unroll
      for (int h = 0; h < NP; ++h) {
        if (h < G) {
          const float pv = ex2_approx(s[h] - (m[h] == -INFINITY ? 0.f : m[h]));
          l[h] += pv;
          *reinterpret_cast<uint16_t*>(pb + h * 128 + ((((kc >> 3) ^ (h & 7))) << 4) +
                                       ((kc & 7) << 1)) = to_bits<T>(pv);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_ready[j & 1]);
    }
    if (ok) {
      // Row sums over the 128 keys of the tile slots, then the outputs.
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int h = 0; h < NP; ++h) l[h] += __shfl_xor_sync(0xffffffffu, l[h], o);
      float* rb = red + (ntiles & 1) * (kSoftWarps * NP);
      if (lane < NP) rb[warp * NP + lane] = pick<NP>(l, lane);
      mbar_arrive(&x_bar[ntiles & 1]);
      ok = decode::warp_all_d(wait_bar(&x_bar[ntiles & 1], (ntiles >> 1) & 1, ctl, kSiteX));
      uint32_t o[NP];
#pragma unroll
      for (int h = 0; h < NP; ++h) o[h] = 0u;
      if (ok && ntiles > 0) {
        ok = decode::warp_all_d(wait_bar(pv_done, (ntiles - 1) & 1, ctl, kSitePv));
        if (ok) {
          tc_fence_after();
          tmem_ld_np<NP>(tO + lane_off, o);
        }
      }
      if (ok) {
        const int dim = krow;  // O^T lane = output dimension
#pragma unroll
        for (int h = 0; h < NP; ++h) {
          if (h < G) {
            const float lt = rb[h] + rb[NP + h] + rb[2 * NP + h] + rb[3 * NP + h];
            const float ov = lt > 0.f ? __uint_as_float(o[h]) / lt : 0.f;
            const float l2 = lt > 0.f ? m[h] + lg2_approx(lt) : -INFINITY;
            if (p.o != nullptr) {
              // One split: this is the result (O rounded, LSE in natural log).
              const size_t row = static_cast<size_t>(b) * p.Hq + g * G + h;
              reinterpret_cast<uint16_t*>(p.o)[row * D + dim] = to_bits<T>(ov);
              if (dim == h && p.lse != nullptr) p.lse[row] = l2 * 0.69314718055994531f;
            } else {
              const size_t row = (static_cast<size_t>(split) * p.B + b) * p.Hq + g * G + h;
              p.part_o[row * D + dim] = ov;
              if (dim == h) p.part_lse[row] = l2;
            }
          }
        }
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

}  // namespace decode_tc
}  // namespace eta
