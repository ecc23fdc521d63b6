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
// Work items are pairs of 128-row query tiles of one (batch, query head). The
// grid is persistent (one CTA per SM); CTA c takes items c, 2G-1-c, 2G+c, ...
// (G = grid size) from a list ordered heaviest first for causal masks, which
// balances the triangular work. Each item streams the key/value tiles of its
// KV head (GQA: kv head = h / (Hq / Hkv)).
// Warp roles (320 threads):
//   warps 0-3  softmax for query tile 0 (one thread per query row)
//   warps 4-7  softmax for query tile 1
//   warp  8    tensor-memory owner; runs the MMA issue loop as a whole warp,
//              one elected lane issuing each tcgen05.mma
//   warp  9    TMA producer: Q tiles, then K_j and V_j through a ring of stages
// Tensor memory (512 columns x 128 lanes): S_0 [0,128), S_1 [128,256),
// O_0 [256, 256+D), O_1 [256+D, 256+2D); the bf16/fp16 probabilities P_t
// overwrite columns [64,128) of S_t once the softmax has read S_t. The MMA
// thread issues, per key tile j: O_t += P_t(j-1) V_{j-1} then S_t = Q_t K_j^T
// for t = 0, 1, so while one softmax group works on its tile the tensor core
// runs the other group's products. tcgen05.mma operations issued by one thread
// execute in issue order, which is what lets S_t(j) reuse the columns that
// P_t(j-1) occupied. The next item's Q loads and first S products overlap the
// current item's epilogue.
//
// Head size 64 has room for P in tensor-memory columns of its own: per tile
// S_t [256t, 256t+128), P_t [256t+128, 256t+192), O_t [256t+192, 256t+256).
// The softmax then releases S_t (s_free) as soon as it has read it, and the
// MMA thread issues S_t(j+1) at once, before P_t(j) V_j: the next scores are
// ready when the softmax finishes a step, so the softmax groups run back to
// back instead of waiting for the product chain. Before writing P_t (and
// before rescaling O_t) the softmax waits for the previous P_t V product
// (pv_done).
//
// Online softmax per row (fp32, log2 domain, c = scale * log2 e):
//   m' = max over the tile of s * c; if m' > m + 8 the row's running max moves
//   to m' and O and l are multiplied by 2^(m - m'); otherwise the stale max is
//   kept (exact: O and l share the same reference, p <= 2^8).
//   p = 2^(s*c - m), l += sum p (unrounded), P = round(p) -> tensor memory.
// Epilogue: O / l rounded to the input type; LSE = ln 2 * (m + log2 l).
//
// Two optional refinements (template knobs):
//   PINGPONG  the two softmax groups take turns (an mbarrier token) for their
//             exponential phase, so the special-function unit serves one group
//             while the tensor core serves the other;
//   POLY8     of every 8 score columns, POLY8 get 2^x from a polynomial on the
//             FMA pipe (ex2_poly) instead of the special-function unit.
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
// SPLIT softmax threads share a query row (SPLIT = 1: 4 warps per query tile;
// SPLIT = 2: 8 warps per tile, each thread taking 64 of the row's 128 scores).
__host__ __device__ constexpr int softmax_warps(int split) { return 4 * NQT * split; }
__host__ __device__ constexpr int kernel_threads(int split) {
  return 32 * (softmax_warps(split) + 2);
}
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
  kSiteQEmpty = 8,
  kSiteTurn = 9,
  kSiteXUp = 10,
  kSiteXDown = 11,
  kSiteSFree = 12,
  kSitePvDone = 13,
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
  // O staging for the TMA-store epilogue: per softmax warp 32 rows x 64 columns.
  static constexpr int kStgWarpBytes = 32 * 128;
  static constexpr int kStgOff = kKVOff + kStages * kTileBytes;
  static constexpr int kBarOff = kStgOff + 8 * kStgWarpBytes;
  // kv_full[S], kv_empty[S], then per tile: q_full, q_empty, s_ready, p_ready,
  // o_done, turn; then drain; then per row quarter of each tile the two
  // exchange barriers of a split row (x_up: part 1 -> part 0, x_down: back);
  // then per tile s_free and pv_done (P in columns of its own, D = 64).
  static constexpr int kNumBars = 2 * kStages + 6 * NQT + 1 + 2 * 4 * NQT + 2 * NQT;
  static constexpr int kCtlOff = kBarOff + kNumBars * 8;
  // Row-statistics exchange between the two threads of a row (SPLIT = 2):
  // one float per query row of each tile.
  static constexpr int kXOff = kCtlOff + 64;
  static constexpr int kSmemBytes = kXOff + NQT * BM * 4 + 1024;  // + runtime 1024-byte alignment
  // P in columns of its own (D = 64): S_t, P_t, O_t in 256 columns per tile.
  static constexpr bool kOwnP = (D == 64);
  static constexpr uint32_t kOCol = 2 * BN;
  __host__ __device__ static constexpr uint32_t s_col(int t) { return kOwnP ? 256u * t : BN * t; }
  __host__ __device__ static constexpr uint32_t o_col(int t) {
    return kOwnP ? 256u * t + BN + 64 : kOCol + D * t;
  }
  // first column of P_t (SPLIT = 1)
  __host__ __device__ static constexpr uint32_t p_base(int t) {
    return kOwnP ? 256u * t + BN : BN * t + kPCol;
  }
  static_assert(kSmemBytes <= 232448, "shared memory");
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
  int BH;          // B * Hq
  int total;       // BH * n_pairs work items
  float scale_log2;
  uint64_t wait_ns;
  int debug_flags;  // bit 0: the producer issues no copies (exercises the wait limit)
  int window;       // causal only: a row keeps its `window` most recent keys (0 = all)
  int head_major;   // causal: query levels in blocks of this many, KV head by KV head
                    // inside a block (0: all heads of a level together)
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

// Make this thread's shared-memory writes visible to the async proxy (TMA).
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2^x on the FMA and integer pipes, for x <= 8.
// Range reduction: n = round(x) (adding 1.5 * 2^23 leaves round(x) in the low
// mantissa bits; exact for |x| < 2^22), f = x - n in [-1/2, 1/2], so
// 2^x = 2^n * 2^f. 2^f is a degree-3 polynomial whose coefficients are the
// minimax fit for relative error on [-1/2, 1/2], obtained with the Remez
// exchange algorithm: max relative error 7.5e-5 (2^-13.7), below the rounding
// of P to bf16 (2^-9) or fp16 (2^-11). 2^n is applied by adding n to the
// exponent field.
constexpr float kExp2C0 = 0.99992805719375610f;
constexpr float kExp2C1 = 0.69326096773147583f;
constexpr float kExp2C2 = 0.24261112511157990f;
constexpr float kExp2C3 = 0.05517166852951050f;

// Two values at once: the adds and the polynomial run as fp32-pair
// instructions. Inputs are clamped to -126 first, so the exponent field never
// underflows; callers use this only where no score is masked (2^-126 stands in
// for anything smaller).
__device__ __forceinline__ uint64_t ex2_poly2(float x0, float x1) {
  const uint64_t x = f2_make(fmaxf(x0, -126.0f), fmaxf(x1, -126.0f));
  const uint64_t magic = f2_make(12582912.0f, 12582912.0f);  // 1.5 * 2^23
  const uint64_t t = f2_add(x, magic);
  const uint64_t n = f2_add(t, f2_make(-12582912.0f, -12582912.0f));
  const uint64_t f = f2_fma(n, f2_make(-1.0f, -1.0f), x);
  uint64_t q = f2_fma(f2_make(kExp2C3, kExp2C3), f, f2_make(kExp2C2, kExp2C2));
  q = f2_fma(q, f, f2_make(kExp2C1, kExp2C1));
  q = f2_fma(q, f, f2_make(kExp2C0, kExp2C0));
  float q0, q1, t0, t1;
  f2_split(q, q0, q1);
  f2_split(t, t0, t1);
  const float r0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  const float r1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
  return f2_make(r0, r1);
}

// Key tiles are counted from the item's first one, jb: query tile t uses steps
// [s_t, n_t), i.e. key tiles jb + s_t .. jb + n_t - 1 (s_t = n_t when the tile
// has no visible key). Without a window jb = s_0 = s_1 = 0.
struct Item {
  int bh;
  int b;
  int kvh;
  int r0;  // first query row of tile 0 (tile 1 starts at r0 + BM)
  int jb;  // first key tile the item loads
  int s0;  // first step of query tile 0
  int s1;  // first step of query tile 1
  int n0;  // end step of query tile 0
  int n1;  // end step of query tile 1
};

// Snake order over the persistent grid: balances items sorted heaviest first.
__device__ __forceinline__ int item_index(int round, int cta, int G) {
  return round * G + ((round & 1) ? (G - 1 - cta) : cta);
}

template <bool CAUSAL>
__device__ __forceinline__ int key_tiles(int r0, const Params& p, int nkv_all) {
  if (r0 >= p.Nq) return 0;
  if (!CAUSAL) return nkv_all;
  const int last_row = min(r0 + BM - 1, p.Nq - 1);
  const long long kmax = static_cast<long long>(last_row) + p.off;
  if (kmax < 0) return 0;
  const long long ntiles = kmax / BN + 1;
  return static_cast<int>(ntiles < nkv_all ? ntiles : nkv_all);
}

// First key tile any row of the tile starting at r0 sees under the window.
template <bool CAUSAL, bool WINDOW>
__device__ __forceinline__ int first_key_tile(int r0, const Params& p) {
  if (!CAUSAL || !WINDOW) return 0;
  const long long k0 = static_cast<long long>(r0) + p.off - p.window + 1;
  return k0 <= 0 ? 0 : static_cast<int>(k0 / BN);
}

template <bool CAUSAL, bool WINDOW = false>
__device__ __forceinline__ Item decode_item(int idx, const Params& p, int nkv_all) {
  Item it;
  int pair;
  if (CAUSAL && p.head_major > 0) {
    // K/V of all heads do not fit in L2. Query levels go in blocks of Lb,
    // heaviest first; inside a block, (batch, KV head) by (batch, KV head),
    // each taking its Lb levels times the query heads of its group. Lb * group
    // is a whole number of rounds of the grid, so the CTAs running at one time
    // stream the K/V of about one KV head, which stays in L2, and every round
    // has the same weights, which the snake order balances.
    const int Lb = p.head_major;
    const int units = p.BH / p.group;  // B * Hkv
    const int blk = Lb * p.group * units;
    const int k = idx / blk;
    const int r = idx - k * blk;
    const int per_unit = min(Lb, p.n_pairs - k * Lb) * p.group;
    const int unit = r / per_unit;
    const int r2 = r - unit * per_unit;
    const int lvl = k * Lb + r2 / p.group;
    const int b = unit / p.Hkv;
    pair = p.n_pairs - 1 - lvl;
    it.bh = b * p.Hq + (unit - b * p.Hkv) * p.group + (r2 - (r2 / p.group) * p.group);
  } else if (CAUSAL) {  // heaviest (last) query tiles first, all heads of one level together
    pair = p.n_pairs - 1 - idx / p.BH;
    it.bh = idx - (idx / p.BH) * p.BH;
  } else {  // consecutive items share a head, so concurrent CTAs share K/V in L2
    it.bh = idx / p.n_pairs;
    pair = idx - it.bh * p.n_pairs;
  }
  it.b = it.bh / p.Hq;
  const int h = it.bh - it.b * p.Hq;
  it.kvh = h / p.group;
  it.r0 = pair * (NQT * BM);
  const int hi0 = key_tiles<CAUSAL>(it.r0, p, nkv_all);
  const int hi1 = key_tiles<CAUSAL>(it.r0 + BM, p, nkv_all);
  const int lo0 = min(first_key_tile<CAUSAL, WINDOW>(it.r0, p), hi0);
  const int lo1 = min(first_key_tile<CAUSAL, WINDOW>(it.r0 + BM, p), hi1);
  it.jb = (hi0 > lo0) ? lo0 : ((hi1 > lo1) ? lo1 : 0);
  it.s0 = (hi0 > lo0) ? lo0 - it.jb : 0;
  it.n0 = (hi0 > lo0) ? hi0 - it.jb : 0;
  it.s1 = (hi1 > lo1) ? lo1 - it.jb : 0;
  it.n1 = (hi1 > lo1) ? hi1 - it.jb : 0;
  return it;
}

// Tensor-memory column (within S_t) of P for keys 16kk .. 16kk + 15.
template <int SPLIT>
__host__ __device__ constexpr uint32_t p_col(int kk) {
  return SPLIT == 1 ? kPCol + kk * 8
                    : static_cast<uint32_t>((kk / (BN / 16 / SPLIT)) * (BN / SPLIT) +
                                            (kk % (BN / 16 / SPLIT)) * 8);
}

// p = 2^(s * c - m) for NC scores of one row: writes P (rounded to T) to
// tensor memory at tP, 32 scores (16 columns) at a time, and returns the fp32
// sum of p. POLY8 of every 8 columns use the polynomial exponential (only for
// tiles without masked scores).
template <typename T, int POLY8, int NC>
__device__ __forceinline__ float exp_tile(const float (&s)[NC], float c, float m_use, uint32_t tP) {
  const uint64_t c2 = f2_make(c, c);
  const uint64_t nm2 = f2_make(-m_use, -m_use);
  uint64_t la = f2_make(0.f, 0.f), lb = la;
#pragma unroll
  for (int ch = 0; ch < NC / 32; ++ch) {
    // 32 columns -> 16 packed words -> tensor memory, chunk by chunk so that
    // the registers of S are released as P is produced.
    uint32_t pk[16];
#pragma unroll
    for (int w = 0; w < 16; ++w) {
      const int k = ch * 32 + 2 * w;
      const uint64_t x2 = f2_fma(f2_make(s[k], s[k + 1]), c2, nm2);
      float x0, x1;
      f2_split(x2, x0, x1);
      const uint64_t e2 =
          ((k & 7) < POLY8) ? ex2_poly2(x0, x1) : f2_make(ex2_approx(x0), ex2_approx(x1));
      if (w & 1)
        lb = f2_add(lb, e2);
      else
        la = f2_add(la, e2);
      float e0, e1;
      f2_split(e2, e0, e1);
      pk[w] = pack2<T>(e0, e1);
    }
    tmem_st_x16(tP + ch * 16, pk);
  }
  float a0, a1, b0, b1;
  f2_split(la, a0, a1);
  f2_split(lb, b0, b1);
  return (a0 + a1) + (b0 + b1);
}

// p = 2^(s * c - m) for scores [C0, C1) of one row: P packed two per word into
// pk (to be stored later), adding the fp32 sum of p into la / lb.
template <typename T, int POLY8, int NC, int C0, int C1>
__device__ __forceinline__ void exp_cols_regs(const float (&s)[NC], uint64_t c2, uint64_t nm2,
                                              uint32_t (&pk)[(C1 - C0) / 2], uint64_t& la,
                                              uint64_t& lb) {
#pragma unroll
  for (int w = 0; w < (C1 - C0) / 2; ++w) {
    const int k = C0 + 2 * w;
    const uint64_t x2 = f2_fma(f2_make(s[k], s[k + 1]), c2, nm2);
    float x0, x1;
    f2_split(x2, x0, x1);
    const uint64_t e2 =
        ((k & 7) < POLY8) ? ex2_poly2(x0, x1) : f2_make(ex2_approx(x0), ex2_approx(x1));
    if (w & 1)
      lb = f2_add(lb, e2);
    else
      la = f2_add(la, e2);
    float e0, e1;
    f2_split(e2, e0, e1);
    pk[w] = pack2<T>(e0, e1);
  }
}

// Own-P layout (d = 64): compute the first half of P into registers before
// waiting for the previous P V product, which may still read P's columns,
// then store it and compute the second half straight into tensor memory (1);
// or wait first and write P as it is computed (0).
#ifndef ETA_PREFILL_OWNP_LATE_WAIT
#define ETA_PREFILL_OWNP_LATE_WAIT 1
#endif

// OUT_F32: O is written as fp32 (O / l, not rounded), for partial results
// that are merged further (tm_o then maps an fp32 tensor with 32 x 32 boxes).
template <int D, typename T, bool CAUSAL, bool WINDOW, int POLY8, bool PINGPONG, int SPLIT = 1,
          bool PREFETCH_Q = false, bool OUT_F32 = false>
__global__ void __launch_bounds__(kernel_threads(SPLIT), 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_o, const Params p) {
  using C = Cfg<D>;
  constexpr int S = C::kStages;
  static_assert(SPLIT == 1 || (SPLIT == 2 && D == 128 && !PINGPONG), "row split");
  constexpr int kMmaWarp = softmax_warps(SPLIT);
  constexpr int kTmaWarp = kMmaWarp + 1;
  constexpr int NC = BN / SPLIT;  // scores per softmax thread and key tile
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);

  uint8_t* sQ = smem + C::kQOff;
  uint8_t* sKV = smem + C::kKVOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + S;
  uint64_t* q_full = kv_empty + S;
  uint64_t* q_empty = q_full + NQT;
  uint64_t* s_ready = q_empty + NQT;
  uint64_t* p_ready = s_ready + NQT;
  uint64_t* o_done = p_ready + NQT;
  uint64_t* turn = o_done + NQT;
  uint64_t* drain = turn + NQT;
  uint64_t* x_up = drain + 1;        // [NQT * 4]
  uint64_t* x_down = x_up + 4 * NQT;  // [NQT * 4]
  uint64_t* s_free = x_down + 4 * NQT;  // [NQT]: the softmax has read S_t (own-P layout)
  uint64_t* pv_done = s_free + NQT;     // [NQT]: P_t V complete (own-P layout)
  constexpr bool OWNP = C::kOwnP;
  static_assert(!OWNP || SPLIT == 1, "own-P layout: one thread per row");
  CtaCtl* ctl = reinterpret_cast<CtaCtl*>(smem + C::kCtlOff);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kCtlOff + 32);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int cta = blockIdx.x;
  const int nkv_all = (p.Nk + BN - 1) / BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < NQT; ++t) {
      mbar_init(&q_full[t], 1);
      mbar_init(&q_empty[t], 1);
      mbar_init(&s_ready[t], 1);
      mbar_init(&p_ready[t], 4 * 32 * SPLIT);
      mbar_init(&o_done[t], 1);
      mbar_init(&turn[t], 4 * 32 * SPLIT);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < 4 * NQT; ++i) {
      mbar_init(&x_up[i], 32);
      mbar_init(&x_down[i], 32);
    }
    for (int t = 0; t < NQT; ++t) {
      mbar_init(&s_free[t], 4 * 32 * SPLIT);
      mbar_init(&pv_done[t], 1);
    }
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
    tma_prefetch_desc(&tm_o);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !(p.debug_flags & 1)) {
      uint32_t L = 0;       // K/V loads issued so far (K_j, V_j alternate)
      int qn[NQT] = {0, 0};  // Q loads issued so far, per tile
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int idx = item_index(r, cta, G);
        if (idx >= p.total) break;
        const Item it = decode_item<CAUSAL, WINDOW>(idx, p, nkv_all);
#pragma unroll
        for (int t = 0; t < NQT; ++t) {
          if ((t ? it.n1 - it.s1 : it.n0 - it.s0) <= 0) continue;
          if (qn[t] > 0 && !(ok = wait_bar(&q_empty[t], (qn[t] - 1) & 1, ctl, kSiteQEmpty)))
            break;
          mbar_arrive_expect_tx(&q_full[t], C::kTileBytes);
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_3d(sQ + t * C::kTileBytes + bx * C::kBoxBytes, &tm_q, &q_full[t], bx * 64,
                        it.r0 + t * BM, it.bh);
          ++qn[t];
        }
        if (PREFETCH_Q) {
          // The next item's Q tiles are read once, from HBM: start them into
          // L2 now (after this item's own Q loads), so that their loads,
          // issued only when this item's last score products have read the
          // current tiles, hit L2.
          const int nidx = item_index(r + 1, cta, G);
          if (nidx < p.total) {
            const Item nx = decode_item<CAUSAL, WINDOW>(nidx, p, nkv_all);
#pragma unroll
            for (int t = 0; t < NQT; ++t) {
              if ((t ? nx.n1 - nx.s1 : nx.n0 - nx.s0) <= 0) continue;
              for (int bx = 0; bx < C::kBoxes; ++bx)
                tma_prefetch_l2_3d(&tm_q, bx * 64, nx.r0 + t * BM, nx.bh);
            }
          }
        }
        const int nmax = max(it.n0, it.n1);
        const int zkv = it.b * p.Hkv + it.kvh;
        for (int l = 0; ok && l < 2 * nmax; ++l, ++L) {
          const uint32_t s = L % S;
          const uint32_t use = L / S;
          if (use > 0 && !(ok = wait_bar(&kv_empty[s], (use - 1) & 1, ctl, kSiteKvEmpty))) break;
          const CUtensorMap* map = (l & 1) ? &tm_v : &tm_k;
          mbar_arrive_expect_tx(&kv_full[s], C::kTileBytes);
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_3d(sKV + s * C::kTileBytes + bx * C::kBoxBytes, map, &kv_full[s], bx * 64,
                        (it.jb + (l >> 1)) * BN, zkv);
        }
      }
      // No copy may still be landing in shared memory when the CTA exits.
#pragma unroll
      for (int t = 0; t < NQT; ++t)
        if (qn[t] > 0) drain_bar(&q_full[t], (qn[t] - 1) & 1, ctl, kSiteDrain);
      for (uint32_t s = 0; s < static_cast<uint32_t>(S) && s < L; ++s) {
        const uint32_t cnt = (L - 1 - s) / S + 1;
        drain_bar(&kv_full[s], (cnt - 1) & 1, ctl, kSiteDrain);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop, so the descriptor arithmetic stays
    // warp-uniform; one elected lane issues each tcgen05 instruction.
    // Descriptors are built once and stepped by adding to the address field of
    // their low word; Q and K are K-major, V is MN-major with its two
    // 64-column halves kBoxBytes apart, and all share the high word.
    constexpr uint32_t fmt = Fmt<T>::value;
    constexpr uint32_t idesc_s = umma_idesc_f16(fmt, BM, BN, 0, 0);
    constexpr uint32_t idesc_pv = umma_idesc_f16(fmt, BM, D, 0, 1);
    const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
    const uint32_t d_hi = static_cast<uint32_t>(dq >> 32);
    const uint32_t q_lo = static_cast<uint32_t>(dq);
    const uint32_t k_lo = static_cast<uint32_t>(smem_desc_sw128(smem_u32(sKV), 16, 1024));
    const uint32_t v_lo =
        static_cast<uint32_t>(smem_desc_sw128(smem_u32(sKV), C::kBoxBytes, 1024));
    uint32_t L = 0;
    int qi[NQT] = {0, 0};
    uint32_t pw[NQT] = {0, 0};
    uint32_t sf[NQT] = {0, 0};  // score products issued per tile (own-P layout)
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int idx = item_index(r, cta, G);
      if (idx >= p.total) break;
      const Item it = decode_item<CAUSAL, WINDOW>(idx, p, nkv_all);
      const int nmax = max(it.n0, it.n1);
      if constexpr (OWNP) {
        // Own-P layout: per key tile j, first the score products S_t(j) (each
        // as soon as the softmax has read S_t(j-1)), then P_t(j-1) V_{j-1}.
        for (int j = 0; ok && j <= nmax; ++j) {
          const uint32_t Lk = L + 2 * j;
          const uint32_t Lv = L + 2 * j - 1;
          bool have_k = false, have_v = false;
#pragma unroll
          for (int t = 0; t < NQT; ++t) {
            const int n = t ? it.n1 : it.n0;
            const int s0 = t ? it.s1 : it.s0;
            if (!ok || !(j >= s0 && j < n)) continue;
            if (!have_k) {
              if (!(ok = warp_all(wait_bar(&kv_full[Lk % S], (Lk / S) & 1, ctl, kSiteKvFull))))
                break;
              tc_fence_after();
              have_k = true;
            }
            if (j == s0) {
              if (!(ok = warp_all(wait_bar(&q_full[t], qi[t] & 1, ctl, kSiteQFull)))) break;
              tc_fence_after();
            }
            if (sf[t] > 0) {  // S_t's columns: the softmax has read the previous scores
              if (!(ok = warp_all(wait_bar(&s_free[t], (sf[t] - 1) & 1, ctl, kSiteSFree)))) break;
              tc_fence_after();
            }
            ++sf[t];
            const uint32_t kd = k_lo + (((Lk % S) * C::kTileBytes) >> 4);
            const uint32_t qd = q_lo + ((t * C::kTileBytes) >> 4);
            const uint32_t tS = tmem + C::s_col(t);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t koff = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
              if (kk == 0)
                umma_ss_w<0>(tS, desc_words(qd + koff, d_hi), desc_words(kd + koff, d_hi), idesc_s);
              else
                umma_ss_w<1>(tS, desc_words(qd + koff, d_hi), desc_words(kd + koff, d_hi), idesc_s);
            }
            umma_commit_w(&s_ready[t]);
            if (j == n - 1) umma_commit_w(&q_empty[t]);
          }
#pragma unroll
          for (int t = 0; t < NQT; ++t) {
            const int n = t ? it.n1 : it.n0;
            const int s0 = t ? it.s1 : it.s0;
            if (!ok || !(j >= 1 && j - 1 >= s0 && j - 1 < n)) continue;
            if (!have_v) {
              if (!(ok = warp_all(wait_bar(&kv_full[Lv % S], (Lv / S) & 1, ctl, kSiteKvFull))))
                break;
              have_v = true;
            }
            if (!(ok = warp_all(wait_bar(&p_ready[t], pw[t] & 1, ctl, kSitePReady)))) break;
            ++pw[t];
            tc_fence_after();
            const uint32_t vd = v_lo + (((Lv % S) * C::kTileBytes) >> 4);
            const uint32_t tP = tmem + C::p_base(t);
            const uint32_t tO = tmem + C::o_col(t);
            if (j - 1 == s0)
              umma_ts_w<0>(tO, tP, desc_words(vd, d_hi), idesc_pv);
            else
              umma_ts_w<1>(tO, tP, desc_words(vd, d_hi), idesc_pv);
#pragma unroll
            for (int kk = 1; kk < BN / 16; ++kk)
              umma_ts_w<1>(tO, tP + kk * 8, desc_words(vd + kk * 128, d_hi), idesc_pv);
            umma_commit_w(&pv_done[t]);
            if (j - 1 == n - 1) umma_commit_w(&o_done[t]);
          }
          if (WINDOW && ok && !have_k && j < nmax) {
            ok = warp_all(wait_bar(&kv_full[Lk % S], (Lk / S) & 1, ctl, kSiteKvFull));
            have_k = ok;
          }
          if (WINDOW && ok && !have_v && j >= 1) {
            ok = warp_all(wait_bar(&kv_full[Lv % S], (Lv / S) & 1, ctl, kSiteKvFull));
            have_v = ok;
          }
          if (have_k) umma_commit_w(&kv_empty[Lk % S]);
          if (have_v) umma_commit_w(&kv_empty[Lv % S]);
        }
      } else {
        for (int j = 0; ok && j <= nmax; ++j) {
          const uint32_t Lk = L + 2 * j;
          const uint32_t Lv = L + 2 * j - 1;
          bool have_k = false, have_v = false;
#pragma unroll
          for (int t = 0; t < NQT; ++t) {
            if (!ok) break;
            const int n = t ? it.n1 : it.n0;
            const int s0 = t ? it.s1 : it.s0;  // this tile's first step
            if (j >= 1 && j - 1 >= s0 && j - 1 < n) {
              // O_t (+)= P_t(j-1) V_{j-1}. The p_ready arrival for an item's
              // first step comes after the softmax group read O_t of its
              // previous item, so O_t is free to be overwritten here.
              if (!have_v) {
                if (!(ok = warp_all(wait_bar(&kv_full[Lv % S], (Lv / S) & 1, ctl, kSiteKvFull))))
                  break;
                have_v = true;
              }
              if (!(ok = warp_all(wait_bar(&p_ready[t], pw[t] & 1, ctl, kSitePReady)))) break;
              ++pw[t];
              tc_fence_after();
              const uint32_t vd = v_lo + (((Lv % S) * C::kTileBytes) >> 4);
              const uint32_t tS = tmem + t * BN;
              const uint32_t tO = tmem + C::kOCol + t * D;
              // P of keys 16kk..16kk+15: 8 columns. With SPLIT = 1 P fills columns
              // [64, 128) of S_t; with SPLIT = 2 the two halves of the row sit at
              // columns [0, 32) and [64, 96), each where its own thread read S.
              // 16 keys = 16 rows of 128 bytes of V (2048 bytes = 128 in the address field)
              if (j - 1 == s0)
                umma_ts_w<0>(tO, tS + p_col<SPLIT>(0), desc_words(vd, d_hi), idesc_pv);
              else
                umma_ts_w<1>(tO, tS + p_col<SPLIT>(0), desc_words(vd, d_hi), idesc_pv);
#pragma unroll
              for (int kk = 1; kk < BN / 16; ++kk)
                umma_ts_w<1>(tO, tS + p_col<SPLIT>(kk), desc_words(vd + kk * 128, d_hi), idesc_pv);
              if (j - 1 == n - 1) umma_commit_w(&o_done[t]);
            }
            if (j >= s0 && j < n) {
              // S_t = Q_t K_j^T
              if (!have_k) {
                if (!(ok = warp_all(wait_bar(&kv_full[Lk % S], (Lk / S) & 1, ctl, kSiteKvFull))))
                  break;
                tc_fence_after();
                have_k = true;
              }
              if (j == s0) {
                if (!(ok = warp_all(wait_bar(&q_full[t], qi[t] & 1, ctl, kSiteQFull)))) break;
                tc_fence_after();
              }
              const uint32_t kd = k_lo + (((Lk % S) * C::kTileBytes) >> 4);
              const uint32_t qd = q_lo + ((t * C::kTileBytes) >> 4);
              const uint32_t tS = tmem + t * BN;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
                if (kk == 0)
                  umma_ss_w<0>(tS, desc_words(qd + koff, d_hi), desc_words(kd + koff, d_hi), idesc_s);
                else
                  umma_ss_w<1>(tS, desc_words(qd + koff, d_hi), desc_words(kd + koff, d_hi), idesc_s);
              }
              umma_commit_w(&s_ready[t]);
              if (j == n - 1) umma_commit_w(&q_empty[t]);
            }
          }
          // A loaded tile that neither query tile uses (a gap between the two
          // tiles' windows; without a window every loaded tile is used) is still
          // waited for and released, so the ring keeps its order.
          if (WINDOW && ok && !have_k && j < nmax) {
            ok = warp_all(wait_bar(&kv_full[Lk % S], (Lk / S) & 1, ctl, kSiteKvFull));
            have_k = ok;
          }
          if (WINDOW && ok && !have_v && j >= 1) {
            ok = warp_all(wait_bar(&kv_full[Lv % S], (Lv / S) & 1, ctl, kSiteKvFull));
            have_v = ok;
          }
          if (have_k) umma_commit_w(&kv_empty[Lk % S]);
          if (have_v) umma_commit_w(&kv_empty[Lv % S]);
        }
      }
      L += 2 * nmax;
      qi[0] += it.n0 > it.s0;
      qi[1] += it.n1 > it.s1;
    }
    // Every MMA must be complete before tensor memory is released.
    umma_commit_w(drain);
    drain_bar(drain, 0, ctl, kSiteDrain);
  } else {
    // ------------------------------------------------------------ softmax
    // Warp w: query tile t = w / (4 SPLIT); row quarter q4 = w % 4 (the
    // tensor-memory lanes a warp may access); column part hw = (w / 4) % SPLIT,
    // i.e. scores [hw NC, (hw + 1) NC) of each of its 32 rows.
    const int t = warp / (4 * SPLIT);
    const int hw = (warp >> 2) % SPLIT;
    const int q4 = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::s_col(t) + hw * NC;
    const uint32_t tP = OWNP ? tmem + lane_off + C::p_base(t)
                             : tmem + lane_off + t * BN + p_col<SPLIT>(hw * (NC / 16));
    const uint32_t tO = tmem + lane_off + C::o_col(t);
    uint32_t np = 0;  // probability tiles written (own-P layout: pv_done phases)
    uint8_t* stg = smem + C::kStgOff + (t * 4 + q4) * C::kStgWarpBytes;  // O staging (hw 0)
    // Split rows: part 1 passes its tile max (then, at the end of an item, its
    // partial row sum) up through xrow; part 0 returns the row max.
    float* xrow = reinterpret_cast<float*>(smem + C::kXOff) + t * BM + q4 * 32 + lane;
    uint64_t* xu = &x_up[t * 4 + q4];
    uint64_t* xd = &x_down[t * 4 + q4];
    uint32_t xp = 0;  // exchange rounds completed
    const float sl2 = p.scale_log2;
    uint32_t sw = 0;  // s_ready phases consumed
    uint32_t od = 0;  // o_done phases consumed
    uint32_t tk = 0;  // turns taken
    bool ok = true;
    if (PINGPONG && t == 1) mbar_arrive(&turn[0]);  // tile 0 takes the first turn
    for (int r = 0; ok; ++r) {
      const int idx = item_index(r, cta, G);
      if (idx >= p.total) break;
      const Item it = decode_item<CAUSAL, WINDOW>(idx, p, nkv_all);
      const int n = t ? it.n1 : it.n0;
      const int s0 = t ? it.s1 : it.s0;  // this tile's first step
      const int rt = it.r0 + t * BM;
      const int row = rt + q4 * 32 + lane;
      float m = -INFINITY;  // running max of s * c (log2 units)
      float l = 0.f;        // running sum of p (this thread's columns)
      for (int i = s0; i < n; ++i) {
        if (!(ok = warp_all(wait_bar(&s_ready[t], sw & 1, ctl, kSiteSReady)))) break;
        ++sw;
        tc_fence_after();
        float s[NC];
        {
          uint32_t rr[NC / 32][32];
#pragma unroll
          for (int h = 0; h < NC / 32; ++h) tmem_ld_x32(tS + h * 32, rr[h]);
#pragma unroll
          for (int h = 0; h < NC / 32; ++h) tmem_wait_ld_x32(rr[h]);
#pragma unroll
          for (int h = 0; h < NC / 32; ++h)
#pragma unroll
            for (int k = 0; k < 32; ++k) s[h * 32 + k] = __uint_as_float(rr[h][k]);
        }
        if (OWNP) {  // S_t read: its columns may take the next scores
          tc_fence_before();
          mbar_arrive(&s_free[t]);
        }
        const int kv0 = (it.jb + i) * BN + hw * NC;  // key of s[0]
        const bool edge = (CAUSAL && kv0 + NC - 1 > rt + p.off) || (kv0 + NC > p.Nk);
        if (edge) {
          const int last = (CAUSAL ? min(row + p.off, p.Nk - 1) : p.Nk - 1) - kv0;
#pragma unroll
          for (int k = 0; k < NC; ++k) s[k] = (k > last) ? -INFINITY : s[k];
        }
        // Sliding window: keys before row + off - window + 1 are out of reach.
        const bool wedge = CAUSAL && WINDOW && kv0 < rt + BM + p.off - p.window;
        if (wedge) {
          const int first = row + p.off - p.window + 1 - kv0;
#pragma unroll
          for (int k = 0; k < NC; ++k) s[k] = (k < first) ? -INFINITY : s[k];
        }
        // four independent chains of 3-input max, NC / 4 columns each
        constexpr int Q = NC / 4;
        float mx0 = fmaxf(s[0], s[1]), mx1 = fmaxf(s[Q], s[Q + 1]);
        float mx2 = fmaxf(s[2 * Q], s[2 * Q + 1]), mx3 = fmaxf(s[3 * Q], s[3 * Q + 1]);
#pragma unroll
        for (int k = 2; k < Q; k += 2) {
          mx0 = fmax3(mx0, s[k], s[k + 1]);
          mx1 = fmax3(mx1, s[Q + k], s[Q + k + 1]);
          mx2 = fmax3(mx2, s[2 * Q + k], s[2 * Q + k + 1]);
          mx3 = fmax3(mx3, s[3 * Q + k], s[3 * Q + k + 1]);
        }
        float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        if (SPLIT == 2) {
          // Both parts must scale the row by the same maximum.
          if (hw == 1) {
            *xrow = m_tile;
            mbar_arrive(xu);
            if (!(ok = warp_all(wait_bar(xd, xp & 1, ctl, kSiteXDown)))) break;
            m_tile = *xrow;
          } else {
            if (!(ok = warp_all(wait_bar(xu, xp & 1, ctl, kSiteXUp)))) break;
            m_tile = fmaxf(m_tile, *xrow);
            *xrow = m_tile;
            mbar_arrive(xd);
          }
          ++xp;
        }
        m_tile *= sl2;
        float alpha = 1.f;
        const bool need = m_tile > m + kRescaleThreshold;
        if (need) {
          alpha = ex2_approx(m - m_tile);  // m = -inf gives 0
          m = m_tile;
          l *= alpha;
        }
        const float m_use = (m == -INFINITY) ? 0.f : m;
        if (PINGPONG && OWNP && np > 0) {
          // Own-P with turns: wait for the previous P_t V product before
          // taking the turn, so a turn is spent on exponentials only.
          if (!(ok = warp_all(wait_bar(&pv_done[t], (np - 1) & 1, ctl, kSitePvDone)))) break;
          tc_fence_after();
        }
        if (PINGPONG) {
          if (!(ok = warp_all(wait_bar(&turn[t], tk & 1, ctl, kSiteTurn)))) break;
          ++tk;
        }
        float lsum;
        if constexpr (OWNP && ETA_PREFILL_OWNP_LATE_WAIT && !PINGPONG) {
          static_assert(NC == 128, "own-P rows");
          const uint64_t c2 = f2_make(sl2, sl2);
          const uint64_t nm2 = f2_make(-m_use, -m_use);
          uint64_t la = f2_make(0.f, 0.f), lb = la;
          uint32_t pa[32], pb[16];
          const bool poly = POLY8 > 0 && !edge && !wedge;  // unmasked tiles only
          if (poly)
            exp_cols_regs<T, POLY8, NC, 0, 64>(s, c2, nm2, pa, la, lb);
          else
            exp_cols_regs<T, 0, NC, 0, 64>(s, c2, nm2, pa, la, lb);
          if (np > 0) {
            if (!(ok = warp_all(wait_bar(&pv_done[t], (np - 1) & 1, ctl, kSitePvDone)))) break;
            tc_fence_after();
          }
          ++np;
          tmem_st_x16(tP, *reinterpret_cast<uint32_t(*)[16]>(pa));
          tmem_st_x16(tP + 16, *reinterpret_cast<uint32_t(*)[16]>(pa + 16));
          if (poly)
            exp_cols_regs<T, POLY8, NC, 64, 96>(s, c2, nm2, pb, la, lb);
          else
            exp_cols_regs<T, 0, NC, 64, 96>(s, c2, nm2, pb, la, lb);
          tmem_st_x16(tP + 32, pb);
          if (poly)
            exp_cols_regs<T, POLY8, NC, 96, 128>(s, c2, nm2, pb, la, lb);
          else
            exp_cols_regs<T, 0, NC, 96, 128>(s, c2, nm2, pb, la, lb);
          tmem_st_x16(tP + 48, pb);
          float a0, a1, b0, b1;
          f2_split(la, a0, a1);
          f2_split(lb, b0, b1);
          lsum = (a0 + a1) + (b0 + b1);
        } else {
          if (OWNP && !PINGPONG && np > 0) {
            // P_t's columns and O_t: the previous P_t V product must be complete.
            if (!(ok = warp_all(wait_bar(&pv_done[t], (np - 1) & 1, ctl, kSitePvDone)))) break;
            tc_fence_after();
          }
          ++np;
          if (POLY8 > 0 && !edge && !wedge)
            lsum = exp_tile<T, POLY8, NC>(s, sl2, m_use, tP);
          else
            lsum = exp_tile<T, 0, NC>(s, sl2, m_use, tP);
        }
        l += lsum;
        if (PINGPONG) mbar_arrive(&turn[t ^ 1]);
        if (i > s0 && __any_sync(0xffffffffu, need)) {
          // O_t was last written by PV_t(i-1), complete before S_t(i) was
          // signalled (own-P layout: waited for through pv_done above). Each
          // part of a split row rescales its share of the columns.
#pragma unroll
          for (int c = hw * (D / 32 / SPLIT); c < (hw + 1) * (D / 32 / SPLIT); ++c) {
            uint32_t o[32];
            tmem_ld_x32(tO + c * 32, o);
            tmem_wait_ld_x32(o);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float a0, a1;
              f2_split(f2_mul(f2_make(__uint_as_float(o[e]), __uint_as_float(o[e + 1])),
                              f2_make(alpha, alpha)),
                       a0, a1);
              o[e] = __float_as_uint(a0);
              o[e + 1] = __float_as_uint(a1);
            }
            tmem_st_x32(tO + c * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_ready[t]);
      }
      if (!ok) break;
      if (PINGPONG) {
        // Keep the turn order in step with the other group: each group takes
        // max(n0, n1) turns per item.
        const int nturns = max(it.n0 - it.s0, it.n1 - it.s1);
        for (int i = n - s0; i < nturns; ++i) {
          if (!(ok = warp_all(wait_bar(&turn[t], tk & 1, ctl, kSiteTurn)))) break;
          ++tk;
          mbar_arrive(&turn[t ^ 1]);
        }
        if (!ok) break;
      }
      if (rt >= p.Nq) continue;  // no rows in this tile
      if (SPLIT == 2) {
        // Part 1 hands its partial row sum to part 0, which writes the row.
        if (hw == 1) {
          *xrow = l;
          mbar_arrive(xu);
          ok = warp_all(wait_bar(xd, xp & 1, ctl, kSiteXDown));
          ++xp;
          if (!ok) break;
          continue;
        }
        if (!(ok = warp_all(wait_bar(xu, xp & 1, ctl, kSiteXUp)))) break;
        l += *xrow;
        mbar_arrive(xd);
        ++xp;
      }
      if (n > s0) {
        if (!(ok = warp_all(wait_bar(&o_done[t], od & 1, ctl, kSiteODone)))) break;
        ++od;
        tc_fence_after();
      }
      const bool has_row = row < p.Nq;
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      if constexpr (OUT_F32) {
        // O in fp32, 32 columns (128 bytes per row) per store: the same
        // swizzled staging of 32 rows x 128 bytes, one 32 x 32 box per store.
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          if (lane == 0) bulk_wait_group_read0();  // the buffer's previous store has read it
          __syncwarp();
          uint32_t o[32];
          if (n > s0) {
            tmem_ld_x32(tO + c * 32, o);
            tmem_wait_ld_x32(o);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0u;
          }
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float a0, a1;
            f2_split(f2_mul(f2_make(__uint_as_float(o[e]), __uint_as_float(o[e + 1])),
                            f2_make(inv_l, inv_l)),
                     a0, a1);
            o[e] = __float_as_uint(a0);
            o[e + 1] = __float_as_uint(a1);
          }
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            uint4* dst = reinterpret_cast<uint4*>(stg + lane * 128 + ((g ^ (lane & 7)) << 4));
            *dst = make_uint4(o[4 * g], o[4 * g + 1], o[4 * g + 2], o[4 * g + 3]);
          }
          fence_async_smem();
          __syncwarp();
          const int y = rt + q4 * 32;
          if (lane == 0 && y < p.Nq) {
            tma_store_3d(&tm_o, stg, c * 32, y, it.bh);
            bulk_commit_group();
          }
        }
      }
      // O in 64-column halves: each lane packs its row's 64 columns into this
      // warp's staging buffer (32 rows x 128 bytes, 128-byte swizzle: 16-byte
      // chunk g of row lane sits at chunk position g ^ (lane % 8)), and one TMA
      // store per half writes the 32 x 64 box (rows past Nq are clipped).
#pragma unroll
      for (int half = 0; half < (OUT_F32 ? 0 : D / 64); ++half) {
        if (lane == 0) bulk_wait_group_read0();  // the buffer's previous store has read it
        __syncwarp();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = half * 2 + cc;
          uint32_t o[32];
          if (n > s0) {
            tmem_ld_x32(tO + c * 32, o);
            tmem_wait_ld_x32(o);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0u;
          }
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float a0, a1;
            f2_split(f2_mul(f2_make(__uint_as_float(o[2 * e]), __uint_as_float(o[2 * e + 1])),
                            f2_make(inv_l, inv_l)),
                     a0, a1);
            w[e] = pack2<T>(a0, a1);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int g = cc * 4 + j;
            uint4* dst = reinterpret_cast<uint4*>(stg + lane * 128 + ((g ^ (lane & 7)) << 4));
            *dst = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          }
        }
        fence_async_smem();
        __syncwarp();
        const int y = rt + q4 * 32;
        if (lane == 0 && y < p.Nq) {
          tma_store_3d(&tm_o, stg, half * 64, y, it.bh);
          bulk_commit_group();
        }
      }
      if (has_row && p.lse != nullptr) {
        p.lse[static_cast<size_t>(it.bh) * p.Nq + row] =
            l > 0.f ? (m + lg2_approx(l)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }

  // Stores of O done before the CTA exits (only part 0 of a row stores).
  if (warp < kMmaWarp && ((warp >> 2) % SPLIT) == 0 && lane == 0) bulk_wait_group0();
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
