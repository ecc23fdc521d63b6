// Exact attention, decode, as one persistent streaming pass on the tensor
// cores (sm_100a), head size 64 or 128, 2 to 32 query heads per KV head.
//
// Generating a token re-reads the whole KV cache of its sequence (first page,
// the token-generation case; zimaspace page, "Reduced IO Is Not the Same as
// Eliminating KV Cache"), so decode is a stream over the cache and its speed
// is the rate at which each SM keeps that stream moving. The work is cut into
// tiles of 128 keys of one (sequence b, KV head g) -- a "segment" -- and the
// tiles of all segments, in order, are divided into contiguous ranges, one
// per CTA (one CTA per SM): equal numbers of tiles, or, for groups above 8
// in batches whose stream plans itself, equal shares of a cost that also
// charges each segment start. A CTA streams its range without a restart at
// segment boundaries: the K/V ring, the score products and the running
// softmax (aikaboom page "11.4d FlashAttention", "Tiling" and "Online
// Softmax") carry on, and at the end of each piece of a segment the CTA
// writes either the result itself (the whole segment lay in its range) or a
// normalised partial with its log-sum-exp, which the gather kernel merges.
//
// Two or three kernels per call:
//   attn_decode_plan_kernel        (batches above 2048 sequences, and the
//                                  whole-segment mode) one CTA: per sequence,
//                                  token offset in the packed cache (int64)
//                                  and tile offset in the global tile order
//                                  (int32 prefix over sequences, KV heads
//                                  included); each CTA's first tile position;
//                                  O = 0, LSE = -inf for empty sequences
//   attn_decode_persistent_kernel  the stream (below); for smaller batches
//                                  each CTA forms the same prefix sums itself
//                                  (and the cost positions, which it records
//                                  for the gather in place of tile offsets)
//   attn_decode_gather_kernel      one warp per (sequence, query head) of a
//                                  segment cut between CTAs: merges its
//                                  partials by their log-sum-exp
//
// Per tile (G query heads of KV head g, padded to NP = 16 or 32):
//   S^T = K_j Q^T      M = 128 keys, N = NP, K = D dims; A = K tile
//                      (K-major), B = Q (K-major); fp32 in tensor memory,
//                      lane = key, column = head (two buffers)
//   softmax            warp w owns keys 32w..32w+31; per head the tile max by
//                      shuffles and across the four warps through shared
//                      memory; p = 2^(s*c - m) with a lazily moved running max
//                      per head; P^T [head][key] rounded to the input type in
//                      shared memory (two buffers); l kept per key slot
//   O^T += V_j^T P^T   M = 128 dims, N = NP, K = 128 keys; A = the V tile read
//                      MN-major (for D = 64 its upper 64 rows read a zeroed
//                      box), B = P^T (K-major); fp32 in tensor memory
// Q of each segment comes in by TMA (two buffers, the next segment's Q loaded
// while the current one runs); K and V by 16-byte cp.async straight into the
// 128-byte-swizzled layout, zero-filled past the segment's last key (the
// packed cache's extent is only known on the device).
//
// Warp roles (HS softmax warps per key quarter): warps 0 .. 4 HS - 1 softmax
// and epilogue, then the tensor memory owner (MMA issue and Q loads, whole
// warp, one elected lane), then three producers, each owning one ring stage.
// Every wait is bounded.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>
#include <type_traits>

#include "common.cuh"
#include "decode_sm100.cuh"

namespace eta {
namespace decode_ps {

constexpr int TK = 128;  // keys per tile
constexpr int kStages = 3;
constexpr int kSoftWarps = 4;  // key quarters of a tile (tensor-memory lane quarters)

// Warp roles for HS softmax warps per key quarter (HS = 2: the two warps of a
// quarter split the heads of its keys): softmax warps 0 .. 4 HS - 1, then the
// MMA warp, then one producer warp per ring stage.
template <int HS>
struct Roles {
  static constexpr int kSoft = kSoftWarps * HS;
  static constexpr int kMma = kSoft;
  static constexpr int kProd0 = kSoft + 1;
  static constexpr int kThreads = 32 * (kProd0 + kStages);
};
constexpr int kThreads = Roles<1>::kThreads;
constexpr float kRescaleThreshold = 8.0f;
constexpr uint32_t kTmemCols = 128;
constexpr int kPlanThreads = 1024;

enum : unsigned {
  kSiteFull = 0x41,
  kSiteEmpty = 0x42,
  kSiteS = 0x43,
  kSiteP = 0x44,
  kSitePv = 0x45,
  kSiteX = 0x46,
  kSiteQ = 0x47,
  kSiteDrain = 0x48,
  kSiteQFree = 0x49,
};

// Bounded mbarrier wait that polls try_wait without a suspend-time hint: the
// stream's waits are short and come every tile. Measured on B200 against the
// sleeping wait: 0.2132 against 0.2153 ms on the ragged group-4 workload,
// 0.2215 / 0.2256 ms at group 8, 0.1478 / 0.1518 ms at group 4 with d = 64.
__device__ __noinline__ bool wait_spin_slow(uint32_t bar, uint32_t parity, CtaCtl* ctl,
                                            unsigned site) {
  const uint64_t t0 = globaltimer_ns();
  volatile int* abort = &ctl->abort;
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((n & 15u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > ctl->wait_ns) {
        *abort = 1;
        record_status(kStatusTimeout | site);
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool wait_bar_spin(uint64_t* bar, uint32_t parity, CtaCtl* ctl,
                                              unsigned site) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  return wait_spin_slow(a, parity, ctl, site);
}

// Byte offset of 16-byte unit u (0..15 along a 256-byte row) of row r in a
// tile of two 128-byte-swizzled boxes (columns 0-63 | 64-127), box_bytes apart.
__device__ __forceinline__ uint32_t sw128_off(int r, int u, int box_bytes) {
  return static_cast<uint32_t>((u >> 3) * box_bytes + r * 128 + (((u & 7) ^ (r & 7)) << 4));
}

// Tensor-memory loads and stores of NP (8, 16 or 32) consecutive columns.
template <int NP>
__device__ __forceinline__ void tmem_ld_np(uint32_t taddr, uint32_t (&r)[NP]);
template <>
__device__ __forceinline__ void tmem_ld_np<8>(uint32_t taddr, uint32_t (&r)[8]) {
  tmem_ld_x8(taddr, r);
  tmem_wait_ld_x8(r);
}
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
__device__ __forceinline__ void tmem_st_np<8>(uint32_t taddr, const uint32_t (&r)[8]) {
  tmem_st_x8(taddr, r);
}
template <>
__device__ __forceinline__ void tmem_st_np<16>(uint32_t taddr, const uint32_t (&r)[16]) {
  tmem_st_x16(taddr, r);
}
template <>
__device__ __forceinline__ void tmem_st_np<32>(uint32_t taddr, const uint32_t (&r)[32]) {
  tmem_st_x32(taddr, r);
}

// fp32 -> bf16 / fp16 bits, round to nearest even.
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

struct PParams {
  const void* q;
  const void* kc;
  const void* vc;
  const int* seqlens;
  const long long* tok_off;  // [B]: token offset of sequence b in the packed cache
  const int* tile_off;       // [B + 1]: first global tile of sequence b (all its KV heads);
                             // with wcost > 0 its first cost position (see wcost)
  void* o;                   // [B][Hq][D], input type (D = 64 or 128: the kernels' template)
  float* lse;                // [B][Hq] natural log, or NULL
  float* part_o;             // [slots][G][D]: normalised partial O of a cut segment
  float* part_lse;           // [slots][G]: its log-sum-exp, log2 units
  int4* starts;              // [nc]: (b, g, i) of each CTA's first tile (equal tile ranges)
  int B;
  int Hq;
  int Hkv;
  int G;
  int window;       // > 0: each new token reads only the last `window` cached tokens
  int seg_aligned;  // 1: CTAs take whole segments (no partials); 0: equal tile ranges
  int inline_plan;  // 1: no plan kernel; each CTA finds its range from seqlens itself
  int wcost;        // inline plan only: each segment costs wcost tiles more than its own, and
                    // the CTAs take equal shares of that cost (0: equal shares of the tiles)
  float scale_log2;
  uint64_t wait_ns;
};

// Programmatic dependent launch: a grid launched with programmatic stream
// serialisation may start before the previous kernel on the stream ends;
// griddepcontrol.wait blocks until that kernel has completed and its memory
// writes are visible, and launch_dependents lets the next such grid start.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Keys of sequence b read: [first_key, len).
__device__ __forceinline__ int first_key(int len, int window) {
  return (window > 0 && len > window) ? len - window : 0;
}

// ------------------------------------------------------------------ plan
// Exclusive prefix sums over the B sequences (one CTA): token offsets of the
// packed cache and tile offsets of the global tile order (Hkv segments of
// ceil(keys read / 128) tiles per sequence). tile_off[B] is the total.
template <int D>
__global__ void __launch_bounds__(kPlanThreads) attn_decode_plan_kernel(const PParams p, int nc) {
  const int* __restrict__ seqlens = p.seqlens;
  long long* __restrict__ tok_off = const_cast<long long*>(p.tok_off);
  int* __restrict__ tile_off = const_cast<int*>(p.tile_off);
  const int B = p.B, Hkv = p.Hkv, window = p.window;
  __shared__ long long s_tok[kPlanThreads / 32];
  __shared__ long long s_til[kPlanThreads / 32];
  griddep_launch_dependents();  // the stream kernel may start its set-up now
  const int per = (B + kPlanThreads - 1) / kPlanThreads;  // consecutive sequences per thread
  const int b0 = threadIdx.x * per;
  const int b1 = min(B, b0 + per);
  long long tok = 0, til = 0;
  for (int b = b0; b < b1; ++b) {
    const int len = max(seqlens[b], 0);
    tok += len;
    til += static_cast<long long>(Hkv) * ((len - first_key(len, window) + TK - 1) / TK);
  }
  // inclusive scan over the block: warps, then warp totals
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long xt = tok, xl = til;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long yt = __shfl_up_sync(0xffffffffu, xt, o);
    const long long yl = __shfl_up_sync(0xffffffffu, xl, o);
    if (lane >= o) {
      xt += yt;
      xl += yl;
    }
  }
  if (lane == 31) {
    s_tok[warp] = xt;
    s_til[warp] = xl;
  }
  __syncthreads();
  if (warp == 0) {
    long long wt = s_tok[lane], wl = s_til[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long yt = __shfl_up_sync(0xffffffffu, wt, o);
      const long long yl = __shfl_up_sync(0xffffffffu, wl, o);
      if (lane >= o) {
        wt += yt;
        wl += yl;
      }
    }
    s_tok[lane] = wt;
    s_til[lane] = wl;
  }
  __syncthreads();
  long long t_run = xt - tok + (warp > 0 ? s_tok[warp - 1] : 0);  // exclusive
  long long l_run = xl - til + (warp > 0 ? s_til[warp - 1] : 0);
  const long long T = s_til[31];  // all tiles
  for (int b = b0; b < b1; ++b) {
    const int len = max(seqlens[b], 0);
    const int nt = (len - first_key(len, window) + TK - 1) / TK;
    tok_off[b] = t_run;
    tile_off[b] = static_cast<int>(l_run);
    if (nt == 0) {
      // An empty sequence: no CTA visits it. O = 0, LSE = -inf.
      for (int h = 0; h < p.Hq; ++h) {
        const size_t row = static_cast<size_t>(b) * p.Hq + h;
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.o) + row * D);
        for (int u = 0; u < D / 8; ++u) dst[u] = make_uint4(0u, 0u, 0u, 0u);
        if (p.lse != nullptr) p.lse[row] = -INFINITY;
      }
    } else if (!p.seg_aligned) {
      // CTAs of the equal tile ranges whose first tile lies in this sequence:
      // CTA c starts at tile c * T / nc.
      const long long span = static_cast<long long>(Hkv) * nt;
      for (long long c = (l_run * nc + T - 1) / T; c < nc && c * T / nc < l_run + span; ++c) {
        const long long lo = c * T / nc;
        if (lo >= (c + 1) * T / nc) continue;  // an empty range: the CTA does nothing
        const int r = static_cast<int>(lo - l_run);
        p.starts[c] = make_int4(b, r / nt, r % nt, 0);
      }
    }
    t_run += len;
    l_run += static_cast<long long>(Hkv) * nt;
  }
  if (threadIdx.x == kPlanThreads - 1) tile_off[B] = static_cast<int>(T);
}

// Tile range [lo, hi) of CTA c of nc in the global tile order.
struct Range {
  long long lo, hi;
};

__device__ __forceinline__ long long segment_start(const PParams& p, long long s, long long T) {
  const long long S = static_cast<long long>(p.B) * p.Hkv;
  if (s >= S) return T;
  const int b = static_cast<int>(s / p.Hkv);
  const int g = static_cast<int>(s - static_cast<long long>(b) * p.Hkv);
  const int nt = (p.tile_off[b + 1] - p.tile_off[b]) / p.Hkv;
  return p.tile_off[b] + static_cast<long long>(g) * nt;
}

__device__ __forceinline__ Range cta_range(const PParams& p, int c, int nc) {
  const long long T = p.tile_off[p.B];
  Range r;
  if (p.seg_aligned) {
    const long long S = static_cast<long long>(p.B) * p.Hkv;
    r.lo = segment_start(p, c * S / nc, T);
    r.hi = segment_start(p, (c + 1) * S / nc, T);
  } else {
    r.lo = c * T / nc;
    r.hi = (c + 1) * T / nc;
  }
  return r;
}

// n / d for 0 <= n, 0 < d: a 32-bit division when both fit (the usual case;
// a 64-bit division is a long instruction sequence on the GPU).
__host__ __device__ __forceinline__ long long div_nonneg(long long n, long long d) {
  if (((n | d) >> 31) == 0)
    return static_cast<long long>(static_cast<unsigned>(n) / static_cast<unsigned>(d));
  return n / d;
}

// The CTA whose equal tile range holds global tile t (tile-balanced mode).
__host__ __device__ __forceinline__ int cta_of(long long t, long long T, int nc) {
  return static_cast<int>(div_nonneg((t + 1) * nc - 1, T));
}

// Position of a global tile: sequence b, KV head g, tile i of nt in the segment.
struct Cursor {
  int b, g, i, nt;
  int len, k0;        // keys read of sequence b: [k0, len)
  long long tok;      // token offset of sequence b

  // Length, first key and tile count of sequence b (tok is kept by the caller).
  __device__ __forceinline__ void load_seq(const PParams& p) {
    len = max(p.seqlens[b], 0);
    k0 = first_key(len, p.window);
    nt = (len - k0 + TK - 1) / TK;
  }
  __device__ __forceinline__ void seek(const PParams& p, long long t) {
    int lo = 0, hi = p.B - 1;  // largest b with tile_off[b] <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.tile_off[mid] <= t)
        lo = mid;
      else
        hi = mid - 1;
    }
    b = lo;
    load_seq(p);
    tok = p.tok_off[b];
    const int r = static_cast<int>(t - p.tile_off[b]);
    g = r / nt;
    i = r - g * nt;
  }
  // Advance one tile (the caller never advances past its range's last tile).
  __device__ __forceinline__ void next(const PParams& p) {
    if (++i < nt) return;
    i = 0;
    if (++g < p.Hkv) return;
    g = 0;
    do {  // the next sequence with keys; token offsets move by each length
      tok += len;
      ++b;
      load_seq(p);
    } while (nt == 0 && b < p.B - 1);
  }
  __device__ __forceinline__ int segment(const PParams& p) const { return b * p.Hkv + g; }
};

template <int NP, int D>
struct PCfg {
  static_assert(NP == 16 || NP == 32, "padded group");
  static_assert(D == 64 || D == 128, "head size");
  static constexpr int kBoxes = D / 64;               // 128-byte-swizzled boxes per row
  static constexpr int kBoxBytes = TK * 128;          // 128 keys x 64 dims
  static constexpr int kTileBytes = kBoxes * kBoxBytes;  // K or V tile
  // A stage holds the K tile, then the V tile. With D = 64 the product
  // O^T += V^T P^T still runs with M = 128 (the layout of the D = 128 pass):
  // its second 64-row half of A reads a zeroed box after the V tile, so rows
  // 64..127 of O^T stay zero and are never stored.
  static constexpr int kZeroBytes = D == 64 ? kBoxBytes : 0;
  static constexpr int kStageBytes = 2 * kTileBytes + kZeroBytes;
  static constexpr int kQBox = NP * 128;              // NP rows x 64 dims (or 64 keys)
  static constexpr int kQBuf = kBoxes * kQBox;        // one Q
  static constexpr int kQOff = kStages * kStageBytes;
  static constexpr int kPBuf = 2 * kQBox;             // P^T: 2 boxes of 64 keys
  static constexpr int kPOff = kQOff + 2 * kQBuf;
  static constexpr int kRedOff = kPOff + 2 * kPBuf;   // [2][warps][NP] floats
  // full[S], empty[S], s_ready[2], p_ready[2], x_bar[2], q_full[2], q_free[2], pv_done[2],
  // drain, first_issued[2], full_v[S], empty_v[S]
  static constexpr int kBarOff = kRedOff + 2 * kSoftWarps * NP * 4;
  static constexpr int kNumBars = 4 * kStages + 10 + 3 + 2;
  static constexpr int kCtlOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kCtlOff + 64 + 1024;  // + runtime 1024-byte alignment
  static_assert(kQOff % 1024 == 0 && kPOff % 1024 == 0 && kQBox % 1024 == 0, "swizzle atoms");
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

// Warp-wide max of x (every lane gets it) by one redux.sync on an
// order-preserving integer image of the float (non-negative floats keep their
// bits; negative ones flip the 31 magnitude bits, so larger magnitudes sort
// lower).
__device__ __forceinline__ float warp_max_redux(float x) {
  const int i = __float_as_int(x);
  const int k = __reduce_max_sync(0xffffffffu, i >= 0 ? i : (i ^ 0x7fffffff));
  return __int_as_float(k >= 0 ? k : (k ^ 0x7fffffff));
}

// Producers issue their first stages one after another (1), so that the
// first tile's bytes are not interleaved with the second and third stages'
// in the memory system, or all at once (0). Measured on B200 (64 sequences of
// 1K-8K tokens): with whole stages released at once, 1 was faster (group 4
// 0.2072 against 0.2092 ms, MQA 0.0597 / 0.0618 ms); with K and V released
// separately, 0 is (group 4 0.1989-0.2009 against 0.2030 ms, group 8 0.2010
// / 0.2046 ms, 512-sequence MQA 0.2194 / 0.2235 ms, group 16 at d = 64
// 0.1580 / 0.1600 ms; MQA equal; 256 short sequences 0.1170 / 0.1150 ms).
#ifndef ETA_DECODE_PS_STAGGER
#define ETA_DECODE_PS_STAGGER 0
#endif

// A stage's K tile is released when the score product has read it and its V
// tile when the P V product has, each loaded on its own barrier, so the next
// K copies start while this tile's softmax runs (1); or the stage is released
// and loaded as a whole (0).
#ifndef ETA_DECODE_PS_KV_SPLIT
#define ETA_DECODE_PS_KV_SPLIT 1
#endif

// Per-tile head maxima by redux.sync (1) or by the shuffle reduce-scatter (0).
#ifndef ETA_DECODE_PS_REDUX
#define ETA_DECODE_PS_REDUX 0
#endif

// After a piece's first tile, the softmax warps first vote (one flag per
// warp through the exchange) on whether any score of the tile lies more than
// the rescale threshold above its head's running maximum; only then are the
// tile maxima reduced and exchanged (1). Or always exchange the maxima (0).
// Both keep the same running maxima, so the results are identical.
#ifndef ETA_DECODE_PS_VOTE
#define ETA_DECODE_PS_VOTE 1
#endif

struct MaxOp {
  __device__ __forceinline__ float operator()(float a, float b) const { return fmaxf(a, b); }
};
struct AddOp {
  __device__ __forceinline__ float operator()(float a, float b) const { return a + b; }
};

// Combine v[0..GP) over the 32 lanes of the warp; lane l returns the result
// for entry l % GP. Butterfly steps with offsets 16 .. GP combine whole
// arrays; then each step with offset M < GP hands over half of the remaining
// entries (a reduce-scatter): (GP - 1) + GP * log2(32 / GP) shuffles in all,
// against 5 * GP for a full butterfly per entry.
template <int GP, typename Op>
__device__ __forceinline__ float reduce_scatter(float (&v)[GP], int lane, Op op) {
#pragma unroll
  for (int M = 16; M >= GP; M >>= 1)
#pragma unroll
    for (int j = 0; j < GP; ++j) v[j] = op(v[j], __shfl_xor_sync(0xffffffffu, v[j], M));
#pragma unroll
  for (int M = GP / 2; M >= 1; M >>= 1) {
    const bool up = (lane & M) != 0;
#pragma unroll
    for (int j = 0; j < M; ++j) {
      const float send = up ? v[j] : v[j + M];
      const float keep = up ? v[j + M] : v[j];
      v[j] = op(keep, __shfl_xor_sync(0xffffffffu, send, M));
    }
  }
  return v[0];
}

// out[h] = op over the four softmax warps of red[w * NP + h], h < GP, read as
// 16-byte vectors (every thread reads the same words: broadcasts).
template <int GP, int NP, typename Op>
__device__ __forceinline__ void gather4(const float* red, float (&out)[GP], Op op) {
  const float4* r4 = reinterpret_cast<const float4*>(red);
#pragma unroll
  for (int q = 0; q < GP / 4; ++q) {
    float4 a = r4[q];
#pragma unroll
    for (int w = 1; w < kSoftWarps; ++w) {
      const float4 b = r4[w * (NP / 4) + q];
      a.x = op(a.x, b.x);
      a.y = op(a.y, b.y);
      a.z = op(a.z, b.z);
      a.w = op(a.w, b.w);
    }
    out[4 * q] = a.x;
    out[4 * q + 1] = a.y;
    out[4 * q + 2] = a.z;
    out[4 * q + 3] = a.w;
  }
}

// NP: MMA width (the group padded to 16 or 32); GP <= NP: the heads the
// softmax processes (the group padded to 4, 8, 16 or 32); HS: softmax warps
// per key quarter (1, 2 or 4), each taking GP / HS >= 4 of the heads.
template <int NP, int GP, int HS, int D, typename T>
__global__ void __launch_bounds__(Roles<HS>::kThreads, 1)
    attn_decode_persistent_kernel(const __grid_constant__ CUtensorMap tm_q, const PParams p) {
  static_assert(GP == 4 || GP == 8 || GP == 16 || GP == 32, "softmax group");
  static_assert(GP <= NP && (GP > 16) == (NP == 32), "widths");
  static_assert((HS == 1 || HS == 2 || HS == 4) && GP % HS == 0 && GP / HS >= 4, "head split");
  using C = PCfg<NP, D>;
  using R = Roles<HS>;
  constexpr int GPT = GP / HS;  // heads per softmax thread
  // Tensor-memory columns a softmax thread moves at a time: its own heads
  // (at least 8; GPT = 4 occurs only with one warp per quarter, whose other 4
  // columns are padding no other warp owns, so the rescale may write them).
  static_assert(HS == 1 || GPT >= 8, "shared quarters need 8 heads per thread");
  constexpr int TW = GPT < 8 ? 8 : GPT;
  const int c = blockIdx.x;

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
  uint64_t* q_free = q_full + 2;
  // pv_done[j % 2] completes once per product PV(j) of the tiles j of that
  // parity: a softmax thread that waits for PV(j) knows PV(j - 2) is done (its
  // S(j) followed it), so the phase it waits for is never ambiguous, whether
  // or not PV(j - 1) has run yet.
  uint64_t* pv_done = q_free + 2;
  uint64_t* drain = pv_done + 2;
  uint64_t* first_issued = drain + 1;  // producer p -> p + 1: its first stage's copies are issued
  // With the K/V split, full / empty track a stage's K tile and these its V tile.
  uint64_t* full_v = first_issued + 2;
  uint64_t* empty_v = full_v + kStages;
  static_assert(sizeof(CtaCtl) <= 16, "control words, then the plan's range ends at +16");
  CtaCtl* ctl = reinterpret_cast<CtaCtl*>(smem + C::kCtlOff);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kCtlOff + 32);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 32) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 32);  // one cp.async arrival per producer lane
      mbar_init(&empty[s], 1);
      mbar_init(&full_v[s], 32);
      mbar_init(&empty_v[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_ready[i], 1);
      mbar_init(&p_ready[i], 32 * R::kSoft);
      mbar_init(&x_bar[i], 32 * R::kSoft);
      mbar_init(&q_full[i], 1);
      mbar_init(&q_free[i], 1);
    }
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(drain, 1);
    mbar_init(&first_issued[0], 1);
    mbar_init(&first_issued[1], 1);
    ctl->abort = 0;
    ctl->wait_ns = p.wait_ns;
    fence_mbar_init();
  }
  if (warp == R::kMma) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
    if (lane == 0) tma_prefetch_desc(&tm_q);
  }
  if constexpr (C::kZeroBytes > 0) {
    // the zeroed second half of each stage's V operand (read by the tensor core)
    for (int i = threadIdx.x; i < kStages * C::kZeroBytes / 16; i += R::kThreads) {
      const int st = i / (C::kZeroBytes / 16), u = i - st * (C::kZeroBytes / 16);
      *reinterpret_cast<uint4*>(smem + st * C::kStageBytes + 2 * C::kTileBytes + u * 16) =
          make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tS0 = tmem;          // S^T buffers: columns [0, NP), [NP, 2 NP)
  const uint32_t tO = tmem + 2 * NP;  // O^T: columns [2 NP, 3 NP)
  const int G = p.G;

  // The kernel launched just before this one (the plan, or the caller's last
  // kernel when the plan is inline) may still be running: this grid starts
  // early (programmatic dependent launch), the set-up above overlaps it, and
  // this wait returns once its writes are visible. The gather grid after this
  // one may then start and wait in the same way.
  griddep_wait();
  griddep_launch_dependents();
  Range rg;
  Cursor cur;
  if (p.inline_plan) {
    // Prefix sums over the sequences in this CTA (small batches): the total
    // tile count, this CTA's range and its first tile, without a plan kernel.
    // Cost positions: each non-empty segment takes wcost positions, then one
    // per tile; CTA c takes the tiles whose positions lie in
    // [c C / nc, (c + 1) C / nc) of the C positions (wcost = 0: equal tile
    // shares). CTA 0 also writes the sequences' first cost positions, which
    // the gather kernel reads, and CTA b % nc writes O = 0, LSE = -inf for an
    // empty sequence b. The token sums carry the count of non-empty sequences
    // in their top 16 bits.
    constexpr long long kSeqOne = 1ll << 48;
    long long* wsum = reinterpret_cast<long long*>(red);  // [warps][2], free before the stream
    volatile long long* start = reinterpret_cast<volatile long long*>(smem + C::kCtlOff + 40);
    const int nthr = R::kThreads, nw = nthr / 32;
    // [0]: the range's end tile, [1]: its first; between the CTA's control
    // words and the tensor-memory address (not in `red`, which the softmax
    // warps take over once the stream runs).
    volatile long long* ends = reinterpret_cast<volatile long long*>(smem + C::kCtlOff + 16);
    const int per = (p.B + nthr - 1) / nthr;
    const int b0 = threadIdx.x * per, b1 = min(p.B, b0 + per);
    const int w = p.wcost;
    long long til = 0, tok = 0;
    for (int b = b0; b < b1; ++b) {
      const int len = max(p.seqlens[b], 0);
      const int nt = (len - first_key(len, p.window) + TK - 1) / TK;
      tok += len + (nt > 0 ? kSeqOne : 0);
      til += static_cast<long long>(p.Hkv) * nt;
    }
    long long xt = til, xk = tok;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long yt = __shfl_up_sync(0xffffffffu, xt, o);
      const long long yk = __shfl_up_sync(0xffffffffu, xk, o);
      if (lane >= o) {
        xt += yt;
        xk += yk;
      }
    }
    if (lane == 31) {
      wsum[2 * warp] = xt;
      wsum[2 * warp + 1] = xk;
    }
    if (threadIdx.x == 0) {
      start[0] = -1;
      ends[0] = -1;  // (no end found: all tiles)
    }
    __syncthreads();
    if (warp == 0) {
      long long wt = lane < nw ? wsum[2 * lane] : 0, wk = lane < nw ? wsum[2 * lane + 1] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long yt = __shfl_up_sync(0xffffffffu, wt, o);
        const long long yk = __shfl_up_sync(0xffffffffu, wk, o);
        if (lane >= o) {
          wt += yt;
          wk += yk;
        }
      }
      __syncwarp();
      if (lane < nw) {
        wsum[2 * lane] = wt;
        wsum[2 * lane + 1] = wk;
      }
    }
    __syncthreads();
    const long long T_all = wsum[2 * (nw - 1)];
    const long long wseg = static_cast<long long>(w) * p.Hkv;  // cost positions before a sequence's tiles
    const long long C_all = T_all + wseg * (wsum[2 * (nw - 1) + 1] >> 48);
    long long l_run = xt - til + (warp > 0 ? wsum[2 * (warp - 1)] : 0);  // exclusive
    long long t_run = xk - tok + (warp > 0 ? wsum[2 * (warp - 1) + 1] : 0);
    long long k_run = l_run + wseg * (t_run >> 48);
    t_run &= kSeqOne - 1;
    const long long x_lo = div_nonneg(c * C_all, gridDim.x);
    const long long x_hi = div_nonneg((c + 1) * C_all, gridDim.x);
    for (int b = b0; b < b1; ++b) {
      const int len = max(p.seqlens[b], 0);
      const int nt = (len - first_key(len, p.window) + TK - 1) / TK;
      const long long span = static_cast<long long>(p.Hkv) * nt;
      const long long kspan = nt > 0 ? span + wseg : 0;
      if (c == 0) const_cast<int*>(p.tile_off)[b] = static_cast<int>(k_run);
      if (nt == 0 && b % static_cast<int>(gridDim.x) == c) {
        for (int h = 0; h < p.Hq; ++h) {
          const size_t row = static_cast<size_t>(b) * p.Hq + h;
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.o) + row * D);
          for (int u = 0; u < D / 8; ++u) dst[u] = make_uint4(0u, 0u, 0u, 0u);
          if (p.lse != nullptr) p.lse[row] = -INFINITY;
        }
      }
      // The tile at or after cost position x of this sequence, as its rank
      // g nt + i among the sequence's tiles (segment g, tile i; one of a
      // segment's wcost leading positions gives its first tile). Segments
      // are stepped over rather than divided: the start of the kernel is
      // kept short (its instructions are fetched cold).
      auto rank_at = [&](long long x) {
        int r = static_cast<int>(x - k_run), g = 0;
        while (r >= nt + w) {
          r -= nt + w;
          ++g;
        }
        return static_cast<long long>(g) * nt + max(r - w, 0);
      };
      if (k_run <= x_lo && x_lo < k_run + kspan) {
        const long long rk = rank_at(x_lo);
        start[0] = b;
        start[1] = rk;
        start[2] = t_run;
        ends[1] = l_run + rk;
      }
      if (k_run <= x_hi && x_hi < k_run + kspan) ends[0] = l_run + rank_at(x_hi);
      l_run += span;
      k_run += kspan;
      t_run += len;
    }
    if (c == 0 && threadIdx.x == 0) const_cast<int*>(p.tile_off)[p.B] = static_cast<int>(C_all);
    __syncthreads();
    rg.lo = rg.hi = 0;  // no tiles at all
    if (start[0] >= 0) {
      rg.lo = ends[1];
      rg.hi = ends[0] >= 0 ? ends[0] : T_all;
    }
    if (rg.lo < rg.hi) {
      cur.b = static_cast<int>(start[0]);
      cur.load_seq(p);
      const int r = static_cast<int>(start[1]);
      cur.g = r / cur.nt;
      cur.i = r - cur.g * cur.nt;
      cur.tok = start[2];
    }
  } else {
    rg = cta_range(p, c, gridDim.x);
    if (rg.hi > rg.lo) {
      if (p.seg_aligned) {
        cur.seek(p, rg.lo);
      } else {  // the plan found this CTA's first tile
        const int4 st = p.starts[c];
        cur.b = st.x;
        cur.load_seq(p);
        cur.tok = p.tok_off[cur.b];
        cur.g = st.y;
        cur.i = st.z;
      }
    }
  }
  const int n = rg.hi > rg.lo ? static_cast<int>(rg.hi - rg.lo) : 0;  // tiles of this CTA

  if (n == 0) {
    // no tiles for this CTA (uniform over the CTA)
  } else if (warp >= R::kProd0) {
    // ------------------------------------------------------------ producers
    // Producer pw fills stage pw with the CTA's tiles pw, pw + 3, ... A cache
    // row is UPR = D / 8 units of 16 bytes; lane l copies unit l % UPR of rows
    // RPI i + l / UPR (RPI = 32 / UPR rows per instruction): each instruction
    // reads whole cache rows.
    constexpr int UPR = D / 8, RPI = 32 / UPR;
    const int pw = warp - R::kProd0;
    bool ok = true;
    const uint32_t kdst = smem_u32(smem + pw * C::kStageBytes);
    const uint32_t vdst = kdst + C::kTileBytes;
    const int u = lane % UPR;
    for (int a = 0; a < pw && a + 1 < n; ++a) cur.next(p);  // to tile pw (if in range)
    for (int j = pw; ok && j < n; j += kStages) {
      const int use = j / kStages;
      if (use > 0 &&
          !(ok = decode::warp_all_d(wait_bar_spin(&empty[pw], (use - 1) & 1, ctl, kSiteEmpty))))
        break;
      if (ETA_DECODE_PS_STAGGER && use == 0 && pw > 0 &&
          !(ok = decode::warp_all_d(wait_bar_spin(&first_issued[pw - 1], 0, ctl, kSiteEmpty))))
        break;  // the first stages go out in order, so the first tile lands first
      const size_t head_base =
          (static_cast<size_t>(cur.tok) * p.Hkv + static_cast<size_t>(cur.g) * cur.len) * D;
      const T* kbase = reinterpret_cast<const T*>(p.kc) + head_base;
      const T* vbase = reinterpret_cast<const T*>(p.vc) + head_base;
      const int t0 = cur.k0 + cur.i * TK;
      if constexpr (ETA_DECODE_PS_KV_SPLIT) {
        // K, then (once PV(j - 3) has read the stage's V tile) V; each
        // arrival fires when all this lane's earlier copies have landed.
#pragma unroll 4
        for (int i = 0; i < TK / RPI; ++i) {
          const int r = RPI * i + lane / UPR;
          const int key = t0 + r;
          const bool valid = key < cur.len;
          const size_t row = static_cast<size_t>(valid ? key : t0);  // t0 < len: a real row
          cp_async16(kdst + sw128_off(r, u, C::kBoxBytes), kbase + row * D + u * 8, valid ? 16u : 0u);
        }
        cp_async_mbar_arrive_noinc(&full[pw]);
        if (use > 0 &&
            !(ok = decode::warp_all_d(wait_bar_spin(&empty_v[pw], (use - 1) & 1, ctl, kSiteEmpty))))
          break;
#pragma unroll 4
        for (int i = 0; i < TK / RPI; ++i) {
          const int r = RPI * i + lane / UPR;
          const int key = t0 + r;
          const bool valid = key < cur.len;
          const size_t row = static_cast<size_t>(valid ? key : t0);
          cp_async16(vdst + sw128_off(r, u, C::kBoxBytes), vbase + row * D + u * 8, valid ? 16u : 0u);
        }
        cp_async_mbar_arrive_noinc(&full_v[pw]);
      } else {
#pragma unroll 4
        for (int i = 0; i < TK / RPI; ++i) {
          const int r = RPI * i + lane / UPR;
          const int key = t0 + r;
          const bool valid = key < cur.len;
          const size_t row = static_cast<size_t>(valid ? key : t0);  // t0 < len: a real row
          const uint32_t nb = valid ? 16u : 0u;                     // 0: zero-fill, no read
          const uint32_t off = sw128_off(r, u, C::kBoxBytes);
          cp_async16(kdst + off, kbase + row * D + u * 8, nb);
          cp_async16(vdst + off, vbase + row * D + u * 8, nb);
        }
        cp_async_mbar_arrive_noinc(&full[pw]);
      }
      if (ETA_DECODE_PS_STAGGER && use == 0 && pw + 1 < kStages) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&first_issued[pw]);
      }
      for (int a = 0; a < kStages && j + 1 + a < n; ++a) cur.next(p);
    }
    cp_async_wait_all();  // no copy may land after the CTA exits
  } else if (warp == R::kMma) {
    // ------------------------------------------------------------ MMA issue and Q loads
    constexpr uint32_t fmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
    constexpr uint32_t idesc_s = umma_idesc_f16(fmt, TK, NP, 0, 0);
    constexpr uint32_t idesc_pv = umma_idesc_f16(fmt, 128, NP, 1, 0);  // M = 128 (zero-padded for D = 64)
    const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
    const uint32_t d_hi = static_cast<uint32_t>(dq >> 32);
    const uint32_t q_lo = static_cast<uint32_t>(dq);
    const uint32_t k_lo = static_cast<uint32_t>(smem_desc_sw128(smem_u32(smem), 16, 1024));
    const uint32_t v_lo = static_cast<uint32_t>(
        smem_desc_sw128(smem_u32(smem + C::kTileBytes), C::kBoxBytes, 1024));
    const uint32_t p_lo = static_cast<uint32_t>(smem_desc_sw128(smem_u32(sP), 16, 1024));
    // Q of piece k goes to buffer k % 2 (its G rows; rows G..NP-1 are zero-filled
    // by the copy as out of bounds). The first piece's Q is loaded here.
    int nq0 = 0, nq1 = 0;  // Q loads issued per buffer (scalars: no local-memory array)
    auto load_q = [&](int buf, int seg) {
      if (buf)
        ++nq1;
      else
        ++nq0;
      if (lane == 0) {
        mbar_arrive_expect_tx(&q_full[buf], C::kQBuf);
        for (int bx = 0; bx < C::kBoxes; ++bx)
          tma_load_3d(sQ + buf * C::kQBuf + bx * C::kQBox, &tm_q, &q_full[buf], bx * 64, 0, seg);
      }
      __syncwarp();
    };
    load_q(0, cur.segment(p));
    bool ok = true;
    int k = -1;                // current piece
    bool prev_first = false;   // tile j - 1 started its piece
    uint32_t qb = 0;
    for (int j = 0; ok && j <= n; ++j) {
      if (j < n) {
        const bool first = (j == 0) || (cur.i == 0);
        const bool last = (j == n - 1) || (cur.i == cur.nt - 1);
        if (first) {
          ++k;
          qb = k & 1;
          if (!(ok = decode::warp_all_d(wait_bar_spin(&q_full[qb], (k >> 1) & 1, ctl, kSiteQ)))) break;
          tc_fence_after();
        }
        // S^T(j) = K_j Q^T into buffer j % 2 (its previous scores, of tile
        // j - 2, were read before p_ready(j - 2), waited for last iteration).
        const int st = j % kStages;
        if (!(ok = decode::warp_all_d(wait_bar_spin(&full[st], (j / kStages) & 1, ctl, kSiteFull))))
          break;
        fence_proxy_async_smem();  // the cp.async data is read by the tensor core
        tc_fence_after();
        const uint32_t kd = k_lo + ((st * C::kStageBytes) >> 4);
        const uint32_t qd = q_lo + ((qb * C::kQBuf) >> 4);
        const uint32_t tS = tS0 + (j & 1) * NP;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
          const uint32_t qo = ((kk >> 2) * C::kQBox + (kk & 3) * 32) >> 4;
          if (kk == 0)
            umma_ss_w<0>(tS, desc_words(kd + ko, d_hi), desc_words(qd + qo, d_hi), idesc_s);
          else
            umma_ss_w<1>(tS, desc_words(kd + ko, d_hi), desc_words(qd + qo, d_hi), idesc_s);
        }
        umma_commit_w(&s_ready[j & 1]);
        if (ETA_DECODE_PS_KV_SPLIT) umma_commit_w(&empty[st]);  // K tile read
        if (last) umma_commit_w(&q_free[qb]);  // Q buffer free once this product is done
        if (first && j + (cur.nt - cur.i) < n) {
          // Load the next piece's Q into the other buffer, which piece k - 1
          // used: wait until its last score product has read it.
          Cursor nx = cur;  // first tile of the next piece, tile j + nt - i (< n)
          for (int a = cur.i; a < cur.nt; ++a) nx.next(p);
          if (k >= 1 && !(ok = decode::warp_all_d(
                              wait_bar_spin(&q_free[qb ^ 1], ((k - 1) >> 1) & 1, ctl, kSiteQFree))))
            break;
          load_q(qb ^ 1, nx.segment(p));
        }
      }
      if (j >= 1) {
        // O^T (+)= V_{j-1}^T P^T(j-1); then stage (j-1) % 3 is free again.
        const int jp = j - 1;
        const int st = jp % kStages;
        if (!(ok = decode::warp_all_d(wait_bar_spin(&p_ready[jp & 1], (jp >> 1) & 1, ctl, kSiteP))))
          break;
        if (ETA_DECODE_PS_KV_SPLIT &&
            !(ok = decode::warp_all_d(
                  wait_bar_spin(&full_v[st], (jp / kStages) & 1, ctl, kSiteFull))))
          break;
        fence_proxy_async_smem();
        tc_fence_after();
        const uint32_t vd = v_lo + ((st * C::kStageBytes) >> 4);
        const uint32_t pd = p_lo + (((jp & 1) * C::kPBuf) >> 4);
#pragma unroll
        for (int kk = 0; kk < TK / 16; ++kk) {
          const uint32_t vo = kk * 128;  // 16 keys = 16 rows of 128 bytes
          const uint32_t po = ((kk >> 2) * C::kQBox + (kk & 3) * 32) >> 4;
          if (prev_first && kk == 0)
            umma_ss_w<0>(tO, desc_words(vd + vo, d_hi), desc_words(pd + po, d_hi), idesc_pv);
          else
            umma_ss_w<1>(tO, desc_words(vd + vo, d_hi), desc_words(pd + po, d_hi), idesc_pv);
        }
        umma_commit_w(ETA_DECODE_PS_KV_SPLIT ? &empty_v[st] : &empty[st]);
        umma_commit_w(&pv_done[jp & 1]);
      }
      if (j < n) {
        prev_first = (j == 0) || (cur.i == 0);
        if (j + 1 < n) cur.next(p);
      }
    }
    // Every MMA and every Q copy must be complete before the CTA exits (a
    // copy issued for a piece is waited for when the piece starts, except on
    // the abort path).
    umma_commit_w(drain);
    drain_bar(drain, 0, ctl, kSiteDrain);
    if (nq0 > 0) drain_bar(&q_full[0], (nq0 - 1) & 1, ctl, kSiteDrain);
    if (nq1 > 0) drain_bar(&q_full[1], (nq1 - 1) & 1, ctl, kSiteDrain);
  } else {
    // ------------------------------------------------------------ softmax and epilogue
    // Warp w owns the keys of quarter q4 = w % 4 (tensor-memory lanes 32 q4 ..
    // 32 q4 + 31) and heads hh GPT .. hh GPT + GPT - 1, hh = w / 4; each
    // thread holds its key's scores of those heads. The padded rows GP..NP-1
    // of both P^T buffers are zeroed once here and never written again, so
    // the products' padded columns stay zero.
    const int q4 = warp & 3;
    const int hh = warp >> 2;
    const int h0 = hh * GPT;                  // first head of this thread
    const int krow = q4 * 32 + lane;          // this thread's key in a tile (tensor-memory lane)
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const float sl2 = p.scale_log2;
    if constexpr (GP < NP) {
      for (int i = threadIdx.x; i < 2 * 2 * (NP - GP) * 8; i += 32 * R::kSoft) {
        const int chunk = i & 7, row = GP + ((i >> 3) % (NP - GP)), box = i / (8 * (NP - GP));
        *reinterpret_cast<uint4*>(sP + box * C::kQBox + row * 128 + chunk * 16) =
            make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
    }
    float m[GPT], l[GPT];
    bool ok = true;
    uint32_t xc = 0;        // uses of the x_bar / red exchange so far
    bool piece_whole = false;
    for (int j = 0; j < n; ++j) {
      const bool first = (j == 0) || (cur.i == 0);
      const bool last = (j == n - 1) || (cur.i == cur.nt - 1);
      if (first) {
        piece_whole = (cur.i == 0);
#pragma unroll
        for (int h = 0; h < GPT; ++h) {
          m[h] = -INFINITY;
          l[h] = 0.f;
        }
      }
      if (last) piece_whole = piece_whole && (cur.i == cur.nt - 1);
      if (!(ok = decode::warp_all_d(wait_bar_spin(&s_ready[j & 1], (j >> 1) & 1, ctl, kSiteS)))) break;
      tc_fence_after();
      uint32_t r[TW];
      tmem_ld_np<(TW)>(tS0 + lane_off + (j & 1) * NP + h0, r);
      const bool valid = cur.k0 + cur.i * TK + krow < cur.len;
      float s[GPT], wm[GPT];
#pragma unroll
      for (int h = 0; h < GPT; ++h) {
        s[h] = (valid && h0 + h < G) ? __uint_as_float(r[h]) * sl2 : -INFINITY;
        wm[h] = s[h];
      }
      float* rb = red + (xc & 1) * (kSoftWarps * NP);
      bool exch = true;  // exchange the tile maxima
      if (ETA_DECODE_PS_VOTE && !first) {
        // Vote: does any score of the tile lie more than the threshold above
        // its head's running maximum? If not, no maximum moves (alpha = 1).
        bool up = false;
#pragma unroll
        for (int h = 0; h < GPT; ++h) up = up || (s[h] > m[h] + kRescaleThreshold);
        up = __any_sync(0xffffffffu, up);
        if (lane == 0) reinterpret_cast<uint32_t*>(rb)[warp] = up ? 1u : 0u;
        mbar_arrive(&x_bar[xc & 1]);
        if (!(ok = decode::warp_all_d(wait_bar_spin(&x_bar[xc & 1], (xc >> 1) & 1, ctl, kSiteX))))
          break;
        ++xc;
        const uint4* f4 = reinterpret_cast<const uint4*>(rb);
        uint32_t any = 0;
#pragma unroll
        for (int v4 = 0; v4 < R::kSoft / 4; ++v4) {
          const uint4 f = f4[v4];
          any |= f.x | f.y | f.z | f.w;
        }
        exch = any != 0;
        rb = red + (xc & 1) * (kSoftWarps * NP);
      }
      float tm[GPT];
      if (exch) {
        // tile max per head: this warp's 32 keys by a reduce-scatter (lane l
        // ends with head h0 + l % GPT), then the four key quarters through
        // shared memory
        if constexpr (ETA_DECODE_PS_REDUX != 0) {
#pragma unroll
          for (int h = 0; h < GPT; ++h) wm[h] = warp_max_redux(wm[h]);
          if (lane == 0) {
            float4* dst = reinterpret_cast<float4*>(rb + q4 * NP + h0);
#pragma unroll
            for (int v4 = 0; v4 < GPT / 4; ++v4)
              dst[v4] = make_float4(wm[4 * v4], wm[4 * v4 + 1], wm[4 * v4 + 2], wm[4 * v4 + 3]);
          }
        } else {
          const float wmax = reduce_scatter<GPT>(wm, lane, MaxOp());
          if (lane < GPT) rb[q4 * NP + h0 + lane] = wmax;
        }
        mbar_arrive(&x_bar[xc & 1]);
        if (!(ok = decode::warp_all_d(wait_bar_spin(&x_bar[xc & 1], (xc >> 1) & 1, ctl, kSiteX))))
          break;
        ++xc;
        gather4<GPT, NP>(rb + h0, tm, MaxOp());
      } else {
#pragma unroll
        for (int h = 0; h < GPT; ++h) tm[h] = -INFINITY;
      }
      float alpha[GPT];
      bool rescale = false;
#pragma unroll
      for (int h = 0; h < GPT; ++h) {
        alpha[h] = 1.f;
        if (tm[h] > m[h] + kRescaleThreshold) {
          alpha[h] = ex2_approx(m[h] - tm[h]);  // m = -inf gives 0
          m[h] = tm[h];
          l[h] *= alpha[h];
          rescale = true;
        }
      }
      if (rescale && !first && q4 * 32 < D) {
        // O^T was last written by PV(j-1) of this piece; wait for it, then
        // scale this warp's 32 dims of its heads by their alpha (lanes D..127
        // of a D = 64 product hold zeros).
        if (!(ok = decode::warp_all_d(
                  wait_bar_spin(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, ctl, kSitePv))))
          break;
        tc_fence_after();
        uint32_t o[TW];
        tmem_ld_np<(TW)>(tO + lane_off + h0, o);
#pragma unroll
        for (int h = 0; h < GPT; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
        tmem_st_np<(TW)>(tO + lane_off + h0, o);
        tmem_wait_st();
      }
      // P^T(j): row h, key krow, in buffer j % 2 (read by PV(j - 2), which
      // completed before S(j) was signalled).
      uint8_t* pb = sP + (j & 1) * C::kPBuf + (krow >> 6) * C::kQBox;
      const int kc = krow & 63;
#pragma unroll
      for (int h = 0; h < GPT; ++h) {
        float pv = 0.f;
        if (h0 + h < G) {
          pv = ex2_approx(s[h] - (m[h] == -INFINITY ? 0.f : m[h]));
          l[h] += pv;
        }
        const int hr = h0 + h;
        *reinterpret_cast<uint16_t*>(pb + hr * 128 + ((((kc >> 3) ^ (hr & 7))) << 4) +
                                     ((kc & 7) << 1)) = to_bits<T>(pv);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_ready[j & 1]);

      if (last) {
        // ---- end of a piece: row sums over the tile's 128 key slots, then O.
        float lt[GPT];
#pragma unroll
        for (int h = 0; h < GPT; ++h) lt[h] = l[h];
        const float wsum = reduce_scatter<GPT>(lt, lane, AddOp());
        float* rl = red + (xc & 1) * (kSoftWarps * NP);
        if (lane < GPT) rl[q4 * NP + h0 + lane] = wsum;
        mbar_arrive(&x_bar[xc & 1]);
        if (!(ok = decode::warp_all_d(wait_bar_spin(&x_bar[xc & 1], (xc >> 1) & 1, ctl, kSiteX)))) break;
        ++xc;
        float tot[GPT];
        gather4<GPT, NP>(rl + h0, tot, AddOp());
        if (!(ok = decode::warp_all_d(wait_bar_spin(&pv_done[j & 1], (j >> 1) & 1, ctl, kSitePv))))
          break;
        tc_fence_after();
        uint32_t o[TW];
        tmem_ld_np<(TW)>(tO + lane_off + h0, o);
        const int dim = krow;  // O^T lane = output dimension
        const int seg = cur.segment(p);
        const size_t row0 = static_cast<size_t>(cur.b) * p.Hq + static_cast<size_t>(cur.g) * G;
#pragma unroll
        for (int h = 0; h < GPT; ++h) {
          const int hg = h0 + h;
          if (hg < G && dim < D) {
            const float ov = tot[h] > 0.f ? __uint_as_float(o[h]) / tot[h] : 0.f;
            const float l2 = tot[h] > 0.f ? m[h] + lg2_approx(tot[h]) : -INFINITY;
            if (piece_whole) {
              // The whole segment lay in this CTA: this is the result.
              reinterpret_cast<uint16_t*>(p.o)[(row0 + hg) * D + dim] = to_bits<T>(ov);
              if (dim == hg && p.lse != nullptr) p.lse[row0 + hg] = l2 * 0.69314718055994531f;
            } else {
              const size_t slot = static_cast<size_t>(seg) + c;
              p.part_o[(slot * G + hg) * D + dim] = ov;
              if (dim == hg) p.part_lse[slot * G + hg] = l2;
            }
          }
        }
        // O^T is overwritten by the next piece's first product only after
        // that piece's first p_ready, which follows this read.
        tc_fence_before();
      }
      if (j + 1 < n) cur.next(p);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == R::kMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ gather
// One warp per (sequence b, query head h): a segment cut between CTAs (in the
// equal-tile-range mode) has one partial per CTA, in slots segment + cta;
// merge them by their log-sum-exp. Segments that lay in one CTA were written
// by it, and empty sequences by the plan kernel; both are skipped.
template <int D, typename T>
__global__ void __launch_bounds__(128) attn_decode_gather_kernel(const PParams p, int nc) {
  constexpr int EPL = D / 32;  // output elements per lane
  griddep_wait();  // the stream kernel's partials and outputs are visible after this
  const long long row = static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<long long>(p.B) * p.Hq) return;
  const int b = static_cast<int>(div_nonneg(row, p.Hq));
  const int h = static_cast<int>(row - static_cast<long long>(b) * p.Hq);
  const int g = h / p.G;
  const int hh = h - g * p.G;
  // tile_off holds cost positions (tile offsets when wcost = 0): a non-empty
  // sequence spans Hkv (nt + wcost) of them, and tile i of its segment g sits
  // at tile_off[b] + g (nt + wcost) + wcost + i.
  const int w = p.wcost;
  const int span = p.tile_off[b + 1] - p.tile_off[b];
  if (span == 0 || p.seg_aligned) return;
  const int nt = span / p.Hkv - w;
  const long long T_all = p.tile_off[p.B];  // all cost positions
  const long long a = p.tile_off[b] + static_cast<long long>(g) * (nt + w) + w;
  const int c0 = cta_of(a, T_all, nc);
  const int c1 = cta_of(a + nt - 1, T_all, nc);
  if (c0 == c1) return;
  const long long seg = static_cast<long long>(b) * p.Hkv + g;
  // CTAs between c0 and c1 with an empty tile range (possible only with
  // fewer tiles than CTAs) wrote nothing: their slots are skipped. The
  // partials of the first kMaxP CTAs are all loaded before any is used, so
  // their loads overlap; a running maximum then folds them (and, for longer
  // cuts, the rest) in.
  const bool all_have = T_all >= nc;
  auto has_tiles = [&](int cc) {
    return all_have || div_nonneg(cc * T_all, nc) < div_nonneg((cc + 1) * T_all, nc);
  };
  constexpr int kMaxP = 6;
  float lse_r[kMaxP], xv[kMaxP][EPL];
#pragma unroll
  for (int k = 0; k < kMaxP; ++k) {
    const int cc = c0 + k;
    lse_r[k] = -INFINITY;
    if (cc <= c1 && has_tiles(cc)) {
      const long long slot = (seg + cc) * p.G + hh;
      lse_r[k] = p.part_lse[slot];
      const float* x = p.part_o + slot * D + lane * EPL;
      if constexpr (EPL == 4) {
        const float4 v = *reinterpret_cast<const float4*>(x);
        xv[k][0] = v.x, xv[k][1] = v.y, xv[k][2] = v.z, xv[k][3] = v.w;
      } else {
        const float2 v = *reinterpret_cast<const float2*>(x);
        xv[k][0] = v.x, xv[k][1] = v.y;
      }
    } else {
#pragma unroll
      for (int e = 0; e < EPL; ++e) xv[k][e] = 0.f;
    }
  }
  float mx = -INFINITY, tot = 0.f;
  float acc[EPL] = {};
  auto fold = [&](float lse, const float (&x)[EPL]) {
    if (lse == -INFINITY) return;
    const float nm = fmaxf(mx, lse);
    const float sc = ex2_approx(mx - nm);  // mx = -inf gives 0
    const float wt = ex2_approx(lse - nm);
    tot = tot * sc + wt;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = fmaf(wt, x[e], acc[e] * sc);
    mx = nm;
  };
#pragma unroll
  for (int k = 0; k < kMaxP; ++k) fold(lse_r[k], xv[k]);
  for (int cc = c0 + kMaxP; cc <= c1; ++cc) {
    if (!has_tiles(cc)) continue;
    const long long slot = (seg + cc) * p.G + hh;
    const float* x = p.part_o + slot * D + lane * EPL;
    float xr[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) xr[e] = x[e];
    fold(p.part_lse[slot], xr);
  }
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  uint32_t pk[EPL / 2];
#pragma unroll
  for (int e = 0; e < EPL / 2; ++e) pk[e] = decode::pack2<T>(acc[2 * e] * inv, acc[2 * e + 1] * inv);
  T* dst = reinterpret_cast<T*>(p.o) + row * D + lane * EPL;
  if constexpr (EPL == 4)
    *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
  else
    *reinterpret_cast<uint32_t*>(dst) = pk[0];
  if (lane == 0 && p.lse != nullptr)
    p.lse[row] = tot > 0.f ? (mx + lg2_approx(tot)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace decode_ps
}  // namespace eta
