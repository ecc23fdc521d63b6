// Exact attention for head sizes the tensor-core prefill kernel does not take
// (any d that is a multiple of 8, from 8 to 256), on CUDA cores in fp32.
//
// Same operation, masks and conventions as the tiled prefill kernel:
// softmax(scale * Q K^T + mask) V with the running-softmax recurrence of the
// aikaboom page "11.4d FlashAttention" ("Online Softmax") over key tiles
// staged in shared memory ("Tiling"); causal masking bottom-right aligned, an
// optional sliding window of the W most recent keys, GQA head map
// h / (Hq / Hkv), and LSE = ln(sum exp(scale * q . k)).
//
// Decode mode (seqlens != NULL): one query row per (batch, query head) over the
// packed ragged cache of attn_decode (sequence b at token offset
// sum_{j<b} L_j, laid out [Hkv][L_b][d]; the offsets from one prefix sum per
// call when given, else summed per CTA); it is the causal case with Nq = 1 and
// Nk = L_b, so a window keeps the last W cached tokens.
//
// Layout of the work: a CTA of 4 warps owns 16 query rows of one (batch, query
// head), 4 rows per warp. Per 32-key tile the whole CTA stages K and V in
// shared memory (rows padded by 16 bytes, so 32 lanes reading 32 different
// rows with 16-byte loads hit distinct banks); then for each of its rows a
// warp computes the 32 scores (lane j: key j, fp32 dot product over d), the
// running max and sum with warp shuffles, and O += P V with lane c owning the
// 8 output columns 8c..8c+7 and p_j broadcast by shuffle.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>

namespace eta {
namespace generic {

constexpr int kRowsPerWarp = 4;
constexpr int kWarps = 4;
constexpr int kRows = kRowsPerWarp * kWarps;  // query rows per CTA
constexpr int kTK = 32;                       // keys per tile
constexpr int kThreads = 32 * kWarps;
constexpr int kMaxD = 256;
constexpr int kGridY = 65535;  // (batch, head) pairs per grid z slice

struct GParams {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  int BH;  // B * Hq
  int Hq;
  int Hkv;
  int Nq;
  int Nk;
  int d;
  int group;  // Hq / Hkv
  int off;    // Nk - Nq
  int causal;
  int window;  // causal only; 0 = no window
  float scale_log2;
  const int* seqlens;  // decode mode when not NULL (Nq = 1, Nk = L_b, causal)
  const long long* tok_off;  // decode: [B] token offsets, or NULL: summed per CTA
};

// Shared-memory row stride in bytes for d 16-bit elements (+16 bytes of pad).
__host__ __device__ constexpr int row_stride(int d) { return d * 2 + 16; }
__host__ __device__ constexpr int smem_bytes(int d) {
  return 2 * kTK * row_stride(d) + kRows * d * 2;
}

template <typename T>
__device__ __forceinline__ void to_f32x8(const uint4& v, float (&f)[8]);
template <>
__device__ __forceinline__ void to_f32x8<__nv_bfloat16>(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
template <>
__device__ __forceinline__ void to_f32x8<__half>(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    f[2 * i] = x.x;
    f[2 * i + 1] = x.y;
  }
}

template <typename T>
__device__ __forceinline__ uint32_t pack_pair(float a, float b);
template <>
__device__ __forceinline__ uint32_t pack_pair<__nv_bfloat16>(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
template <>
__device__ __forceinline__ uint32_t pack_pair<__half>(float a, float b) {
  __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Keys a query row sees: [lo, hi] (inclusive), clipped to [0, Nk - 1];
// empty when lo > hi.
__device__ __forceinline__ void visible_range(const GParams& p, int row, int& lo, int& hi) {
  lo = 0;
  hi = p.Nk - 1;
  if (p.causal) {
    hi = min(hi, row + p.off);
    if (p.window > 0) lo = max(0, row + p.off - p.window + 1);
  }
}

// OUT_F32: O is written as fp32 (not rounded), for partial results merged further.
template <typename T, bool OUT_F32 = false>
__global__ void __launch_bounds__(kThreads) attn_generic_kernel(const GParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int d = p.d;
  const int stride = row_stride(d);
  uint8_t* sK = smem;
  uint8_t* sV = smem + kTK * stride;
  T* sQ = reinterpret_cast<T*>(smem + 2 * kTK * stride);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.z * kGridY + blockIdx.y;
  if (bh >= p.BH) return;  // tail of the last z slice (block-uniform)
  const int b = bh / p.Hq;
  const int h = bh - b * p.Hq;
  const int kvh = h / p.group;
  const int r0 = blockIdx.x * kRows;
  const int nchunk = d / 8;  // 16-byte chunks per row

  GParams pp = p;  // per-CTA view: decode mode sets this sequence's length
  size_t kv_off = (static_cast<size_t>(b) * p.Hkv + kvh) * static_cast<size_t>(p.Nk) * d;
  if (p.seqlens != nullptr) {
    __shared__ long long s_tok;
    __shared__ int s_len;
    if (warp == 0) {
      long long acc = 0;
      if (p.tok_off == nullptr)
        for (int j = lane; j < b; j += 32) acc += max(p.seqlens[j], 0);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) {
        s_tok = p.tok_off != nullptr ? p.tok_off[b] : acc;
        s_len = max(p.seqlens[b], 0);
      }
    }
    __syncthreads();
    pp.Nk = s_len;
    pp.off = s_len - 1;  // Nq = 1
    kv_off = (static_cast<size_t>(s_tok) * p.Hkv + static_cast<size_t>(kvh) * s_len) * d;
  }
  const T* qg = reinterpret_cast<const T*>(p.q) + (static_cast<size_t>(bh) * p.Nq) * d;
  const T* kg = reinterpret_cast<const T*>(p.k) + kv_off;
  const T* vg = reinterpret_cast<const T*>(p.v) + kv_off;

  // Q rows of this CTA (rows past Nq are zero).
  for (int i = threadIdx.x; i < kRows * nchunk; i += kThreads) {
    const int rr = i / nchunk, c = i - rr * nchunk;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r0 + rr < p.Nq)
      v = *reinterpret_cast<const uint4*>(qg + static_cast<size_t>(r0 + rr) * d + c * 8);
    *reinterpret_cast<uint4*>(sQ + rr * d + c * 8) = v;
  }

  // Key range any row of the CTA sees.
  int klo = pp.Nk, khi = -1;
  for (int rr = 0; rr < kRows; ++rr) {
    const int row = r0 + rr;
    if (row >= p.Nq) break;
    int lo, hi;
    visible_range(pp, row, lo, hi);
    if (lo <= hi) {
      klo = min(klo, lo);
      khi = max(khi, hi);
    }
  }

  float m[kRowsPerWarp], l[kRowsPerWarp], o[kRowsPerWarp][8];
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[i][e] = 0.f;
  }

  const int t_first = klo <= khi ? klo / kTK : 0;
  const int t_last = klo <= khi ? khi / kTK : -1;
  for (int t = t_first; t <= t_last; ++t) {
    const int kv0 = t * kTK;
    __syncthreads();  // the previous tile is no longer read
    for (int i = threadIdx.x; i < kTK * nchunk; i += kThreads) {
      const int j = i / nchunk, c = i - j * nchunk;
      uint4 kv = make_uint4(0u, 0u, 0u, 0u), vv = kv;
      if (kv0 + j < pp.Nk) {
        kv = *reinterpret_cast<const uint4*>(kg + static_cast<size_t>(kv0 + j) * d + c * 8);
        vv = *reinterpret_cast<const uint4*>(vg + static_cast<size_t>(kv0 + j) * d + c * 8);
      }
      *reinterpret_cast<uint4*>(sK + j * stride + c * 16) = kv;
      *reinterpret_cast<uint4*>(sV + j * stride + c * 16) = vv;
    }
    __syncthreads();

#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
      const int rr = warp * kRowsPerWarp + i;
      const int row = r0 + rr;
      if (row >= p.Nq) continue;  // warp-uniform
      int lo, hi;
      visible_range(pp, row, lo, hi);
      // score of key kv0 + lane
      float s = 0.f;
      const T* qrow = sQ + rr * d;
      for (int c = 0; c < nchunk; ++c) {
        float qf[8], kf[8];
        to_f32x8<T>(*reinterpret_cast<const uint4*>(qrow + c * 8), qf);
        to_f32x8<T>(*reinterpret_cast<const uint4*>(sK + lane * stride + c * 16), kf);
#pragma unroll
        for (int e = 0; e < 8; ++e) s = fmaf(qf[e], kf[e], s);
      }
      const int key = kv0 + lane;
      const bool vis = key >= lo && key <= hi;
      s = vis ? s * p.scale_log2 : -INFINITY;
      const float m_new = fmaxf(m[i], warp_max(s));
      if (m_new == -INFINITY) continue;  // no visible key for this row yet
      const float alpha = exp2f(m[i] - m_new);  // m = -inf gives 0
      const float pj = exp2f(s - m_new);
      l[i] = l[i] * alpha + warp_sum(pj);
      m[i] = m_new;
#pragma unroll
      for (int e = 0; e < 8; ++e) o[i][e] *= alpha;
      for (int j = 0; j < kTK; ++j) {
        const float pb = __shfl_sync(0xffffffffu, pj, j);  // every lane takes part
        if (lane < nchunk) {
          float vf[8];
          to_f32x8<T>(*reinterpret_cast<const uint4*>(sV + j * stride + lane * 16), vf);
#pragma unroll
          for (int e = 0; e < 8; ++e) o[i][e] = fmaf(pb, vf[e], o[i][e]);
        }
      }
    }
  }

  // Epilogue: O / l rounded to T, LSE in natural-log units.
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    const int row = r0 + warp * kRowsPerWarp + i;
    if (row >= p.Nq) continue;
    const float inv = l[i] > 0.f ? 1.f / l[i] : 0.f;
    if (OUT_F32 && lane < nchunk) {
      float* dst = reinterpret_cast<float*>(p.o) + (static_cast<size_t>(bh) * p.Nq + row) * d +
                   lane * 8;
      *reinterpret_cast<float4*>(dst) =
          make_float4(o[i][0] * inv, o[i][1] * inv, o[i][2] * inv, o[i][3] * inv);
      *reinterpret_cast<float4*>(dst + 4) =
          make_float4(o[i][4] * inv, o[i][5] * inv, o[i][6] * inv, o[i][7] * inv);
    } else if (lane < nchunk) {
      uint4 w;
      w.x = pack_pair<T>(o[i][0] * inv, o[i][1] * inv);
      w.y = pack_pair<T>(o[i][2] * inv, o[i][3] * inv);
      w.z = pack_pair<T>(o[i][4] * inv, o[i][5] * inv);
      w.w = pack_pair<T>(o[i][6] * inv, o[i][7] * inv);
      *reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.o) +
                                (static_cast<size_t>(bh) * p.Nq + row) * d + lane * 8) = w;
    }
    if (lane == 0 && p.lse != nullptr)
      p.lse[static_cast<size_t>(bh) * p.Nq + row] =
          l[i] > 0.f ? (m[i] + log2f(l[i])) * 0.69314718055994531f : -INFINITY;
  }
}

}  // namespace generic
}  // namespace eta
