// Log-sum-exp merge of partial attention results (context-parallel prefill).
//
// A query row's attention over a key set K = K_1 u K_2 (disjoint) follows
// from the two partial results over K_1 and K_2: with LSE_i the log-sum-exp of
// the row's scores over K_i and O_i the softmax-weighted value sum over K_i,
//     LSE = ln(e^LSE_1 + e^LSE_2),   O = e^(LSE_1 - LSE) O_1 + e^(LSE_2 - LSE) O_2.
// This is the running-statistics rescale of the aikaboom page "11.4d
// FlashAttention" ("Online Softmax") applied to whole key blocks; the decode
// split combine is the same identity over many splits.
//
// attn_merge_kernel folds one partial (O_part in the input dtype or fp32,
// LSE_part fp32) into an fp32 accumulator (o_acc, lse_acc) in place and optionally
// writes the merged O rounded to the input dtype. A row whose accumulator LSE
// is -inf is empty: its o_acc is not read. Each row is owned by the lanes of
// one warp (8 columns per lane), so the row's LSE is read by all of them
// before one lane overwrites it.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>
#include <cstdint>

namespace eta {
namespace merge {

constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&f)[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&f)[8]) {
  const uint4 v = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
template <>
__device__ __forceinline__ void load8<__half>(const __half* p, float (&f)[8]) {
  const uint4 v = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    f[2 * i] = x.x;
    f[2 * i + 1] = x.y;
  }
}

template <typename T>
__device__ __forceinline__ uint32_t pack2(float a, float b);
template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
template <>
__device__ __forceinline__ uint32_t pack2<__half>(float a, float b) {
  __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&f)[8]) {
  const float4 x = *reinterpret_cast<const float4*>(p);
  const float4 y = *reinterpret_cast<const float4*>(p + 4);
  f[0] = x.x; f[1] = x.y; f[2] = x.z; f[3] = x.w;
  f[4] = y.x; f[5] = y.y; f[6] = y.z; f[7] = y.w;
}

// T: type of the rounded output o_out; TP: type of the partial O (T, or fp32
// for unrounded partials).
template <typename T, typename TP = T>
__global__ void __launch_bounds__(kThreads)
    attn_merge_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc,
                      const TP* __restrict__ o_part, const float* __restrict__ lse_part,
                      T* __restrict__ o_out, long long rows, int d) {
  const int cpr = d >> 3;          // 8-column chunks per row (1..32)
  const int rpw = 32 / cpr;        // rows per warp pass
  const int lane = threadIdx.x & 31;
  const int sub = lane / cpr;      // which of the warp's rows this lane serves
  const int c = lane - sub * cpr;  // chunk within the row
  const bool active = sub < rpw;
  const long long warps = static_cast<long long>(gridDim.x) * (kThreads / 32);
  const long long w0 = static_cast<long long>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
  for (long long base = w0 * rpw; base < rows; base += warps * rpw) {
    const long long r = base + sub;
    const bool live = active && r < rows;
    float la = -INFINITY, lp = -INFINITY;
    if (live) {
      la = lse_acc[r];
      lp = lse_part[r];
    }
    const float mx = fmaxf(la, lp);
    float ln = -INFINITY, wa = 0.f, wp = 0.f;
    if (mx != -INFINITY) {
      wa = la == -INFINITY ? 0.f : expf(la - mx);
      wp = lp == -INFINITY ? 0.f : expf(lp - mx);
      const float s = wa + wp;
      ln = mx + logf(s);
      wa /= s;
      wp /= s;
    }
    if (live) {
      float a[8], pf[8];
      float* acc = o_acc + r * d + c * 8;
      if (wa != 0.f) {
        const float4 x = *reinterpret_cast<const float4*>(acc);
        const float4 y = *reinterpret_cast<const float4*>(acc + 4);
        a[0] = x.x; a[1] = x.y; a[2] = x.z; a[3] = x.w;
        a[4] = y.x; a[5] = y.y; a[6] = y.z; a[7] = y.w;
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) a[e] = 0.f;
      }
      if (wp != 0.f) {
        load8<TP>(o_part + r * d + c * 8, pf);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) pf[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) a[e] = wa * a[e] + wp * pf[e];
      *reinterpret_cast<float4*>(acc) = make_float4(a[0], a[1], a[2], a[3]);
      *reinterpret_cast<float4*>(acc + 4) = make_float4(a[4], a[5], a[6], a[7]);
      if (o_out != nullptr) {
        uint4 w;
        w.x = pack2<T>(a[0], a[1]);
        w.y = pack2<T>(a[2], a[3]);
        w.z = pack2<T>(a[4], a[5]);
        w.w = pack2<T>(a[6], a[7]);
        *reinterpret_cast<uint4*>(o_out + r * d + c * 8) = w;
      }
    }
    __syncwarp();  // every lane of the row has read lse_acc[r]
    if (live && c == 0) lse_acc[r] = ln;
  }
}

}  // namespace merge
}  // namespace eta
