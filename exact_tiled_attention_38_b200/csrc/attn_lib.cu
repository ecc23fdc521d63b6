// C-ABI boundary of the attention library: argument checks, TMA descriptor
// encoding, kernel selection, launch configuration and error codes. Every
// step of the computation runs in the kernels:
//   prefill_sm100.cuh    prefill, d = 64 / 128 (tcgen05, TMA)
//   decode_sm100.cuh     decode split pass on CUDA cores (d = 64; d = 128
//                        with one query head per KV head), the LSE combine
//                        and the token-offset scan of large batches
//   decode_ps_sm100.cuh  decode as one persistent streaming pass on tcgen05
//                        (d = 128, groups 2..32): plan, stream, gather
//   generic_fwd.cuh      prefill and decode for the other head sizes
//   merge.cuh            LSE merge of partial results (context parallelism)
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <type_traits>

#include "../../include/attn.h"
#include "decode_ps_sm100.cuh"
#include "decode_sm100.cuh"
#include "generic_fwd.cuh"
#include "merge.cuh"
#include "prefill_sm100.cuh"

namespace eta {
namespace api {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(ptr);
  }();
  return fn;
}

// The CUDA error behind the calling thread's most recent ATTN_ERR_CUDA.
thread_local int g_last_cuda_error = 0;

inline int cuda_fail(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  return ATTN_ERR_CUDA;
}

// Status of the launch just made on this thread.
inline int launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ATTN_OK : cuda_fail(e);
}

// A setup step (a kernel attribute) done once per device and remembered: the
// attribute applies to the current device only, so a process that drives
// several GPUs needs it on each.
struct PerDeviceOnce {
  std::mutex mu;
  bool done[64] = {};
  cudaError_t err[64] = {};
  template <typename F>
  cudaError_t run(F&& step) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!done[dev]) {
      err[dev] = step();
      done[dev] = true;
    }
    return err[dev];
  }
};

struct DeviceInfo {
  int sm_count = 0;
  long long l2_bytes = 0;
  bool sm100 = false;
};

// Per-device properties, queried once per device.
int device_info(DeviceInfo* out) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  static bool have[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!have[dev]) {
    int major = 0, minor = 0, sms = 0, l2 = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    cache[dev].sm_count = sms;
    cache[dev].l2_bytes = l2;
    cache[dev].sm100 = (major == 10 && minor == 0);
    have[dev] = true;
  }
  *out = cache[dev];
  return ATTN_OK;
}

// Stream-ordered workspace for attn_decode: a memory pool owned by the library
// (one per device). Freed blocks stay cached up to kPoolKeepBytes, so a caller
// that synchronises between calls does not pay for unmapping and re-mapping
// device memory on every call (the device's default pool releases its free
// memory at synchronisation points). The caller's own pools are untouched.
constexpr uint64_t kPoolKeepBytes = 256ull << 20;

int workspace_pool(cudaMemPool_t* out) {
  static std::mutex mu;
  static cudaMemPool_t pools[64];
  static bool have[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!have[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    if (cudaMemPoolCreate(&pools[dev], &props) != cudaSuccess) return ATTN_ERR_CUDA;
    uint64_t keep = kPoolKeepBytes;
    if (cudaMemPoolSetAttribute(pools[dev], cudaMemPoolAttrReleaseThreshold, &keep) !=
        cudaSuccess)
      return ATTN_ERR_CUDA;
    have[dev] = true;
  }
  *out = pools[dev];
  return ATTN_OK;
}

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

inline bool scale_ok(float s) { return std::isfinite(s) && s > 0.f; }

// Head sizes: 64 and 128 run on the tensor-core kernels; any other multiple of
// 8 from 8 to 256 runs on the CUDA-core generic kernel.
inline bool tensor_core_d(int d) { return d == 64 || d == 128; }
inline bool generic_d(int d) { return d >= 8 && d <= generic::kMaxD && d % 8 == 0; }

template <typename T, bool OUT_F32 = false>
int launch_generic(generic::GParams p, int BH, int Nq, cudaStream_t st) {
  p.BH = BH;
  const int ny = BH < generic::kGridY ? BH : generic::kGridY;
  const dim3 grid((Nq + generic::kRows - 1) / generic::kRows, ny,
                  (BH + generic::kGridY - 1) / generic::kGridY);
  generic::attn_generic_kernel<T, OUT_F32>
      <<<grid, generic::kThreads, generic::smem_bytes(p.d), st>>>(p);
  return launch_status();
}

// 3-D map over a [Z][rows][D] tensor of 16-bit elements, box 64 x box_rows x 1,
// 128-byte swizzle, zero fill outside the tensor (loads) / clipping (stores).
int encode_3d(CUtensorMap* map, const void* base, bool bf16, int D, long long rows, long long Z,
              unsigned box_rows = 128) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return ATTN_ERR_CUDA;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(Z)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                                 static_cast<cuuint64_t>(rows) * D * 2};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// 3-D map over a [Z][rows][D] fp32 tensor, box 32 x 32 x 1 (128-byte rows),
// 128-byte swizzle; used for stores of unrounded partial outputs.
int encode_3d_f32(CUtensorMap* map, const void* base, int D, long long rows, long long Z) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return ATTN_ERR_CUDA;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(Z)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 4,
                                 static_cast<cuuint64_t>(rows) * D * 4};
  const cuuint32_t box[3] = {32, 32, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// O = 0, LSE = -inf for `rows` rows (every row has an empty key set).
template <typename T>
__global__ void fill_empty_kernel(T* o, float* lse, long long rows, int D) {
  const long long n = rows * D;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    o[i] = T(0.f);
    if (lse != nullptr && i % D == 0) lse[i / D] = -INFINITY;
  }
}

template <typename T>
int launch_fill_empty(void* o, float* lse, long long rows, int D, cudaStream_t st) {
  const long long n = rows * D;
  const int threads = 256;
  const long long want = (n + threads - 1) / threads;
  const int blocks = static_cast<int>(want < 4096 ? (want > 0 ? want : 1) : 4096);
  fill_empty_kernel<T><<<blocks, threads, 0, st>>>(reinterpret_cast<T*>(o), lse, rows, D);
  return launch_status();
}

// Prefill kernel knob: POLY8 of every 8 score columns take 2^x from the FMA
// polynomial instead of the special-function unit.
#ifndef ETA_PREFILL_POLY8
#define ETA_PREFILL_POLY8 0
#endif
// The same for d = 64, whose exponential phase keeps the special-function
// unit busy while both softmax groups of a CTA run it. Measured on B200
// (causal 2K / non-causal 4K, d = 64): 0.0665-0.0676 / 0.373 ms without,
// 0.0717 / 0.399 ms with 2, 0.0737 / 0.408 ms with 4, 0.0814 / 0.469 ms with 6.
#ifndef ETA_PREFILL_POLY8_D64
#define ETA_PREFILL_POLY8_D64 0
#endif

// Prefill kernel knob: L2 prefetch of the next item's query tiles, issued by
// the producer right after the current item's own query loads. Measured
// slower on B200 on the 2K causal MHA workload, whether issued before or after
// those loads (0.0840 ms against 0.0819 ms without, in interleaved runs on one
// box; 32K causal GQA within noise), so it is off.
#ifndef ETA_PREFILL_PREFETCH_Q
#define ETA_PREFILL_PREFETCH_Q 0
#endif

// Prefill kernel knob: softmax threads per query row for d = 128 (1 or 2).
// Two threads per row (576-thread CTAs, 96 registers: five warps share an SM
// sub-partition's register file) pass the same parity tests but measured about
// 10 % slower on B200 (2K causal MHA 0.094 ms against 0.084 ms, 32K causal GQA
// 7.60 ms against 6.86 ms): a row's two warps sit on the same sub-partition,
// whose special-function unit bounds the exponentials either way, and the
// row-max exchange and register spills add to every step.
#ifndef ETA_PREFILL_SPLIT
#define ETA_PREFILL_SPLIT 1
#endif

// The two softmax groups of a d = 64 CTA take turns for their exponentials
// (1), so that one group's exponentials overlap the other's score loads, row
// maxima and stores instead of both contending for the special-function unit
// at once; or run freely (0). Measured on B200: 0.0717 ms against 0.0676 ms
// (causal 2K) and 0.397 against 0.371 ms (non-causal 4K) with turns.
#ifndef ETA_PREFILL_PINGPONG64
#define ETA_PREFILL_PINGPONG64 0
#endif

template <int D, typename T, bool CAUSAL, bool WINDOW = false, bool OUT_F32 = false>
int launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                   const CUtensorMap& to, const prefill::Params& p, int grid, cudaStream_t st) {
  constexpr int SPLIT = D == 128 ? ETA_PREFILL_SPLIT : 1;
  constexpr bool PINGPONG = D == 64 && ETA_PREFILL_PINGPONG64;
  constexpr int POLY8 = D == 64 ? ETA_PREFILL_POLY8_D64 : ETA_PREFILL_POLY8;
  auto kern = prefill::attn_prefill_kernel<D, T, CAUSAL, WINDOW, POLY8, PINGPONG, SPLIT,
                                           ETA_PREFILL_PREFETCH_Q != 0, OUT_F32>;
  constexpr int smem = prefill::Cfg<D>::kSmemBytes;
  static PerDeviceOnce attr;
  const cudaError_t attr_err = attr.run([&]() {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (attr_err != cudaSuccess) return cuda_fail(attr_err);
  kern<<<grid, prefill::kernel_threads(SPLIT), smem, st>>>(tq, tk, tv, to, p);
  return launch_status();
}

// Prefill knob: KV-head-major order of causal items when K/V exceed L2 (1) or
// always all heads of a query level together (0).
#ifndef ETA_PREFILL_HEAD_MAJOR
#define ETA_PREFILL_HEAD_MAJOR 1
#endif

// OUT_F32: o is float32 (the unrounded O of a partial result), else T.
template <typename T, bool OUT_F32 = false>
int fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
        int Nq, int Nk, int d, float scale, int causal, cudaStream_t st, uint64_t wait_ns,
        int debug_flags, int window = 0) {
  if (B < 0 || Nq < 0 || Nk < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || !scale_ok(scale))
    return ATTN_ERR_INVALID;
  if (window < 0 || (window > 0 && !causal)) return ATTN_ERR_INVALID;
  if (!tensor_core_d(d) && (!generic_d(d) || debug_flags != 0)) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(Nq) > 65535LL * prefill::NQT * prefill::BM) return ATTN_ERR_INVALID;
  if (static_cast<long long>(B) * Hq > 0x7fffffffLL) return ATTN_ERR_INVALID;
  if (B == 0 || Nq == 0) return ATTN_OK;
  if (o == nullptr || !aligned(o, 16) || (lse != nullptr && !aligned(lse, 4)))
    return ATTN_ERR_INVALID;
  if (Nk > 0 && (q == nullptr || k == nullptr || v == nullptr || !aligned(q, 16) ||
                 !aligned(k, 16) || !aligned(v, 16)))
    return ATTN_ERR_INVALID;
  DeviceInfo info;
  if (device_info(&info) != ATTN_OK) return ATTN_ERR_CUDA;
  if (!info.sm100) return ATTN_ERR_UNSUPPORTED;
  if (Nk == 0) {
    using TO = typename std::conditional<OUT_F32, float, T>::type;
    return launch_fill_empty<TO>(o, lse, static_cast<long long>(B) * Hq * Nq, d, st);
  }
  if (!tensor_core_d(d)) {
    generic::GParams g;
    g.q = q;
    g.k = k;
    g.v = v;
    g.o = o;
    g.lse = lse;
    g.Hq = Hq;
    g.Hkv = Hkv;
    g.Nq = Nq;
    g.Nk = Nk;
    g.d = d;
    g.group = Hq / Hkv;
    g.off = Nk - Nq;
    g.causal = causal ? 1 : 0;
    g.window = window;
    g.scale_log2 = scale * 1.4426950408889634f;
    g.seqlens = nullptr;
    g.tok_off = nullptr;
    return launch_generic<T, OUT_F32>(g, B * Hq, Nq, st);
  }

  constexpr bool bf16 = std::is_same<T, __nv_bfloat16>::value;
  CUtensorMap tq, tk, tv, to;
  int rc = encode_3d(&tq, q, bf16, d, Nq, static_cast<long long>(B) * Hq);
  if (rc == ATTN_OK)
    rc = OUT_F32 ? encode_3d_f32(&to, o, d, Nq, static_cast<long long>(B) * Hq)
                 : encode_3d(&to, o, bf16, d, Nq, static_cast<long long>(B) * Hq, 32);
  if (rc == ATTN_OK) rc = encode_3d(&tk, k, bf16, d, Nk, static_cast<long long>(B) * Hkv);
  if (rc == ATTN_OK) rc = encode_3d(&tv, v, bf16, d, Nk, static_cast<long long>(B) * Hkv);
  if (rc != ATTN_OK) return rc;

  prefill::Params p;
  p.o = o;
  p.lse = lse;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.group = Hq / Hkv;
  p.n_pairs = (Nq + prefill::NQT * prefill::BM - 1) / (prefill::NQT * prefill::BM);
  p.off = Nk - Nq;
  p.BH = B * Hq;
  const long long total = static_cast<long long>(p.BH) * p.n_pairs;
  if (total > 0x7fffffffLL) return ATTN_ERR_INVALID;
  p.total = static_cast<int>(total);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_ns = wait_ns;
  p.debug_flags = debug_flags;
  p.window = window;
  const int grid = static_cast<int>(total < info.sm_count ? total : info.sm_count);
  // Causal items go KV head by KV head, in blocks of query levels, when the K
  // and V of all heads are larger than L2 (otherwise all heads of a query
  // level run together, which balances the triangular work more finely). A
  // block holds lcm(grid, group) / group levels: a whole number of rounds.
  const long long kv_bytes = 2LL * B * Hkv * static_cast<long long>(Nk) * d * 2;
  p.head_major = 0;
  if (causal && kv_bytes > info.l2_bytes && ETA_PREFILL_HEAD_MAJOR) {
    int a = grid, b = p.group;
    while (b != 0) {
      const int t = a % b;
      a = b;
      b = t;
    }
    p.head_major = grid / a;  // lcm(grid, group) / group
  }
  if constexpr (OUT_F32) {
    if (window > 0) return ATTN_ERR_INVALID;
    if (d == 128)
      return causal ? launch_prefill<128, T, true, false, true>(tq, tk, tv, to, p, grid, st)
                    : launch_prefill<128, T, false, false, true>(tq, tk, tv, to, p, grid, st);
    return causal ? launch_prefill<64, T, true, false, true>(tq, tk, tv, to, p, grid, st)
                  : launch_prefill<64, T, false, false, true>(tq, tk, tv, to, p, grid, st);
  }
  if (window > 0)
    return d == 128 ? launch_prefill<128, T, true, true>(tq, tk, tv, to, p, grid, st)
                    : launch_prefill<64, T, true, true>(tq, tk, tv, to, p, grid, st);
  if (d == 128)
    return causal ? launch_prefill<128, T, true>(tq, tk, tv, to, p, grid, st)
                  : launch_prefill<128, T, false>(tq, tk, tv, to, p, grid, st);
  return causal ? launch_prefill<64, T, true>(tq, tk, tv, to, p, grid, st)
                : launch_prefill<64, T, false>(tq, tk, tv, to, p, grid, st);
}

// Query heads one split CTA serves: the group padded to 4; larger groups are
// split into chunks of 4 heads, each chunk reading the cache. A tile of 8
// heads (ETA_DECODE_MAX_GP=8) reads the cache half as often, but its 8 output
// rows per lane need 216 registers (one resident CTA fewer per SM) and each
// key batch carries twice the shuffle and FMA work: measured on B200 for
// B=64, 1024..8192 tokens, d=128, it took 0.674 / 0.435 / 0.627 ms for
// groups of 8 / 32 (MQA) / 16 against 0.441 / 0.256 / 0.402 ms with 4, and
// the same 0.248 ms for a group of 4.
#ifndef ETA_DECODE_MAX_GP
#define ETA_DECODE_MAX_GP 4
#endif
static_assert(ETA_DECODE_MAX_GP == 4 || ETA_DECODE_MAX_GP == 8, "decode group tile");
inline int decode_group_tile(int G) { return (G <= 4 || ETA_DECODE_MAX_GP == 4) ? 4 : 8; }

// Split-KV count: enough CTAs for about ETA_DECODE_WAVES waves of resident
// split CTAs (3 resident per SM), at most 64 splits.
#ifndef ETA_DECODE_WAVES
#define ETA_DECODE_WAVES 8
#endif
// Persistent streaming pass (decode_ps_sm100.cuh) for d = 128 and
// ETA_DECODE_PS_MIN_G to 32 query heads per KV head; 0 turns it off (the
// CUDA-core split pass then takes every group). Measured on B200 (64
// sequences of 1K-8K tokens, d = 128, median of 30 launches, L2 flushed):
// group 4 0.236 ms against 0.246 ms on the CUDA-core pass; groups of 8 / 16 /
// 32 0.238 / 0.240 / 0.088 ms against 0.248 / 0.256 / 0.099 ms on an earlier
// tensor-core pass with one CTA per (sequence, KV head, split) and a combine
// kernel (removed); a single head per KV head (MHA) 0.236 ms against 0.232 ms
// on the CUDA-core pass, which keeps it.
#ifndef ETA_DECODE_PS_MIN_G
#define ETA_DECODE_PS_MIN_G 2
#endif
// Softmax warps per key quarter in the persistent pass, by group size (each
// thread takes GP / HS of the heads of its key, at least 8 when HS > 1).
// Measured on B200 (64 sequences of 1K-8K tokens, median of 30 launches):
// groups of 16 at d = 64 0.1846 ms with 2 warps per quarter against 0.2174 ms
// with 1; at d = 128 0.2379 against 0.2358 ms before the K/V split and the
// tile-max vote, 0.1948-0.1969 against 0.2051 ms after them; groups of 32
// (MQA) 0.0658 / 0.0515 ms with 4 against 0.0679 / 0.0556 ms with 2 at
// d = 128 / 64.
#ifndef ETA_DECODE_PS_HS16_D64
#define ETA_DECODE_PS_HS16_D64 2
#endif
#ifndef ETA_DECODE_PS_HS16_D128
#define ETA_DECODE_PS_HS16_D128 2
#endif
#ifndef ETA_DECODE_PS_HS32
#define ETA_DECODE_PS_HS32 4
#endif
// The same pass for d = 64 and ETA_DECODE_PS64_MIN_G to 32 query heads per KV
// head (0 turns it off); the CUDA-core pass reads the cache once per chunk of
// 4 heads, so larger groups at d = 64 belong here.
#ifndef ETA_DECODE_PS64_MIN_G
#define ETA_DECODE_PS64_MIN_G 2
#endif
inline bool decode_use_ps(int G, int d) {
  if (G > 32) return false;
  if (d == 128) return ETA_DECODE_PS_MIN_G > 0 && G >= ETA_DECODE_PS_MIN_G;
  if (d == 64) return ETA_DECODE_PS64_MIN_G > 0 && G >= ETA_DECODE_PS64_MIN_G;
  return false;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Device workspace of the persistent pass, byte offsets: the plan (token
// offsets int64 [B], tile offsets int32 [B + 1]) and, when CTAs take equal
// tile ranges, each CTA's first tile (int4 [nc]) and the partials of segments
// cut between CTAs (slot segment + cta: B * Hkv + nc - 1 slots of G rows).
struct PsLayout {
  size_t tok_off, tile_off, starts, part_o, part_lse, total;
};
inline PsLayout ps_layout(int B, int Hkv, int G, int d, int nc, bool partials) {
  PsLayout L;
  L.tok_off = 0;
  L.tile_off = align_up(static_cast<size_t>(B) * 8, 256);
  size_t end = L.tile_off + (static_cast<size_t>(B) + 1) * 4;
  L.starts = L.part_o = L.part_lse = 0;
  if (partials) {
    const size_t slots = static_cast<size_t>(B) * Hkv + nc - 1;
    L.starts = align_up(end, 256);
    end = L.starts + static_cast<size_t>(nc) * 16;
    L.part_o = align_up(end, 256);
    end = L.part_o + slots * G * d * 4;
    L.part_lse = align_up(end, 256);
    end = L.part_lse + slots * G * 4;
  }
  L.total = align_up(end, 256);
  return L;
}

int decode_splits(int B, int Hq, int Hkv, int sm_count) {
  const int G = Hq / Hkv;
  const int GP = decode_group_tile(G);
  const int nchunk = (G + GP - 1) / GP;
  const long long units = static_cast<long long>(B) * Hkv * nchunk;
  const long long resident = 3LL * sm_count;
  long long ns = units > 0 ? (ETA_DECODE_WAVES * resident + units - 1) / units : 1;
  if (ns < 1) ns = 1;
  if (ns > 64) ns = 64;
  return static_cast<int>(ns);
}

template <int D, int GP, typename T>
int launch_decode_split(const decode::DParams& p, cudaStream_t st) {
  auto kern = decode::attn_decode_split_kernel<D, GP, T>;
  constexpr int smem = decode::DCfg<D, GP>::kSmemBytes;
  static PerDeviceOnce attr;
  const cudaError_t attr_err = attr.run([&]() {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (attr_err != cudaSuccess) return cuda_fail(attr_err);
  const dim3 grid(static_cast<unsigned>(p.nsplit), static_cast<unsigned>(p.Hkv * p.nchunk),
                  static_cast<unsigned>(p.B));
  kern<<<grid, decode::kThreads, smem, st>>>(p);
  return launch_status();
}

// Token offsets of a large batch's sequences in the packed cache (one scan
// per call); smaller batches leave `tok_off` NULL and each CTA sums at most
// kOffsetsMinBatch lengths itself.
inline bool decode_needs_offsets(int B) { return B > decode::kOffsetsMinBatch; }
inline size_t offsets_bytes(int B) {
  return decode_needs_offsets(B) ? align_up(static_cast<size_t>(B) * 8, 256) : 0;
}
int launch_decode_offsets(const int32_t* seqlens, long long* tok_off, int B, cudaStream_t st) {
  decode::attn_decode_offsets_kernel<<<1, decode::kOffThreads, 0, st>>>(seqlens, tok_off, B);
  return launch_status();
}

// Plan, persistent stream and gather of the d = 128 decode; `ws` holds the
// layout `L`. seg_aligned: whole segments per CTA (L has no partials, and
// there is nothing to gather).
template <int NP, int GP, int HS, int D, typename T>
int launch_decode_ps(const CUtensorMap& tq, decode_ps::PParams p, const PsLayout& L, char* ws,
                     int nc, cudaStream_t st) {
  auto kern = decode_ps::attn_decode_persistent_kernel<NP, GP, HS, D, T>;
  constexpr int smem = decode_ps::PCfg<NP, D>::kSmemBytes;
  static PerDeviceOnce attr;
  const cudaError_t attr_err = attr.run([&]() {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (attr_err != cudaSuccess) return cuda_fail(attr_err);
  p.tok_off = reinterpret_cast<long long*>(ws + L.tok_off);
  p.tile_off = reinterpret_cast<int*>(ws + L.tile_off);
  p.starts = L.starts ? reinterpret_cast<int4*>(ws + L.starts) : nullptr;
  p.part_o = L.part_o ? reinterpret_cast<float*>(ws + L.part_o) : nullptr;
  p.part_lse = L.part_lse ? reinterpret_cast<float*>(ws + L.part_lse) : nullptr;
  if (!p.inline_plan) {
    decode_ps::attn_decode_plan_kernel<D><<<1, decode_ps::kPlanThreads, 0, st>>>(p, nc);
    const int rc = launch_status();
    if (rc != ATTN_OK) return rc;
  }
  // The stream and gather kernels are launched as programmatic dependents:
  // each may start before the previous kernel ends and waits on the device
  // (griddepcontrol.wait) for its results, so launch gaps overlap work.
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(nc));
  cfg.blockDim = dim3(decode_ps::Roles<HS>::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tq, p);
  if (e != cudaSuccess) return cuda_fail(e);
  if (p.seg_aligned) return launch_status();  // no cut segments, nothing to gather
  const long long rows = static_cast<long long>(p.B) * p.Hq;
  cfg.gridDim = dim3(static_cast<unsigned>((rows + 3) / 4));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  e = cudaLaunchKernelEx(&cfg, decode_ps::attn_decode_gather_kernel<D, T>, p, nc);
  if (e != cudaSuccess) return cuda_fail(e);
  return launch_status();
}

template <int D, typename T>
int launch_decode_ps_group(const CUtensorMap& tq, const decode_ps::PParams& p, const PsLayout& L,
                           char* ws, int nc, cudaStream_t st) {
  if (p.G <= 4) return launch_decode_ps<16, 4, 1, D, T>(tq, p, L, ws, nc, st);
  if (p.G <= 8) return launch_decode_ps<16, 8, 1, D, T>(tq, p, L, ws, nc, st);
  if (p.G <= 16)
    return launch_decode_ps<16, 16, D == 64 ? ETA_DECODE_PS_HS16_D64 : ETA_DECODE_PS_HS16_D128, D, T>(
        tq, p, L, ws, nc, st);
  return launch_decode_ps<32, 32, ETA_DECODE_PS_HS32, D, T>(tq, p, L, ws, nc, st);
}

// Batches of up to this many sequences skip the plan kernel: each CTA of the
// persistent pass sums the lengths itself (one read of B lengths per CTA).
// Measured on B200 (64 sequences of 1K-8K tokens): group 4 0.2093 against
// 0.2112 ms with the plan kernel, group 16 0.2276 / 0.2358 ms, MQA 0.0617 /
// 0.0638 ms; 8 sequences of 16K-32K 0.1459 / 0.1539 ms.
#ifndef ETA_DECODE_INLINE_PLAN_MAX_B
#define ETA_DECODE_INLINE_PLAN_MAX_B 2048
#endif

// Cost of a segment start, in tiles, when the persistent pass's CTAs split
// the work among themselves (batches of up to ETA_DECODE_INLINE_PLAN_MAX_B
// sequences): a CTA that starts more pieces then takes fewer tiles. Groups of
// 9 to 16 and of 17 to 32 query heads; smaller groups split by tiles alone
// (their softmax step is short, so a piece costs little more than its tiles).
// Measured on B200 (64 sequences of 1K-8K tokens) against equal tile shares:
// group 16 at d = 64 0.1477-0.1497 against 0.1581-0.1600 ms, MQA at d = 64
// 0.0412-0.0418 / 0.0433 ms with 3 (0.0433 with 2); group 16 and MQA at
// d = 128 and 512-sequence MQA equal.
#ifndef ETA_DECODE_PS_SEG_COST16
#define ETA_DECODE_PS_SEG_COST16 2
#endif
#ifndef ETA_DECODE_PS_SEG_COST32
#define ETA_DECODE_PS_SEG_COST32 3
#endif

// The persistent decode for d = 64 and 128: q's tensor map (rows of the G
// heads of one KV head, box padded to NP rows), then the three kernels. `ws`
// must hold ps_layout(B, Hkv, G, d, nc, !seg_aligned).
template <typename T>
int decode_ps_run(const void* q, const void* kc, const void* vc, const int32_t* seqlens, void* o,
                  float* lse, int B, int Hq, int Hkv, int d, float scale, int window, char* ws,
                  bool seg_aligned, int nc, cudaStream_t st) {
  constexpr bool bf16 = std::is_same<T, __nv_bfloat16>::value;
  const int G = Hq / Hkv;
  const int NP = G <= 16 ? 16 : 32;
  CUtensorMap tq;
  const int rc = encode_3d(&tq, q, bf16, d, G, static_cast<long long>(B) * Hkv,
                           static_cast<unsigned>(NP));
  if (rc != ATTN_OK) return rc;
  decode_ps::PParams p;
  p.q = q;
  p.kc = kc;
  p.vc = vc;
  p.seqlens = seqlens;
  p.o = o;
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.window = window;
  p.seg_aligned = seg_aligned ? 1 : 0;
  p.inline_plan = (!seg_aligned && B <= ETA_DECODE_INLINE_PLAN_MAX_B) ? 1 : 0;
  p.wcost = !p.inline_plan ? 0
            : G <= 8       ? 0
            : G <= 16      ? ETA_DECODE_PS_SEG_COST16
                           : ETA_DECODE_PS_SEG_COST32;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_ns = kDefaultWaitNs;
  const PsLayout L = ps_layout(B, Hkv, G, d, nc, !seg_aligned);
  return d == 128 ? launch_decode_ps_group<128, T>(tq, p, L, ws, nc, st)
                  : launch_decode_ps_group<64, T>(tq, p, L, ws, nc, st);
}

template <int D, typename T>
int launch_decode_combine(const float* po, const float* pl, void* o, float* lse, int rows,
                          int nsplit, cudaStream_t st) {
  const int blocks = (rows + 3) / 4;
  decode::attn_decode_combine_kernel<D, T>
      <<<blocks, 128, 0, st>>>(po, pl, reinterpret_cast<T*>(o), lse, rows, nsplit);
  return launch_status();
}

template <int D, typename T>
int decode_launch_all(const decode::DParams& p, void* o, float* lse, cudaStream_t st) {
  if (p.tok_off != nullptr) {
    const int rc = launch_decode_offsets(p.seqlens, const_cast<long long*>(p.tok_off), p.B, st);
    if (rc != ATTN_OK) return rc;
  }
#if ETA_DECODE_MAX_GP == 8
  const int GP = decode_group_tile(p.G);
  int rc = GP == 4 ? launch_decode_split<D, 4, T>(p, st) : launch_decode_split<D, 8, T>(p, st);
#else
  int rc = launch_decode_split<D, 4, T>(p, st);
#endif
  if (rc != ATTN_OK) return rc;
  return launch_decode_combine<D, T>(p.part_o, p.part_lse, o, lse, p.B * p.Hq, p.nsplit, st);
}

// Decode for head sizes other than 64 and 128: the generic kernel in decode
// mode, one CTA per (sequence, query head). `tok_off`: room for B token
// offsets, filled here by the scan, or NULL (each CTA sums them).
template <typename T>
int decode_generic(const void* q, const void* kc, const void* vc, const int32_t* seqlens,
                   void* o, float* lse, int B, int Hq, int Hkv, int d, float scale, int window,
                   long long* tok_off, cudaStream_t st) {
  if (tok_off != nullptr) {
    const int rc = launch_decode_offsets(seqlens, tok_off, B, st);
    if (rc != ATTN_OK) return rc;
  }
  generic::GParams g;
  g.q = q;
  g.k = kc;
  g.v = vc;
  g.o = o;
  g.lse = lse;
  g.Hq = Hq;
  g.Hkv = Hkv;
  g.Nq = 1;
  g.Nk = 0;  // per sequence, from seqlens
  g.d = d;
  g.group = Hq / Hkv;
  g.off = 0;
  g.causal = 1;
  g.window = window;
  g.scale_log2 = scale * 1.4426950408889634f;
  g.seqlens = seqlens;
  g.tok_off = tok_off;
  return launch_generic<T>(g, B * Hq, 1, st);
}

template <typename T>
int decode_run(const void* q, const void* kc, const void* vc, const int32_t* seqlens, void* o,
               float* lse, int B, int Hq, int Hkv, int d, float scale, cudaStream_t st,
               int window = 0) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || !scale_ok(scale) || window < 0)
    return ATTN_ERR_INVALID;
  if (!tensor_core_d(d) && !generic_d(d)) return ATTN_ERR_UNSUPPORTED;
  if (tensor_core_d(d) && B > 65535) return ATTN_ERR_UNSUPPORTED;  // one grid z slice per sequence
  if (static_cast<long long>(B) * Hq > 0x7fffffffLL / 4) return ATTN_ERR_INVALID;
  if (B == 0) return ATTN_OK;
  if (q == nullptr || kc == nullptr || vc == nullptr || seqlens == nullptr || o == nullptr ||
      !aligned(q, 16) || !aligned(kc, 16) || !aligned(vc, 16) || !aligned(o, 16) ||
      !aligned(seqlens, 4) || (lse != nullptr && !aligned(lse, 4)))
    return ATTN_ERR_INVALID;
  DeviceInfo info;
  if (device_info(&info) != ATTN_OK) return ATTN_ERR_CUDA;
  if (!info.sm100) return ATTN_ERR_UNSUPPORTED;
  cudaMemPool_t pool;
  if (!tensor_core_d(d)) {
    if (!decode_needs_offsets(B))
      return decode_generic<T>(q, kc, vc, seqlens, o, lse, B, Hq, Hkv, d, scale, window,
                               nullptr, st);
    void* ws = nullptr;
    if (workspace_pool(&pool) != ATTN_OK) return ATTN_ERR_CUDA;
    if (cudaMallocFromPoolAsync(&ws, offsets_bytes(B), pool, st) != cudaSuccess)
      return ATTN_ERR_CUDA;
    const int rc = decode_generic<T>(q, kc, vc, seqlens, o, lse, B, Hq, Hkv, d, scale, window,
                                     static_cast<long long*>(ws), st);
    const cudaError_t fe = cudaFreeAsync(ws, st);
    if (rc != ATTN_OK) return rc;
    return fe == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  if (decode_use_ps(Hq / Hkv, d)) {
    const int nc = info.sm_count;
    const PsLayout L = ps_layout(B, Hkv, Hq / Hkv, d, nc, true);
    void* ws = nullptr;
    if (workspace_pool(&pool) != ATTN_OK) return ATTN_ERR_CUDA;
    if (cudaMallocFromPoolAsync(&ws, L.total, pool, st) != cudaSuccess) return ATTN_ERR_CUDA;
    const int rc = decode_ps_run<T>(q, kc, vc, seqlens, o, lse, B, Hq, Hkv, d, scale, window,
                                    static_cast<char*>(ws), false, nc, st);
    const cudaError_t fe = cudaFreeAsync(ws, st);
    if (rc != ATTN_OK) return rc;
    return fe == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }

  decode::DParams p;
  p.q = q;
  p.kc = kc;
  p.vc = vc;
  p.seqlens = seqlens;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  const int GP = decode_group_tile(p.G);
  p.nchunk = (p.G + GP - 1) / GP;
  p.nsplit = decode_splits(B, Hq, Hkv, info.sm_count);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_ns = kDefaultWaitNs;
  p.window = window;

  // Workspace: the token offsets (large batches), then the split partials.
  const size_t rows = static_cast<size_t>(B) * Hq;
  const size_t off_bytes = offsets_bytes(B);
  const size_t bytes = off_bytes + static_cast<size_t>(p.nsplit) * rows * (d + 1) * sizeof(float);
  void* ws = nullptr;
  if (workspace_pool(&pool) != ATTN_OK) return ATTN_ERR_CUDA;
  if (cudaMallocFromPoolAsync(&ws, bytes, pool, st) != cudaSuccess) return ATTN_ERR_CUDA;
  p.tok_off = off_bytes ? static_cast<long long*>(ws) : nullptr;
  p.part_o = reinterpret_cast<float*>(static_cast<char*>(ws) + off_bytes);
  p.part_lse = p.part_o + static_cast<size_t>(p.nsplit) * rows * d;
  const int rc = d == 128 ? decode_launch_all<128, T>(p, o, lse, st)
                          : decode_launch_all<64, T>(p, o, lse, st);
  const cudaError_t fe = cudaFreeAsync(ws, st);
  if (rc != ATTN_OK) return rc;
  return fe == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace api
}  // namespace eta

namespace eta {
namespace api {

// T: type of o_out; TP: type of o_part (T, or float for unrounded partials).
template <typename T, typename TP = T>
int merge_run(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
              void* o_out, long long rows, int d, cudaStream_t st) {
  if (rows < 0 || !generic_d(d)) return rows < 0 ? ATTN_ERR_INVALID : ATTN_ERR_UNSUPPORTED;
  if (rows > (0x7fffffffffffLL / d)) return ATTN_ERR_INVALID;
  if (rows == 0) return ATTN_OK;
  if (o_acc == nullptr || lse_acc == nullptr || o_part == nullptr || lse_part == nullptr ||
      !aligned(o_acc, 16) || !aligned(o_part, 16) || !aligned(lse_acc, 4) ||
      !aligned(lse_part, 4) || (o_out != nullptr && !aligned(o_out, 16)))
    return ATTN_ERR_INVALID;
  DeviceInfo info;
  if (device_info(&info) != ATTN_OK) return ATTN_ERR_CUDA;
  if (!info.sm100) return ATTN_ERR_UNSUPPORTED;
  const int rpw = 32 / (d / 8);
  const long long rows_per_block = static_cast<long long>(rpw) * (merge::kThreads / 32);
  const long long want = (rows + rows_per_block - 1) / rows_per_block;
  const long long cap = 8LL * info.sm_count;  // grid-stride beyond 8 blocks per SM
  const int blocks = static_cast<int>(want < cap ? want : cap);
  merge::attn_merge_kernel<T, TP><<<blocks, merge::kThreads, 0, st>>>(
      o_acc, lse_acc, reinterpret_cast<const TP*>(o_part), lse_part, reinterpret_cast<T*>(o_out),
      rows, d);
  return launch_status();
}

}  // namespace api
}  // namespace eta

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
             int Hkv, int Nq, int Nk, int d, float scale, int causal, attn_stream_t stream) {
  return eta::api::fwd<__nv_bfloat16>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                                      reinterpret_cast<cudaStream_t>(stream),
                                      eta::kDefaultWaitNs, 0);
}

int attn_fwd_f16(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                 int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                 attn_stream_t stream) {
  return eta::api::fwd<__half>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                               reinterpret_cast<cudaStream_t>(stream), eta::kDefaultWaitNs, 0);
}

int attn_decode(const void* q, const void* kcache, const void* vcache, const int32_t* seqlens,
                void* o, float* lse, int B, int Hq, int Hkv, int d, float scale,
                attn_stream_t stream) {
  return eta::api::decode_run<__nv_bfloat16>(q, kcache, vcache, seqlens, o, lse, B, Hq, Hkv, d,
                                             scale, reinterpret_cast<cudaStream_t>(stream));
}

int attn_decode_f16(const void* q, const void* kcache, const void* vcache,
                    const int32_t* seqlens, void* o, float* lse, int B, int Hq, int Hkv, int d,
                    float scale, attn_stream_t stream) {
  return eta::api::decode_run<__half>(q, kcache, vcache, seqlens, o, lse, B, Hq, Hkv, d, scale,
                                      reinterpret_cast<cudaStream_t>(stream));
}

int attn_decode_num_splits(int B, int Hq, int Hkv, int d) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID;
  if (!eta::api::tensor_core_d(d)) return eta::api::generic_d(d) ? 1 : ATTN_ERR_UNSUPPORTED;
  if (eta::api::decode_use_ps(Hq / Hkv, d)) return 1;  // one streaming pass, no fixed split
  eta::api::DeviceInfo info;
  if (eta::api::device_info(&info) != ATTN_OK) return ATTN_ERR_CUDA;
  return eta::api::decode_splits(B, Hq, Hkv, info.sm_count);
}

const char* attn_strerror(int code) {
  switch (code) {
    case ATTN_OK:
      return "ok";
    case ATTN_ERR_INVALID:
      return "invalid argument (null or misaligned pointer, bad size, Hq % Hkv != 0, or scale "
             "not finite and > 0)";
    case ATTN_ERR_UNSUPPORTED:
      return "unsupported (head dim not a multiple of 8 in [8, 256]; decode with d = 64 or 128 "
             "and B > 65,535; or a device other than sm_100)";
    case ATTN_ERR_CUDA:
      return "CUDA runtime error";
    case ATTN_ERR_TIMEOUT:
      return "a device-side wait gave up; outputs of that launch are undefined";
    case ATTN_ERR_SCRATCH:
      return "attn_decode_noalloc: one split of the CUDA-core decode pass (B * Hq * (d + 1) "
             "floats, plus B int64 token offsets above 1024 sequences) exceeds its fixed array "
             "of 2,097,152 floats";
    default:
      return "unknown error code";
  }
}

int attn_get_device_status(attn_stream_t stream, unsigned int* raw_code) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, eta::g_status, sizeof(v)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (v != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(eta::g_status, &zero, sizeof(zero)) != cudaSuccess)
      return ATTN_ERR_CUDA;
  }
  if (raw_code != nullptr) *raw_code = v;
  return v == 0 ? ATTN_OK : ATTN_ERR_TIMEOUT;
}

int attn_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int Hq, int Hkv, int Nq, int Nk, int d, float scale, int window,
                    attn_stream_t stream) {
  if (window < 1) return ATTN_ERR_INVALID;
  return eta::api::fwd<__nv_bfloat16>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, 1,
                                      reinterpret_cast<cudaStream_t>(stream),
                                      eta::kDefaultWaitNs, 0, window);
}

int attn_fwd_window_f16(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int Hq, int Hkv, int Nq, int Nk, int d, float scale, int window,
                        attn_stream_t stream) {
  if (window < 1) return ATTN_ERR_INVALID;
  return eta::api::fwd<__half>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, 1,
                               reinterpret_cast<cudaStream_t>(stream), eta::kDefaultWaitNs, 0,
                               window);
}

int attn_decode_window(const void* q, const void* kcache, const void* vcache,
                       const int32_t* seqlens, void* o, float* lse, int B, int Hq, int Hkv, int d,
                       float scale, int window, attn_stream_t stream) {
  if (window < 1) return ATTN_ERR_INVALID;
  return eta::api::decode_run<__nv_bfloat16>(q, kcache, vcache, seqlens, o, lse, B, Hq, Hkv, d,
                                             scale, reinterpret_cast<cudaStream_t>(stream),
                                             window);
}

int attn_decode_window_f16(const void* q, const void* kcache, const void* vcache,
                           const int32_t* seqlens, void* o, float* lse, int B, int Hq, int Hkv,
                           int d, float scale, int window, attn_stream_t stream) {
  if (window < 1) return ATTN_ERR_INVALID;
  return eta::api::decode_run<__half>(q, kcache, vcache, seqlens, o, lse, B, Hq, Hkv, d, scale,
                                      reinterpret_cast<cudaStream_t>(stream), window);
}

int attn_last_cuda_error(void) { return eta::api::g_last_cuda_error; }

int attn_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
               void* o_out, long long rows, int d, attn_stream_t stream) {
  return eta::api::merge_run<__nv_bfloat16>(o_acc, lse_acc, o_part, lse_part, o_out, rows, d,
                                            reinterpret_cast<cudaStream_t>(stream));
}

int attn_merge_f16(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                   void* o_out, long long rows, int d, attn_stream_t stream) {
  return eta::api::merge_run<__half>(o_acc, lse_acc, o_part, lse_part, o_out, rows, d,
                                     reinterpret_cast<cudaStream_t>(stream));
}

int attn_fwd_partial(const void* q, const void* k, const void* v, float* o, float* lse, int B,
                     int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                     attn_stream_t stream) {
  return eta::api::fwd<__nv_bfloat16, true>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                                            reinterpret_cast<cudaStream_t>(stream),
                                            eta::kDefaultWaitNs, 0);
}

int attn_fwd_partial_f16(const void* q, const void* k, const void* v, float* o, float* lse, int B,
                         int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                         attn_stream_t stream) {
  return eta::api::fwd<__half, true>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                                     reinterpret_cast<cudaStream_t>(stream), eta::kDefaultWaitNs,
                                     0);
}

int attn_merge_partial(float* o_acc, float* lse_acc, const float* o_part, const float* lse_part,
                       void* o_out, long long rows, int d, attn_stream_t stream) {
  return eta::api::merge_run<__nv_bfloat16, float>(o_acc, lse_acc, o_part, lse_part, o_out, rows,
                                                   d, reinterpret_cast<cudaStream_t>(stream));
}

int attn_merge_partial_f16(float* o_acc, float* lse_acc, const float* o_part,
                           const float* lse_part, void* o_out, long long rows, int d,
                           attn_stream_t stream) {
  return eta::api::merge_run<__half, float>(o_acc, lse_acc, o_part, lse_part, o_out, rows, d,
                                            reinterpret_cast<cudaStream_t>(stream));
}

int attn_fwd_stall_test(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                        unsigned int wait_us, attn_stream_t stream) {
  if (wait_us < 1 || wait_us > 1000000) return ATTN_ERR_INVALID;
  return eta::api::fwd<__nv_bfloat16>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                                      reinterpret_cast<cudaStream_t>(stream),
                                      static_cast<uint64_t>(wait_us) * 1000ull, 1);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode without any allocation.
//
// attn_decode takes its split-KV scratch from cudaMallocAsync. Some callers
// cannot allocate device memory at the point where they run attention: a
// serving engine that hands nearly all of HBM to its own KV-cache pool at
// start-up (so an extra allocation can fail, or fragment that pool), code on a
// latency-critical path where an allocator call may take a lock or synchronise,
// and runtimes that fix their whole memory plan before the first request. For
// them, attn_decode_noalloc runs the same two decode kernels with the scratch
// taken from a fixed array in this library's device memory instead.
namespace eta {
namespace api {

// Capacity of the fixed scratch, in floats (8 MiB). Every GPU that loads the
// library holds this much device memory until the process exits.
constexpr size_t kNoAllocScratchFloats = size_t(2) << 20;

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

// On the host, g_noalloc_scratch names a host-side stand-in, not device
// memory: a kernel handed that name would fault or, where the GPU can reach
// host memory, silently use the wrong memory. The device address is looked up
// here with the device current, once per device and context: the context's
// unique id is remembered with the address, so after cudaDeviceReset (which
// ends the context and the module with it) the next call looks the address up
// again instead of using a dead one.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(ptr);
}

// Unique id of the calling thread's current context; 0 if there is none.
unsigned long long current_context_id() {
  static const CtxGetCurrentFn get_ctx = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (get_ctx == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

int noalloc_scratch(float** out) {
  static std::mutex mu;
  static float* addr[64] = {};
  static unsigned long long ctx_id[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long id = current_context_id();
  if (addr[dev] == nullptr || id == 0 || id != ctx_id[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return ATTN_ERR_CUDA;
    addr[dev] = static_cast<float*>(p);
    ctx_id[dev] = current_context_id();  // the look-up made the context current if it was not
  }
  *out = addr[dev];
  return ATTN_OK;
}

template <typename T>
int decode_run_noalloc(const void* q, const void* kc, const void* vc, const int32_t* seqlens,
                       void* o, float* lse, int B, int Hq, int Hkv, int d, float scale,
                       cudaStream_t st) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || !scale_ok(scale)) return ATTN_ERR_INVALID;
  if (!tensor_core_d(d) && !generic_d(d)) return ATTN_ERR_UNSUPPORTED;
  if (tensor_core_d(d) && B > 65535) return ATTN_ERR_UNSUPPORTED;  // one grid z slice per sequence
  if (static_cast<long long>(B) * Hq > 0x7fffffffLL / 4) return ATTN_ERR_INVALID;
  if (B == 0) return ATTN_OK;
  if (q == nullptr || kc == nullptr || vc == nullptr || seqlens == nullptr || o == nullptr ||
      !aligned(q, 16) || !aligned(kc, 16) || !aligned(vc, 16) || !aligned(o, 16) ||
      !aligned(seqlens, 4) || (lse != nullptr && !aligned(lse, 4)))
    return ATTN_ERR_INVALID;
  if (!tensor_core_d(d)) {
    // The generic kernel needs scratch only for the token offsets of a large
    // batch; beyond the scratch's capacity (a million sequences) each CTA
    // sums them itself.
    DeviceInfo info;
    if (device_info(&info) != ATTN_OK) return ATTN_ERR_CUDA;
    if (!info.sm100) return ATTN_ERR_UNSUPPORTED;
    long long* tok_off = nullptr;
    if (decode_needs_offsets(B) && offsets_bytes(B) <= kNoAllocScratchFloats * sizeof(float)) {
      float* scratch = nullptr;
      if (noalloc_scratch(&scratch) != ATTN_OK) return ATTN_ERR_CUDA;
      tok_off = reinterpret_cast<long long*>(scratch);
    }
    return decode_generic<T>(q, kc, vc, seqlens, o, lse, B, Hq, Hkv, d, scale, 0, tok_off, st);
  }
  DeviceInfo info;
  if (device_info(&info) != ATTN_OK) return ATTN_ERR_CUDA;
  if (!info.sm100) return ATTN_ERR_UNSUPPORTED;
  if (decode_use_ps(Hq / Hkv, d)) {
    // The plan always fits (B <= 65,535); the partials of equal tile ranges
    // when they fit, else every CTA takes whole segments and writes its
    // results directly.
    const int nc = info.sm_count;
    const size_t cap = kNoAllocScratchFloats * sizeof(float);
    const bool seg_aligned = ps_layout(B, Hkv, Hq / Hkv, d, nc, true).total > cap;
    if (ps_layout(B, Hkv, Hq / Hkv, d, nc, !seg_aligned).total > cap) return ATTN_ERR_SCRATCH;
    float* scratch = nullptr;
    if (noalloc_scratch(&scratch) != ATTN_OK) return ATTN_ERR_CUDA;
    return decode_ps_run<T>(q, kc, vc, seqlens, o, lse, B, Hq, Hkv, d, scale, 0,
                            reinterpret_cast<char*>(scratch), seg_aligned, nc, st);
  }

  decode::DParams p;
  p.q = q;
  p.kc = kc;
  p.vc = vc;
  p.seqlens = seqlens;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  const int GP = decode_group_tile(p.G);
  p.nchunk = (p.G + GP - 1) / GP;
  // Scratch: the token offsets of a large batch, then the split partials.
  // One split needs B * Hq * (d + 1) floats; fewer splits than attn_decode's
  // count are used when that count does not fit, and a call where not one
  // split fits is refused.
  const size_t rows = static_cast<size_t>(B) * Hq;
  const size_t off_bytes = offsets_bytes(B);
  const size_t cap = kNoAllocScratchFloats * sizeof(float);
  const size_t per_split = rows * (d + 1) * sizeof(float);
  const size_t fit = off_bytes < cap ? (cap - off_bytes) / per_split : 0;
  const int want = decode_splits(B, Hq, Hkv, info.sm_count);
  p.nsplit = static_cast<int>(fit < static_cast<size_t>(want) ? fit : want);
  if (p.nsplit < 1) return ATTN_ERR_SCRATCH;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_ns = kDefaultWaitNs;
  p.window = 0;
  float* scratch = nullptr;
  if (noalloc_scratch(&scratch) != ATTN_OK) return ATTN_ERR_CUDA;
  // Every offset and partial slot is written before it is read, so nothing
  // in the scratch has to start at zero.
  char* base = reinterpret_cast<char*>(scratch);
  p.tok_off = off_bytes ? reinterpret_cast<long long*>(base) : nullptr;
  p.part_o = reinterpret_cast<float*>(base + off_bytes);
  p.part_lse = p.part_o + static_cast<size_t>(p.nsplit) * rows * d;
  return d == 128 ? decode_launch_all<128, T>(p, o, lse, st)
                  : decode_launch_all<64, T>(p, o, lse, st);
}

}  // namespace api
}  // namespace eta

extern "C" int attn_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                                   const int32_t* seqlens, void* o, float* lse, int B, int Hq,
                                   int Hkv, int d, float scale, attn_stream_t stream) {
  return eta::api::decode_run_noalloc<__nv_bfloat16>(q, kcache, vcache, seqlens, o, lse, B, Hq,
                                                     Hkv, d, scale,
                                                     reinterpret_cast<cudaStream_t>(stream));
}
