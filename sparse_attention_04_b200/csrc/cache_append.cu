// cache_append.cu -- the cache write of the newest tokens, and act_quant of
// the indexer queries for the e4m3 path.
//
// "DeepSeek-V3.2-Exp - Keep top-k positions", Indexer.forward: q and k are
// quantised by act_quant (block size 128) before fp8_index, the new keys go
// into the key cache beside their scales (k_cache[start:end] = k_fp8), and
// the per-head weights are multiplied by q's scale.  The latent cache takes
// the new latent row (the kv_cache / pe_cache writes of the MLA listing).
// act_quant itself is not printed on the pages; as for the inputs of the
// e4m3 workload: one block = one 128-element vector, scale = amax / 448 in
// fp32 (1 when amax = 0), codes = e4m3 nearest to x / scale, ties to even,
// saturating.  Both divisions are IEEE round-to-nearest, so the codes are
// the same bits any fp32 implementation of that rule produces.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "dsa_internal.h"
#include "sm100.cuh"

namespace dsa {
namespace {

// One warp quantises one 128-element bf16 vector: lane l holds elements
// 4l .. 4l+3.  Returns the block's scale (in every lane).
__device__ __forceinline__ float quantize128(const __nv_bfloat16* __restrict__ src, uint8_t* __restrict__ dst,
                                             int lane) {
  const uint2 raw = *reinterpret_cast<const uint2*>(src + 4 * lane);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
  float amax = fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(b.x), fabsf(b.y)));
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  const __nv_fp8x2_storage_t lo =
      __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(a.x, scale), __fdiv_rn(a.y, scale)), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi =
      __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(b.x, scale), __fdiv_rn(b.y, scale)), __NV_SATFINITE, __NV_E4M3);
  *reinterpret_cast<uint32_t*>(dst + 4 * lane) = (uint32_t)lo | ((uint32_t)hi << 16);
  return scale;
}

// One warp per new token (b, t): its rows sit at offsets[b+1] - T + t.
__global__ void __launch_bounds__(256)
    cache_append_kernel(const __nv_bfloat16* __restrict__ k_new, const __nv_bfloat16* __restrict__ kv_new,
                        const int32_t* __restrict__ off, int B, int T, int fp8, void* __restrict__ k_cache,
                        float* __restrict__ k_scale, __nv_bfloat16* __restrict__ kv_cache, int64_t kv_rows,
                        int32_t* status) {
  grid_dependency_wait();  // the new rows may come from the previous kernel
  allow_dependents_launch();
  const int lane = threadIdx.x & 31;
  const int64_t tok = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (tok >= (int64_t)B * T) return;
  const int b = (int)(tok / T), t = (int)(tok - (int64_t)b * T);
  const int32_t lo = off[b], hi = off[b + 1];
  if (lo < 0 || hi - lo < T || (int64_t)hi > kv_rows) {
    if (lane == 0) report(status, DSA_ERR_BAD_OFFSETS);
    return;
  }
  const int64_t row = (int64_t)hi - T + t;
  if (kv_new) {
    const uint4* src = reinterpret_cast<const uint4*>(kv_new + tok * kDQK);
    uint4* dst = reinterpret_cast<uint4*>(kv_cache + row * kDQK);
#pragma unroll
    for (int c = 0; c < 3; ++c)
      if (lane + 32 * c < kDQK / 8) dst[lane + 32 * c] = src[lane + 32 * c];
  }
  if (k_new) {
    if (fp8) {
      const float sc = quantize128(k_new + tok * kDI, reinterpret_cast<uint8_t*>(k_cache) + row * kDI, lane);
      if (lane == 0) k_scale[row] = sc;
    } else if (lane < kDI / 8) {
      reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(k_cache) + row * kDI)[lane] =
          reinterpret_cast<const uint4*>(k_new + tok * kDI)[lane];
    }
  }
}

// One warp per (row, head) vector: codes, and w_out = w * scale (fp32).
__global__ void __launch_bounds__(256)
    quantize_queries_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ w, int64_t n_vec,
                            uint8_t* __restrict__ q8, float* __restrict__ w_out) {
  grid_dependency_wait();
  allow_dependents_launch();
  const int lane = threadIdx.x & 31;
  const int64_t v = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (v >= n_vec) return;
  const float sc = quantize128(q + v * kDI, q8 + v * kDI, lane);
  if (lane == 0) w_out[v] = w[v] * sc;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

int dsa_cache_append(const void* k_new, const void* kv_new, const int32_t* offsets, int B, int T, int idx_dtype,
                     void* k_idx_cache, float* k_scale_cache, void* kv_cache, int64_t kv_rows, int32_t* dev_status,
                     void* stream) {
  if (B <= 0 || T <= 0 || (int64_t)B * T > ((int64_t)1 << 24) || !offsets) return DSA_ERR_INVALID_ARG;
  if (!k_new && !kv_new) return DSA_ERR_INVALID_ARG;
  if (idx_dtype != DSA_BF16 && idx_dtype != DSA_E4M3) return DSA_ERR_INVALID_ARG;
  if (k_new && (!k_idx_cache || !aligned16(k_new) || !aligned16(k_idx_cache))) return DSA_ERR_INVALID_ARG;
  if (k_new && idx_dtype == DSA_E4M3 && !k_scale_cache) return DSA_ERR_INVALID_ARG;
  if (kv_new && (!kv_cache || !aligned16(kv_new) || !aligned16(kv_cache))) return DSA_ERR_INVALID_ARG;
  if (kv_rows < T || kv_rows > ((int64_t)1 << 31) - 1) return DSA_ERR_INVALID_ARG;
  const int64_t toks = (int64_t)B * T;
  const cudaError_t e = launch_pdl(cache_append_kernel, dim3((unsigned)((toks + 7) / 8)), dim3(256), 0,
                                   reinterpret_cast<cudaStream_t>(stream),
                                   reinterpret_cast<const __nv_bfloat16*>(k_new),
                                   reinterpret_cast<const __nv_bfloat16*>(kv_new), offsets, B, T,
                                   idx_dtype == DSA_E4M3 ? 1 : 0, k_idx_cache, k_scale_cache,
                                   reinterpret_cast<__nv_bfloat16*>(kv_cache), kv_rows, dev_status);
  return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

int dsa_quantize_queries(const void* q_idx, const float* w, int n_rows, void* q_idx_e4m3, float* w_out,
                         void* stream) {
  if (n_rows <= 0 || n_rows > (1 << 24) || !q_idx || !w || !q_idx_e4m3 || !w_out) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(q_idx_e4m3)) return DSA_ERR_INVALID_ARG;
  const int64_t n_vec = (int64_t)n_rows * kHI;
  const cudaError_t e = launch_pdl(quantize_queries_kernel, dim3((unsigned)((n_vec + 7) / 8)), dim3(256), 0,
                                   reinterpret_cast<cudaStream_t>(stream),
                                   reinterpret_cast<const __nv_bfloat16*>(q_idx), w, n_vec,
                                   reinterpret_cast<uint8_t*>(q_idx_e4m3), w_out);
  return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // extern "C"
