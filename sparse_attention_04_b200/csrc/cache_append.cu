// cache_append.cu -- preparation of the indexer's inputs: the rotary
// embedding and Hadamard rotation of q/k, the cache write of the newest
// tokens, and act_quant of the indexer queries for the e4m3 path.
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

#include <algorithm>

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

__device__ __forceinline__ float bf16_round(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

// Indexer pre-stage ("Keep top-k positions", Indexer.forward: the rope part
// of q/k through apply_rotary_emb(., freqs_cis, False), then
// rotate_activation).  A 128-vector is held by a lane pair, the 16-byte
// chunks alternating between the two lanes so that every load and store
// instruction of the warp covers whole 32-byte sectors: lane hh holds chunks
// 2k + hh (k = 0..7), i.e. e[8k + m] = entry 16k + 8hh + m.  Entry bits 0-2
// and 4-6 are therefore inside a lane and bit 3 is the pair's lane bit.
// Rope entry i pairs with entry i + 32 (not interleaved), which is e[j] and
// e[j + 16] of the same lane; each lane rotates its 32 rope entries and
// rounds them to bf16 (the model keeps q/k in bf16).  Then the
// Sylvester-order Walsh-Hadamard transform runs as seven butterfly stages,
// six inside the lane and one across the pair; the caller scales the result
// by 128^-1/2 and rounds it to bf16.  Every lane of the warp must call this
// (the last stage's shuffle spans the warp).
__device__ __forceinline__ void rope_hadamard128(float (&e)[64], int32_t p, const float* __restrict__ rope_cos,
                                                 const float* __restrict__ rope_sin, int hh) {
  const float* cp = rope_cos + (int64_t)p * 32 + 8 * hh;
  const float* sp = rope_sin + (int64_t)p * 32 + 8 * hh;
#pragma unroll
  for (int k = 0; k < 2; ++k) {  // entries 16k + 8hh + m, m < 8: angle index i = 16k + 8hh + m
    const float4 c0 = __ldg(reinterpret_cast<const float4*>(cp + 16 * k));
    const float4 c1 = __ldg(reinterpret_cast<const float4*>(cp + 16 * k + 4));
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(sp + 16 * k));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(sp + 16 * k + 4));
    const float c[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    const float sn[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int j = 8 * k + m;
      const float a = e[j], b = e[j + 16];  // entries i and i + 32
      // (a, b) -> (a cos - b sin, a sin + b cos)
      e[j] = bf16_round(fmaf(a, c[m], -(b * sn[m])));
      e[j + 16] = bf16_round(fmaf(a, sn[m], b * c[m]));
    }
  }
  // Hadamard butterflies: (u, w) -> (u + w, u - w), u the entry whose bit is clear
#pragma unroll
  for (int bit = 1; bit < 64; bit <<= 1) {  // local bits 0-5 = entry bits 0-2, 4-6
    // two butterflies per packed add: j and the next j with the bit clear
    const int nxt = bit == 1 ? 2 : 1;
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      if ((j & bit) || (j & nxt)) continue;
      const int j2 = j + nxt;
      const float2 u = make_float2(e[j], e[j2]), w = make_float2(e[j | bit], e[j2 | bit]);
      const float2 sm = __fadd2_rn(u, w);
      const float2 df = __ffma2_rn(w, make_float2(-1.f, -1.f), u);
      e[j] = sm.x;
      e[j2] = sm.y;
      e[j | bit] = df.x;
      e[j2 | bit] = df.y;
    }
  }
  const float sg = hh ? -1.f : 1.f;  // entry bit 3: the pair's upper lane takes u - w
#pragma unroll
  for (int j = 0; j < 64; ++j) {
    const float q = __shfl_xor_sync(0xffffffffu, e[j], 1);
    e[j] = fmaf(sg, e[j], q);
  }
}

// Persistent warps over batches of 16 vectors (one per lane pair): the next
// batch's loads are issued before the current batch is transformed, so that
// memory and arithmetic overlap.  In place is fine: a warp reads a batch
// before writing it, and batches are disjoint.
constexpr int kPrestageVPW = 16;
__device__ __forceinline__ void prestage_load(const __nv_bfloat16* __restrict__ x, int64_t v, bool live, int hh,
                                              uint4 (&raw)[8]) {
  if (!live) return;
  const uint4* src = reinterpret_cast<const uint4*>(x + v * kDI) + hh;
#pragma unroll
  for (int k = 0; k < 8; ++k) raw[k] = src[2 * k];
}

__global__ void __launch_bounds__(256, 2)
    rope_hadamard_kernel(const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ pos, int64_t n_vec,
                         int vec_per_row, const float* __restrict__ rope_cos, const float* __restrict__ rope_sin,
                         int rope_len, __nv_bfloat16* y, int32_t* status) {
  grid_dependency_wait();  // q/k may come from the previous kernel
  allow_dependents_launch();
  const int lane = threadIdx.x & 31, hh = lane & 1;
  const int64_t n_batches = (n_vec + kPrestageVPW - 1) / kPrestageVPW;
  const int64_t stride = (int64_t)gridDim.x * 8;
  int64_t bt = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  uint4 raw[8];
  int64_t v = bt * kPrestageVPW + (lane >> 1);
  prestage_load(x, v, bt < n_batches && v < n_vec, hh, raw);
  for (; bt < n_batches; bt += stride) {  // warp-uniform
    const bool live = v < n_vec;
    float e[64];
    int32_t p = 0;
    if (live) {
      p = pos[v / vec_per_row];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t w4[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[m]));
          e[8 * k + 2 * m] = f.x;
          e[8 * k + 2 * m + 1] = f.y;
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 64; ++j) e[j] = 0.f;
    }
    // the next batch's loads fly while this one is transformed
    const int64_t v_next = (bt + stride) * kPrestageVPW + (lane >> 1);
    prestage_load(x, v_next, bt + stride < n_batches && v_next < n_vec, hh, raw);
    const bool p_ok = p >= 0 && p < rope_len;
    if (live && !p_ok && hh == 0) report(status, DSA_ERR_BAD_INDEX);
    rope_hadamard128(e, p_ok ? p : 0, rope_cos, rope_sin, hh);  // every lane takes part in the shuffles
    if (live && p_ok) {
      constexpr float kScale = 0.08838834764831845f;  // 128^-1/2
      uint4* dst = reinterpret_cast<uint4*>(y + v * kDI) + hh;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        uint32_t w4[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const __nv_bfloat162 r =
              __floats2bfloat162_rn(e[8 * k + 2 * m] * kScale, e[8 * k + 2 * m + 1] * kScale);
          w4[m] = *reinterpret_cast<const uint32_t*>(&r);
        }
        dst[2 * k] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
    }
    v = v_next;
  }
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

int dsa_indexer_prestage(const void* x, const int32_t* pos, int n_rows, int vec_per_row, const float* rope_cos,
                         const float* rope_sin, int rope_len, void* y, int32_t* dev_status, void* stream) {
  if (!x || !pos || !rope_cos || !rope_sin || !y) return DSA_ERR_INVALID_ARG;
  if (n_rows <= 0 || vec_per_row <= 0 || rope_len <= 0) return DSA_ERR_INVALID_ARG;
  if ((int64_t)n_rows * vec_per_row > ((int64_t)1 << 31)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned16(rope_cos) || !aligned16(rope_sin)) return DSA_ERR_INVALID_ARG;
  const int64_t n_vec = (int64_t)n_rows * vec_per_row;
  const int64_t n_batches = (n_vec + kPrestageVPW - 1) / kPrestageVPW;  // one warp each, 8 per CTA
  const int64_t grid = std::min<int64_t>((n_batches + 7) / 8, (int64_t)device_info().sm_count * 2);
  const cudaError_t e = launch_pdl(rope_hadamard_kernel, dim3((unsigned)grid), dim3(256), 0,
                                   reinterpret_cast<cudaStream_t>(stream),
                                   reinterpret_cast<const __nv_bfloat16*>(x), pos, n_vec, vec_per_row, rope_cos,
                                   rope_sin, rope_len, reinterpret_cast<__nv_bfloat16*>(y), dev_status);
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
