// topk.cu -- stage 2: per-query top-k selection with a fixed tie rule.
//
// "DeepSeek-V3.2-Exp - Keep top-k positions": topk(min(index_topk, end_pos))
// over the masked indexer scores, i.e. M^sel keeps each query's k
// highest-scoring positions.  This kernel returns the kept SET, ascending by
// position, padded with -1; ties are broken by lower position first and -0.0
// equals +0.0, so the result is unique and deterministic.
//
// One CTA (1024 threads) per query row.  The valid positions of a row are the
// causal prefix s < L = min(end_pos, start + t + 1).  Algorithm:
//   1. map every score to an order-preserving 32-bit key (larger = better);
//   2. radix-select the k-th largest key tau with three digit passes
//      (11, 11, 10 bits, most significant first) over shared-memory
//      histograms, narrowing to the elements that share the digits found;
//   3. one stable compaction pass in position order keeps every key > tau and
//      the first (k - #greater) keys == tau, writing positions ascending.
// Keys stay in shared memory when the row fits (<= kSmemKeys), else each pass
// re-reads the scores (they were just written and sit in L2).
#include "dsa_internal.h"
#include "sm100.cuh"

namespace dsa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kSmemKeys = 48 * 1024;  // 192 KiB of keys

struct TopkSmem {
  uint32_t hist[kBins];
  uint32_t warp_tot[kWarps];
  uint32_t sel_digit;
  uint32_t sel_remaining;
  uint32_t carry;
  uint32_t pad;
};

// Exclusive block-wide scan of one uint32 per thread; returns the thread's
// exclusive prefix and writes the block total to *total.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, TopkSmem& sm, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) sm.warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = sm.warp_tot[lane];
    uint32_t ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += u;
    }
    sm.warp_tot[lane] = ti - t;  // exclusive warp offsets
    if (lane == 31) sm.carry = ti;
  }
  __syncthreads();
  const uint32_t res = sm.warp_tot[warp] + incl - v;
  *total = sm.carry;
  __syncthreads();
  return res;
}

__device__ __forceinline__ uint32_t load_key(const float* __restrict__ row, const uint32_t* keys,
                                             bool in_smem, int s) {
  return in_smem ? keys[s] : float_order_key(__ldg(row + s));
}

__global__ void __launch_bounds__(kThreads, 1)
    topk_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ off,
                int B, int T, int k, int32_t* __restrict__ indices, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + sizeof(TopkSmem));

  const int r = blockIdx.x;
  const int b = r / T, t = r - (r / T) * T;
  int32_t* out = indices + (int64_t)r * k;
  const int E = off[b + 1] - off[b];
  if (E < T || (int64_t)E > ld || off[b] < 0) {
    for (int j = threadIdx.x; j < k; j += kThreads) out[j] = -1;
    if (threadIdx.x == 0) report(status, DSA_ERR_BAD_OFFSETS);
    return;
  }
  const int L = E - T + t + 1;  // causal prefix: every valid position
  const float* row = scores + (int64_t)r * ld;

  if (L <= k) {  // every valid position is kept
    for (int j = threadIdx.x; j < k; j += kThreads) out[j] = j < L ? j : -1;
    return;
  }

  const bool in_smem = L <= kSmemKeys;
  // ---- digit passes
  uint32_t prefix = 0, pmask = 0, remaining = (uint32_t)k;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass];
    const uint32_t nb = 1u << widths[pass];
    for (int i = threadIdx.x; i < kBins; i += kThreads) sm.hist[i] = 0;
    __syncthreads();
    if (pass == 0 && in_smem) {
      for (int s = threadIdx.x; s < L; s += kThreads) {
        const uint32_t key = float_order_key(__ldg(row + s));
        keys[s] = key;
        atomicAdd(&sm.hist[key >> shift], 1u);
      }
    } else {
      for (int s = threadIdx.x; s < L; s += kThreads) {
        const uint32_t key = load_key(row, keys, in_smem, s);
        if ((key & pmask) == prefix) atomicAdd(&sm.hist[(key >> shift) & (nb - 1)], 1u);
      }
    }
    __syncthreads();
    // Bins in descending digit order: thread i owns digits nb-1-2i and nb-2-2i
    // (nb/2 <= 1024 threads cover them all).
    const int d_hi = (int)nb - 1 - 2 * (int)threadIdx.x;
    const uint32_t c_hi = d_hi >= 0 ? sm.hist[d_hi] : 0u;
    const uint32_t c_lo = d_hi - 1 >= 0 ? sm.hist[d_hi - 1] : 0u;
    uint32_t tot;
    const uint32_t above = block_excl_scan(c_hi + c_lo, sm, &tot);
    if (d_hi >= 0) {
      if (above < remaining && remaining <= above + c_hi) {
        sm.sel_digit = (uint32_t)d_hi;
        sm.sel_remaining = remaining - above;
      } else if (d_hi - 1 >= 0 && above + c_hi < remaining && remaining <= above + c_hi + c_lo) {
        sm.sel_digit = (uint32_t)(d_hi - 1);
        sm.sel_remaining = remaining - above - c_hi;
      }
    }
    __syncthreads();
    prefix |= sm.sel_digit << shift;
    pmask |= (nb - 1) << shift;
    remaining = sm.sel_remaining;
    __syncthreads();
  }
  const uint32_t tau = prefix;
  const uint32_t need_eq = remaining;  // keys equal to tau to keep, lowest positions first

  // ---- stable compaction in position order
  constexpr int V = 8;  // positions per thread per tile
  uint32_t gt_carry = 0, eq_carry = 0;
#pragma unroll 1
  for (int base = 0; base < L; base += kThreads * V) {
    const int s0 = base + threadIdx.x * V;
    uint32_t kk[V];
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int s = s0 + j;
      kk[j] = s < L ? load_key(row, keys, in_smem, s) : 0u;
      gt += (s < L && kk[j] > tau);
      eq += (s < L && kk[j] == tau);
    }
    uint32_t tot;
    const uint32_t packed = block_excl_scan(gt | (eq << 16), sm, &tot);
    uint32_t g = gt_carry + (packed & 0xFFFFu);
    uint32_t q = eq_carry + (packed >> 16);
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int s = s0 + j;
      if (s >= L) break;
      if (kk[j] > tau) {
        out[g + min(q, need_eq)] = s;
        ++g;
      } else if (kk[j] == tau) {
        if (q < need_eq) out[g + q] = s;
        ++q;
      }
    }
    gt_carry += tot & 0xFFFFu;
    eq_carry += tot >> 16;
  }
  for (int j = threadIdx.x; j < k; j += kThreads)
    if (j >= k) out[j] = -1;  // k_eff == k whenever L > k: nothing to pad
}

}  // namespace

int launch_topk(const TopkArgs& a, cudaStream_t stream) {
  const size_t smem = sizeof(TopkSmem) + sizeof(uint32_t) * kSmemKeys;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return DSA_ERR_CUDA;
    attr_set = true;
  }
  const int rows = a.B * a.T;
  topk_kernel<<<rows, kThreads, smem, stream>>>(a.scores, a.ld, a.offsets, a.B, a.T, a.k, a.indices,
                                               a.status);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
