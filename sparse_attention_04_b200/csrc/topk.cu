// topk.cu -- stage 2: per-query top-k selection with a fixed tie rule.
//
// "DeepSeek-V3.2-Exp - Keep top-k positions": topk(min(index_topk, end_pos))
// over the masked indexer scores, i.e. M^sel keeps each query's k
// highest-scoring positions.  This kernel returns the kept SET, ascending by
// position, padded with -1; ties are broken by lower position first and -0.0
// equals +0.0, so the result is unique and deterministic.
//
// Kernels, chosen per launch by the score pitch ld (launch_topk):
//   ld <= 8192 (causal prefill, short decode rows): topk_rows_kernel, one
//     256-thread CTA per row with the row's keys in registers (16 per thread
//     up to 4096 positions, 32 above);
//   8192 < ld <= 131072 (long decode rows): topk_cluster_kernel, one
//     thread-block cluster per row (8 CTAs of 512 threads for up to three
//     rows, 4 CTAs of 1024 threads from four rows on), each CTA holding a
//     slice of the row in shared memory;
//   ld > 131072: topk_kernel, one 1024-thread CTA per row: the bitmap path
//     below for rows of up to 131072 valid positions, exact 11/11/10-bit
//     digit passes over the whole row for longer ones.
// Scores are mapped to order-preserving 32-bit keys (larger score = larger
// key); the valid positions of a row are its causal prefix s < L = end_pos -
// T + t + 1.  Each kernel finds the k-th largest key tau and how many keys
// equal to tau are kept (the lowest positions), then writes the kept
// positions ascending.
//
// topk_kernel's bitmap path:
//   A. histogram of the top 12 key bits (shared atomics);
//      a suffix scan finds the bin d* holding the k-th largest key;
//   B. one pass marks, in a bitmap whose word w covers positions 32w..32w+31
//      (thread-owned, so no atomics), every key whose bin is above d*, and
//      copies the keys of bin d* (the candidates) into shared memory;
//   C. two digit passes over the candidates only fix the exact k-th key tau
//      and how many keys equal to tau are kept (the lowest positions, found by
//      a scan over a second bitmap);
//   D. one block scan of the words' popcounts writes the kept positions in
//      ascending order.
// Its digit-pass path (rows above 131072 positions, or more candidates than
// the buffer holds, e.g. massive ties): three 11/11/10-bit digit passes over
// the whole row and a stable scan-based compaction.
#include <cooperative_groups.h>

#include "dsa_internal.h"
#include "sm100.cuh"

namespace dsa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins12 = 4096;            // top-12-bit histogram
constexpr int kMaxWords = 4096;          // bitmap words: rows up to 131072 positions
constexpr int kWordsPerThread = kMaxWords / kThreads;
constexpr int kCap = 8192;               // candidate buffer (keys of the threshold bin)
constexpr int kFallbackSmemKeys = 2 * kMaxWords + 2 * kCap;  // the same bytes reused as keys

struct TopkSmem {
  uint32_t warp_tot[kWarps];
  uint32_t carry;
  uint32_t sel_digit;
  uint32_t sel_remaining;
  uint32_t n_cand;
  uint32_t pad[12];
  uint32_t hist[kBins12];
};
// dynamic layout after TopkSmem: bitmap[kMaxWords] | eqmap[kMaxWords] |
// cand_key[kCap] | cand_pos[kCap]   (the fallback reuses it as a key array)
constexpr size_t kSmemBytes = sizeof(TopkSmem) + sizeof(uint32_t) * (2 * kMaxWords + 2 * kCap);

// Exclusive block-wide scan of one uint32 per thread (NT threads); returns the
// thread's exclusive prefix and writes the block total to *total.
template <int NT = kThreads, class SM>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, SM& sm, uint32_t* total) {
  constexpr int NW = NT / 32;
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
    const uint32_t t = lane < NW ? sm.warp_tot[lane] : 0u;
    uint32_t ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += u;
    }
    if (lane < NW) sm.warp_tot[lane] = ti - t;  // exclusive warp offsets
    if (lane == NW - 1) sm.carry = ti;
  }
  __syncthreads();
  const uint32_t res = sm.warp_tot[warp] + incl - v;
  *total = sm.carry;
  __syncthreads();
  return res;
}

// Finds, over `nb` histogram bins in descending digit order, the bin holding
// the `remaining`-th largest element.  Writes sm.sel_digit and sm.sel_remaining
// (the rank inside that bin).  Every thread must call it.
template <int NT = kThreads, class SM>
__device__ __forceinline__ void select_bin(SM& sm, const uint32_t* hist, int nb, uint32_t remaining) {
  const int per = nb / NT;  // bins per thread, descending (at most 16)
  uint32_t c[16];
  uint32_t sum = 0;
  const int top = nb - 1 - per * (int)threadIdx.x;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    c[j] = j < per ? hist[top - j] : 0u;
    sum += c[j];
  }
  uint32_t tot;
  uint32_t above = block_excl_scan<NT>(sum, sm, &tot);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    if (j < per && above < remaining && remaining <= above + c[j]) {
      sm.sel_digit = (uint32_t)(top - j);
      sm.sel_remaining = remaining - above;
    }
    above += c[j];
  }
  __syncthreads();
}

__device__ __forceinline__ uint32_t load_key(const float* __restrict__ row, int s) {
  return float_order_key(__ldg(row + s));
}

// Keys of positions 32w .. 32w+31; bits of *valid_bits mark positions < L.
__device__ __forceinline__ void load_word(const float* __restrict__ row, int L, int w, uint32_t (&kk)[32],
                                          uint32_t* valid_bits) {
  const int s0 = 32 * w;
  if (s0 + 32 <= L) {
    const float4* p = reinterpret_cast<const float4*>(row + s0);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 v = __ldg(p + j);
      kk[4 * j + 0] = float_order_key(v.x);
      kk[4 * j + 1] = float_order_key(v.y);
      kk[4 * j + 2] = float_order_key(v.z);
      kk[4 * j + 3] = float_order_key(v.w);
    }
    *valid_bits = 0xffffffffu;
  } else {
    uint32_t vb = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const bool ok = s0 + j < L;
      kk[j] = ok ? load_key(row, s0 + j) : 0u;
      vb |= (ok ? 1u : 0u) << j;
    }
    *valid_bits = vb;
  }
}

// Keys of positions KPT*w .. KPT*w + KPT-1 (KPT = 16 or 32); bits of
// *valid_bits mark positions < L.
template <int KPT>
__device__ __forceinline__ void load_keys(const float* __restrict__ row, int L, int w, uint32_t (&kk)[KPT],
                                          uint32_t* valid_bits) {
  const int s0 = KPT * w;
  if (s0 + KPT <= L) {
    const float4* p = reinterpret_cast<const float4*>(row + s0);
#pragma unroll
    for (int j = 0; j < KPT / 4; ++j) {
      const float4 v = __ldg(p + j);
      kk[4 * j + 0] = float_order_key(v.x);
      kk[4 * j + 1] = float_order_key(v.y);
      kk[4 * j + 2] = float_order_key(v.z);
      kk[4 * j + 3] = float_order_key(v.w);
    }
    *valid_bits = KPT == 32 ? 0xffffffffu : (1u << KPT) - 1u;
  } else {
    uint32_t vb = 0;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      const bool ok = s0 + j < L;
      kk[j] = ok ? load_key(row, s0 + j) : 0u;
      vb |= (ok ? 1u : 0u) << j;
    }
    *valid_bits = vb;
  }
}

// Writes the positions of the set bits of bitmap[0 .. n_words) ascending into out.
template <class SM>
__device__ __forceinline__ void emit_bitmap(SM& sm, const uint32_t* bitmap, int n_words, int32_t* out) {
  const int w0 = threadIdx.x * kWordsPerThread;
  uint32_t cnt = 0;
  for (int j = 0; j < kWordsPerThread; ++j)
    if (w0 + j < n_words) cnt += __popc(bitmap[w0 + j]);
  uint32_t tot;
  uint32_t pos = block_excl_scan(cnt, sm, &tot);
  for (int j = 0; j < kWordsPerThread; ++j) {
    if (w0 + j >= n_words) break;
    uint32_t bits = bitmap[w0 + j];
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      out[pos++] = 32 * (w0 + j) + b;
    }
  }
}

// Three 11/11/10-bit digit passes over the whole row and a stable compaction.
template <int NT = kThreads, class SM>
__device__ void radix_select_fallback(SM& sm, uint32_t* keys, int key_cap, const float* __restrict__ row, int L,
                                      int k, int32_t* __restrict__ out) {
  const bool in_smem = L <= key_cap;
  uint32_t prefix = 0, pmask = 0, remaining = (uint32_t)k;
  uint32_t* hist = sm.hist;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nb = pass == 2 ? 1024 : 2048;
    for (int i = threadIdx.x; i < kBins12; i += NT) hist[i] = 0;
    __syncthreads();
    for (int s = threadIdx.x; s < L; s += NT) {
      uint32_t key;
      if (pass == 0) {
        key = load_key(row, s);
        if (in_smem) keys[s] = key;
      } else {
        key = in_smem ? keys[s] : load_key(row, s);
      }
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
    select_bin<NT>(sm, hist, nb, remaining);
    prefix |= sm.sel_digit << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
    remaining = sm.sel_remaining;
    __syncthreads();
  }
  const uint32_t tau = prefix, need_eq = remaining;
  constexpr int V = 8;
  uint32_t gt_carry = 0, eq_carry = 0;
#pragma unroll 1
  for (int base = 0; base < L; base += NT * V) {
    const int s0 = base + threadIdx.x * V;
    uint32_t kk[V];
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int s = s0 + j;
      kk[j] = s < L ? (in_smem ? keys[s] : load_key(row, s)) : 0u;
      gt += (s < L && kk[j] > tau);
      eq += (s < L && kk[j] == tau);
    }
    uint32_t tot;
    const uint32_t packed = block_excl_scan<NT>(gt | (eq << 16), sm, &tot);
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
}

// ============================================================================
// Short rows (ld <= kRowMaxLen: causal prefill, short decode): one CTA of
// 256 threads per row, thread t holding the keys of positions KPT*t ..
// KPT*t + KPT-1 in registers (KPT = 16 for rows of up to 4096 positions, else
// 32), so the row is read once and no candidate buffer is needed.
//   A  12-bit histogram (shared atomics) -> bin d* of the k-th largest key
//   B  two 10-bit histograms over the keys in d* (from the registers) -> the
//      exact k-th key tau and how many keys equal to tau are kept
//   C  keep every key > tau and the need_eq lowest positions equal to tau
//      (a block scan ranks the ties), then one more block scan places each
//      thread's kept positions in the ascending output.
// 16 KB of shared memory and at most 64 registers: four rows run per SM (a
// single 1024-thread CTA for a 32K-key decode row measured 8.5 us slower
// than the cluster kernel below).
constexpr int kRowThreads = 256;
constexpr int kRowMaxLen = kRowThreads * 32;
template <int NT>
struct RowSmem {
  uint32_t warp_tot[NT / 32];
  uint32_t carry;
  uint32_t sel_digit;
  uint32_t sel_remaining;
  uint32_t pad[5];
  uint32_t hist[kBins12];
};

template <int NT, int KPT>
__global__ void __launch_bounds__(NT, NT <= 256 ? 4 : 1)  // four rows per SM at 256 threads (64 registers)
    topk_rows_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ off, int B, int T,
                     int k, int32_t* __restrict__ indices, int32_t* status) {
  __shared__ RowSmem<NT> sm;
  grid_dependency_wait();  // scores come from the previous kernel
  allow_dependents_launch();
  const int r = blockIdx.x;
  const int b = r / T, t = r - (r / T) * T;
  int32_t* out = indices + (int64_t)r * k;
  const int E = off[b + 1] - off[b];
  if (E < T || (int64_t)E > ld || off[b] < 0) {
    for (int j = threadIdx.x; j < k; j += NT) out[j] = -1;
    if (threadIdx.x == 0) report(status, DSA_ERR_BAD_OFFSETS);
    return;
  }
  const int L = E - T + t + 1;  // causal prefix: every valid position (<= ld <= kRowMaxLen)
  if (L <= k) {  // every valid position is kept
    for (int j = threadIdx.x; j < k; j += NT) out[j] = j < L ? j : -1;
    return;
  }
  const float* row = scores + (int64_t)r * ld;
  const int w = threadIdx.x;
  uint32_t kk[KPT], vb = 0;  // the keys of positions KPT*w .. KPT*w + KPT-1
  if (KPT * w < L) {
    load_keys<KPT>(row, L, w, kk, &vb);
  } else {
#pragma unroll
    for (int j = 0; j < KPT; ++j) kk[j] = 0u;
  }
  for (int i = threadIdx.x; i < kBins12; i += NT) sm.hist[i] = 0;
  __syncthreads();

  // ---- A: top 12 bits
#pragma unroll
  for (int j = 0; j < KPT; ++j)
    if ((vb >> j) & 1u) atomicAdd(&sm.hist[kk[j] >> 20], 1u);
  __syncthreads();
  select_bin<NT>(sm, sm.hist, kBins12, (uint32_t)k);

  // ---- B: bits 19..10, then 9..0, of the keys sharing the prefix so far
  uint32_t prefix = sm.sel_digit << 20, pmask = 0xFFF00000u, remaining = sm.sel_remaining;
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    const int shift = pass == 0 ? 10 : 0;
    for (int i = threadIdx.x; i < 1024; i += NT) sm.hist[i] = 0;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < KPT; ++j)
      if (((vb >> j) & 1u) && (kk[j] & pmask) == prefix) atomicAdd(&sm.hist[(kk[j] >> shift) & 1023u], 1u);
    __syncthreads();
    select_bin<NT>(sm, sm.hist, 1024, remaining);
    prefix |= sm.sel_digit << shift;
    pmask |= 1023u << shift;
    remaining = sm.sel_remaining;
  }
  const uint32_t tau = prefix, need_eq = remaining;

  // ---- C: keys above tau, plus the lowest positions equal to tau
  uint32_t keep = 0, eq = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const bool valid = (vb >> j) & 1u;
    keep |= (valid && kk[j] > tau ? 1u : 0u) << j;
    eq |= (valid && kk[j] == tau ? 1u : 0u) << j;
  }
  uint32_t tot;
  uint32_t rank = block_excl_scan<NT>(__popc(eq), sm, &tot);
  while (eq && rank < need_eq) {
    const uint32_t low = eq & (0u - eq);
    keep |= low;
    eq ^= low;
    ++rank;
  }
  uint32_t pos = block_excl_scan<NT>(__popc(keep), sm, &tot);
  while (keep) {
    const int j = __ffs(keep) - 1;
    keep &= keep - 1;
    out[pos++] = KPT * w + j;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    topk_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ off,
                int B, int T, int k, int32_t* __restrict__ indices, int32_t* status) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(smem_raw);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem_raw + sizeof(TopkSmem));
  uint32_t* eqmap = bitmap + kMaxWords;
  uint32_t* cand_key = eqmap + kMaxWords;
  uint32_t* cand_pos = cand_key + kCap;

  grid_dependency_wait();  // scores come from the previous kernel
  allow_dependents_launch();
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
  if (L > kMaxWords * 32) {
    radix_select_fallback(sm, bitmap, kFallbackSmemKeys, row, L, k, out);
    return;
  }

  const int n_words = (L + 31) >> 5;
  for (int i = threadIdx.x; i < kBins12; i += kThreads) sm.hist[i] = 0;
  if (threadIdx.x == 0) sm.n_cand = 0;
  __syncthreads();

  // ---- A: histogram of the top 12 bits
  auto hist_word = [&](const uint32_t (&kk)[32], uint32_t vb) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if ((vb >> j) & 1u) atomicAdd(&sm.hist[kk[j] >> 20], 1u);
  };
#pragma unroll 1
  for (int i = 0; i < kWordsPerThread; ++i) {
    const int w = threadIdx.x + i * kThreads;
    if (w >= n_words) break;
    uint32_t kk[32], vb = 0;
    load_word(row, L, w, kk, &vb);
    hist_word(kk, vb);
  }
  __syncthreads();
  select_bin(sm, sm.hist, kBins12, (uint32_t)k);
  const uint32_t dstar = sm.sel_digit;
  const uint32_t need_in_bin = sm.sel_remaining;  // how many keys of bin d* are kept

  // ---- B: bitmap of keys above bin d*, candidates of bin d*
#pragma unroll 1
  for (int i = 0; i < kWordsPerThread; ++i) {
    const int w = threadIdx.x + i * kThreads;
    if (w >= n_words) break;
    uint32_t kk[32], vb;
    load_word(row, L, w, kk, &vb);  // second read of the row: it is in L2
    uint32_t bits = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const uint32_t bin = kk[j] >> 20;
      if ((vb >> j) & 1u) {
        if (bin > dstar) {
          bits |= 1u << j;
        } else if (bin == dstar) {
          const uint32_t slot = atomicAdd(&sm.n_cand, 1u);
          if (slot < kCap) {
            cand_key[slot] = kk[j];
            cand_pos[slot] = 32 * w + j;
          }
        }
      }
    }
    bitmap[w] = bits;
    eqmap[w] = 0;
  }
  __syncthreads();
  const uint32_t n_cand = sm.n_cand;
  if (n_cand > kCap) {  // too many keys share the threshold bin: exact slow path
    radix_select_fallback(sm, bitmap, kFallbackSmemKeys, row, L, k, out);
    return;
  }

  // ---- C: exact threshold among the candidates (low 20 bits: 10 + 10)
  uint32_t prefix = dstar << 20, pmask = 0xFFF00000u, remaining = need_in_bin;
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    const int shift = pass == 0 ? 10 : 0;
    for (int i = threadIdx.x; i < 1024; i += kThreads) sm.hist[i] = 0;
    __syncthreads();
    for (uint32_t c = threadIdx.x; c < n_cand; c += kThreads) {
      const uint32_t key = cand_key[c];
      if ((key & pmask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 1023u], 1u);
    }
    __syncthreads();
    select_bin(sm, sm.hist, 1024, remaining);
    prefix |= sm.sel_digit << shift;
    pmask |= 1023u << shift;
    remaining = sm.sel_remaining;
    __syncthreads();
  }
  const uint32_t tau = prefix, need_eq = remaining;
  for (uint32_t c = threadIdx.x; c < n_cand; c += kThreads) {
    const uint32_t key = cand_key[c], s = cand_pos[c];
    if (key > tau) atomicOr(&bitmap[s >> 5], 1u << (s & 31));
    else if (key == tau) atomicOr(&eqmap[s >> 5], 1u << (s & 31));
  }
  __syncthreads();
  // keep the need_eq lowest positions whose key equals tau
  {
    const int w0 = threadIdx.x * kWordsPerThread;
    uint32_t cnt = 0;
    for (int j = 0; j < kWordsPerThread; ++j)
      if (w0 + j < n_words) cnt += __popc(eqmap[w0 + j]);
    uint32_t tot;
    uint32_t rank = block_excl_scan(cnt, sm, &tot);
    for (int j = 0; j < kWordsPerThread; ++j) {
      if (w0 + j >= n_words) break;
      uint32_t bits = eqmap[w0 + j], keep = 0;
      while (bits && rank < need_eq) {
        const uint32_t low = bits & (0u - bits);
        keep |= low;
        bits ^= low;
        ++rank;
      }
      if (keep) bitmap[w0 + j] |= keep;
    }
  }
  __syncthreads();
  // ---- D: ascending output (exactly k positions: L > k here)
  emit_bitmap(sm, bitmap, n_words, out);
}


// ============================================================================
// Cluster variant for long rows: CS CTAs (one thread-block cluster) per row,
// each owning a contiguous, word-aligned slice of positions.  Two cluster
// barriers in all:
//   1  every CTA loads its slice (keys kept in shared memory), builds the
//      12-bit histogram of its keys and 64 coarse sums of 64 bins each
//   -- barrier 1 --
//   2  every CTA reads the coarse sums of all CTAs, then the 64 fine bins of
//      the coarse bin holding the k-th largest key (distributed shared
//      memory), and so finds bin d* and the count of keys above it -- the
//      same answer in every CTA
//   3  every CTA marks its keys above bin d* in a bitmap and sends its keys
//      in bin d* (the candidates), their count and its above-count to every
//      CTA of the cluster
//   -- barrier 2 --
//   4  every CTA fixes the exact threshold tau over all candidates and its
//      own output offset and tie quota, then writes its kept positions.
// If any CTA has more candidates than its send buffer holds (massive ties),
// rank 0 redoes the row with the exact digit-pass fallback.
template <int CS>
struct ClusterCfg {
  static constexpr int kThreads = CS >= 8 ? 512 : 1024;
  static constexpr int kWarps = kThreads / 32;
  static constexpr int kSliceMax = 131072 / CS;          // positions per CTA
  static constexpr int kSliceWords = kSliceMax / 32;
  static constexpr int kPerSrc = 4096 / CS;                // candidates a CTA may send (107 KB in all: two CTAs per SM)
  static_assert(kSliceWords <= kThreads, "one bitmap word per thread");
  static_assert(CS <= kWarps && CS <= 32 && 32 % CS == 0, "per-source counting and lane groups");
};

template <int CS>
struct ClusterSmem {
  using C = ClusterCfg<CS>;
  uint32_t warp_tot[32];
  uint32_t carry, sel_digit, sel_remaining, n_cand;
  uint32_t above_local, mode, J, aboveJ;
  uint32_t all_coarse[CS][64];         // every CTA's coarse sums (pushed before barrier 1)
  uint32_t tot_coarse[64];             // cluster-wide coarse sums
  uint32_t tot_fine[64];               // cluster-wide fine bins of the chosen coarse bin
  uint32_t g_cnt[CS], g_above[CS];     // from every CTA: candidate count, keys above d*
  uint32_t c_gt[CS], c_eq[CS];         // per source: candidates above / equal to tau
  uint32_t hist[kBins12];              // 12-bit histogram of this slice, later scratch
  uint32_t bitmap[C::kSliceWords];
  uint32_t eqmap[C::kSliceWords];
  uint32_t cand_key[C::kPerSrc];
  uint32_t cand_pos[C::kPerSrc];
  alignas(16) uint32_t keys[C::kSliceMax];  // written as uint4
  uint32_t g_key[CS][C::kPerSrc];      // candidates from every CTA
};

// Over 64 bins in descending bin order (bins[63] first), finds the bin that
// holds the `need`-th largest element.  One warp; every lane gets the answer.
__device__ __forceinline__ void warp_select64(const uint32_t* bins, uint32_t need, int lane, int* bin,
                                              uint32_t* above) {
  const uint32_t c0 = bins[63 - lane], c1 = bins[31 - lane];
  uint32_t i0 = c0, i1 = c1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u0 = __shfl_up_sync(0xffffffffu, i0, o), u1 = __shfl_up_sync(0xffffffffu, i1, o);
    if (lane >= o) {
      i0 += u0;
      i1 += u1;
    }
  }
  i1 += __shfl_sync(0xffffffffu, i0, 31);
  const unsigned b0 = __ballot_sync(0xffffffffu, i0 >= need);
  const unsigned b1 = __ballot_sync(0xffffffffu, i1 >= need);
  int d;
  uint32_t ab;
  if (b0) {
    d = __ffs(b0) - 1;
    ab = __shfl_sync(0xffffffffu, i0 - c0, d);
  } else if (b1) {
    const int l = __ffs(b1) - 1;
    d = 32 + l;
    ab = __shfl_sync(0xffffffffu, i1 - c1, l);
  } else {  // fewer elements than need: cannot happen for L > k; take the lowest bin
    d = 63;
    ab = __shfl_sync(0xffffffffu, i1 - c1, 31);
  }
  *bin = 63 - d;
  *above = ab;
}

template <int CS>
__global__ void __launch_bounds__(ClusterCfg<CS>::kThreads, ClusterCfg<CS>::kThreads == 512 ? 2 : 1)
    topk_cluster_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ off, int B,
                        int T, int k, int32_t* __restrict__ indices, int32_t* status) {
  using Cfg = ClusterCfg<CS>;
  constexpr int NT = Cfg::kThreads;
  constexpr uint32_t kPerSrc = Cfg::kPerSrc;
  constexpr int BPT = kBins12 / NT, TPC = 64 / BPT;  // fine bins per thread, threads per coarse bin
  static_assert(BPT * NT == kBins12 && TPC <= 32, "coarse sums");
  static_assert(offsetof(ClusterSmem<CS>, keys) % 16 == 0, "16-byte key stores");
  namespace cg = cooperative_groups;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  ClusterSmem<CS>& sm = *reinterpret_cast<ClusterSmem<CS>*>(smem_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  grid_dependency_wait();  // scores come from the previous kernel
  allow_dependents_launch();
  const int r = blockIdx.x / CS;
  const int b = r / T, t = r - (r / T) * T;
  int32_t* out = indices + (int64_t)r * k;
  const int E = off[b + 1] - off[b];
  if (E < T || (int64_t)E > ld || off[b] < 0) {  // same verdict in every CTA of the cluster
    if (rank == 0) {
      for (int j = threadIdx.x; j < k; j += NT) out[j] = -1;
      if (threadIdx.x == 0) report(status, DSA_ERR_BAD_OFFSETS);
    }
    return;
  }
  const int L = E - T + t + 1;
  const float* row = scores + (int64_t)r * ld;
  if (L <= k) {
    if (rank == 0)
      for (int j = threadIdx.x; j < k; j += NT) out[j] = j < L ? j : -1;
    return;
  }
  // slice of this CTA, word aligned (the host sends only rows of <= 131072 positions here)
  const int S = (((L + CS - 1) / CS) + 31) & ~31;
  const int s_lo = min(rank * S, L), s_hi = min(s_lo + S, L);
  const int n = s_hi - s_lo;
  const int n_words = (n + 31) >> 5;
  cluster_arrive_relaxed();  // "started"; waited for before the first remote store

  // ---- 1: keys and 12-bit histogram of the slice, coarse sums
  for (int i = threadIdx.x; i < kBins12; i += NT) sm.hist[i] = 0;
  if (threadIdx.x == 0) {
    sm.n_cand = 0;
    sm.above_local = 0;
  }
  __syncthreads();
  {
    const float4* r4 = reinterpret_cast<const float4*>(row + s_lo);  // s_lo is a multiple of 32
    uint4* k4 = reinterpret_cast<uint4*>(sm.keys);
    const int n4 = n >> 2;
    for (int i4 = threadIdx.x; i4 < n4; i4 += NT) {
      const float4 v = __ldg(r4 + i4);
      const uint4 kk = make_uint4(float_order_key(v.x), float_order_key(v.y), float_order_key(v.z),
                                  float_order_key(v.w));
      k4[i4] = kk;
      atomicAdd(&sm.hist[kk.x >> 20], 1u);
      atomicAdd(&sm.hist[kk.y >> 20], 1u);
      atomicAdd(&sm.hist[kk.z >> 20], 1u);
      atomicAdd(&sm.hist[kk.w >> 20], 1u);
    }
    for (int s = 4 * n4 + threadIdx.x; s < n; s += NT) {
      const uint32_t key = float_order_key(__ldg(row + s_lo + s));
      sm.keys[s] = key;
      atomicAdd(&sm.hist[key >> 20], 1u);
    }
  }
  __syncthreads();
  {
    uint32_t v = 0;
#pragma unroll
    for (int j = 0; j < BPT; ++j) v += sm.hist[BPT * threadIdx.x + j];
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    if (TPC > 8) v += __shfl_xor_sync(0xffffffffu, v, 8);
    // every lane of the TPC-lane group now holds coarse sum c = tid/TPC; the
    // group pushes it to all CTAs, lane i of the group to CTAs i, i+TPC, ...
    const uint32_t c = threadIdx.x / TPC;
    cluster_wait();
#pragma unroll
    for (int i = 0; i < (CS + TPC - 1) / TPC; ++i) {
      const int q = (lane % TPC) + TPC * i;
      if (q < CS) cluster.map_shared_rank(&sm, q)->all_coarse[rank][c] = v;
    }
  }
  cluster.sync();  // 1: every histogram is complete and every coarse sum delivered

  // ---- 2: bin d* from the cluster-wide histogram (the same in every CTA).
  if (threadIdx.x < 64) {
    uint32_t v = 0;
#pragma unroll
    for (int q = 0; q < CS; ++q) v += sm.all_coarse[q][threadIdx.x];
    sm.tot_coarse[threadIdx.x] = v;
  }
  __syncthreads();
  if (warp == 0) {
    int J;
    uint32_t ab;
    warp_select64(sm.tot_coarse, (uint32_t)k, lane, &J, &ab);
    if (lane == 0) {
      sm.J = (uint32_t)J;
      sm.aboveJ = ab;
    }
  }
  __syncthreads();
  const uint32_t J = sm.J, aboveJ = sm.aboveJ;
  {  // the 64 fine bins of coarse bin J from every CTA: entry e = j * CS + q;
     // a thread issues all its remote loads before it uses any
    constexpr int PER = (64 * CS + NT - 1) / NT;
    uint32_t v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = threadIdx.x + i * NT;
      v[i] = e < 64 * CS ? cluster.map_shared_rank(sm.hist, e % CS)[64 * J + e / CS] : 0u;
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = threadIdx.x + i * NT;
      uint32_t x = v[i];
#pragma unroll
      for (int o = CS / 2; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      if (e < 64 * CS && e % CS == 0) sm.tot_fine[e / CS] = x;
    }
  }
  __syncthreads();
  if (warp == 0) {
    int jf;
    uint32_t ab;
    warp_select64(sm.tot_fine, (uint32_t)k - aboveJ, lane, &jf, &ab);
    if (lane == 0) {
      sm.sel_digit = 64 * J + (uint32_t)jf;
      sm.sel_remaining = (uint32_t)k - aboveJ - ab;
    }
  }
  __syncthreads();
  const uint32_t dstar = sm.sel_digit;
  const uint32_t need_in_bin = sm.sel_remaining;  // keys of bin d* that are kept (>= 1)

  // ---- 3: bitmap of keys above d*, candidates in d*, sent to every CTA
  {
    uint32_t above = 0;
    for (int w = warp; w < n_words; w += Cfg::kWarps) {
      const int s = 32 * w + lane;
      const bool valid = s < n;
      const uint32_t key = valid ? sm.keys[s] : 0u;
      const uint32_t bin = key >> 20;
      const uint32_t up = __ballot_sync(0xffffffffu, valid && bin > dstar);
      const uint32_t cand = __ballot_sync(0xffffffffu, valid && bin == dstar);
      if (cand) {
        uint32_t base = 0;
        if (lane == 0) base = atomicAdd(&sm.n_cand, (uint32_t)__popc(cand));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (valid && bin == dstar) {
          const uint32_t slot = base + __popc(cand & ((1u << lane) - 1u));
          if (slot < kPerSrc) {
            sm.cand_key[slot] = key;
            sm.cand_pos[slot] = (uint32_t)s;
          }
        }
      }
      if (lane == 0) {
        sm.bitmap[w] = up;
        sm.eqmap[w] = 0;
      }
      above += __popc(up);
    }
    for (int w = n_words + threadIdx.x; w < Cfg::kSliceWords; w += NT) {
      sm.bitmap[w] = 0;
      sm.eqmap[w] = 0;
    }
    if (lane == 0 && above) atomicAdd(&sm.above_local, above);
    __syncthreads();
    const uint32_t nc = sm.n_cand;
    const bool fits = nc <= kPerSrc;
    if (fits) {  // warp w sends to CTA w % CS, the warps of a destination splitting the list
      constexpr int WPD = Cfg::kWarps / CS;
      uint32_t* dst = cluster.map_shared_rank(&sm, warp % CS)->g_key[rank];
      for (uint32_t c = lane + 32 * (warp / CS); c < nc; c += 32 * WPD) dst[c] = sm.cand_key[c];
    }
    if (threadIdx.x < CS) {
      ClusterSmem<CS>* dst = cluster.map_shared_rank(&sm, (int)threadIdx.x);
      dst->g_cnt[rank] = fits ? nc : 0xFFFFFFFFu;  // overflow marker
      dst->g_above[rank] = sm.above_local;
    }
  }
  cluster.sync();  // 2: no remote shared-memory access after this point

  // ---- 4: exact threshold tau over every candidate, this CTA's offsets, output
  {
    bool bad = false;
#pragma unroll
    for (int q = 0; q < CS; ++q) bad |= sm.g_cnt[q] == 0xFFFFFFFFu;
    if (bad) {  // a CTA had too many keys in bin d*: rank 0 redoes the row alone
      if (rank == 0) radix_select_fallback<NT>(sm, sm.keys, Cfg::kSliceMax, row, L, k, out);
      return;
    }
  }
  constexpr int WPS = Cfg::kWarps / CS;  // warps per source CTA
  const int src = warp % CS;
  const uint32_t src_cnt = sm.g_cnt[src];
  uint32_t prefix = dstar << 20, pmask = 0xFFF00000u, remaining = need_in_bin;
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    const int shift = pass == 0 ? 10 : 0;
    for (int i = threadIdx.x; i < 1024; i += NT) sm.hist[i] = 0;
    __syncthreads();
    for (uint32_t c = lane + 32 * (warp / CS); c < src_cnt; c += 32 * WPS) {
      const uint32_t key = sm.g_key[src][c];
      if ((key & pmask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 1023u], 1u);
    }
    __syncthreads();
    select_bin<NT>(sm, sm.hist, 1024, remaining);
    prefix |= sm.sel_digit << shift;
    pmask |= 1023u << shift;
    remaining = sm.sel_remaining;
    __syncthreads();
  }
  const uint32_t tau = prefix, need_eq = remaining;
  if (threadIdx.x < CS) {
    sm.c_gt[threadIdx.x] = 0;
    sm.c_eq[threadIdx.x] = 0;
  }
  __syncthreads();
  {  // per source: candidates above and equal to tau
    uint32_t gt = 0, eq = 0;
    for (uint32_t c = lane + 32 * (warp / CS); c < src_cnt; c += 32 * WPS) {
      const uint32_t key = sm.g_key[src][c];
      gt += key > tau;
      eq += key == tau;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      gt += __shfl_xor_sync(0xffffffffu, gt, o);
      eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    if (lane == 0 && (gt | eq)) {
      atomicAdd(&sm.c_gt[src], gt);
      atomicAdd(&sm.c_eq[src], eq);
    }
  }
  __syncthreads();
  uint32_t out_base = 0, eq_base = 0;  // what the lower slices keep
  for (int q = 0; q < rank; ++q) {
    const uint32_t taken = eq_base >= need_eq ? 0u : min(sm.c_eq[q], need_eq - eq_base);
    eq_base += sm.c_eq[q];
    out_base += sm.g_above[q] + sm.c_gt[q] + taken;
  }
  for (uint32_t c = threadIdx.x; c < sm.n_cand; c += NT) {
    const uint32_t key = sm.cand_key[c], s = sm.cand_pos[c];
    if (key > tau) atomicOr(&sm.bitmap[s >> 5], 1u << (s & 31));
    else if (key == tau) atomicOr(&sm.eqmap[s >> 5], 1u << (s & 31));
  }
  __syncthreads();
  {  // one scan gives, per bitmap word, the kept keys above tau and the keys
     // equal to tau before it; equal keys are kept in position order while
     // their rank over the whole row is below need_eq
    const int w = threadIdx.x;
    const uint32_t up = w < Cfg::kSliceWords ? sm.bitmap[w] : 0u;
    uint32_t eqb = w < Cfg::kSliceWords ? sm.eqmap[w] : 0u;
    uint32_t tot;
    const uint32_t packed = block_excl_scan<NT>((uint32_t)__popc(up) | ((uint32_t)__popc(eqb) << 16), sm, &tot);
    uint32_t rk = eq_base + (packed >> 16);  // rank of this word's first equal key
    const uint32_t quota = need_eq > eq_base ? need_eq - eq_base : 0u;
    const uint32_t eq_kept_before = min(packed >> 16, quota);
    uint32_t keep = 0;
    while (eqb && rk < need_eq) {
      const uint32_t low = eqb & (0u - eqb);
      keep |= low;
      eqb ^= low;
      ++rk;
    }
    uint32_t bits = up | keep;
    uint32_t pos = out_base + (packed & 0xFFFFu) + eq_kept_before;
    while (bits) {
      const int bb = __ffs(bits) - 1;
      bits &= bits - 1;
      out[pos++] = s_lo + 32 * w + bb;
    }
  }
}

template <int CS>
int launch_cluster(const TopkArgs& a, cudaStream_t stream) {
  auto kern = topk_cluster_kernel<CS>;
  const size_t smem = sizeof(ClusterSmem<CS>);
  static PerDeviceOnce attrs_set;  // per template instance
  if (attrs_set.run([&] {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess && CS > 8) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        return e;
      }) != cudaSuccess)
    return DSA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.B * a.T * CS));
  cfg.blockDim = dim3(ClusterCfg<CS>::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a.scores, a.ld, a.offsets, a.B, a.T, a.k, a.indices,
                                           a.status);
  return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace

// Rows longer than kClusterMinLd positions go to the cluster kernel: 8 CTAs
// of 512 threads per row for up to three rows (a single 32K row: 27.3 us per
// decode step against 28.3 with 16 CTAs and 27.9 with 4), 4 CTAs of 1024
// threads per row from four rows on (four 131K rows: 47.0 against 47.7 us;
// 32 rows: 178 against 182 us).  Shorter rows (prefill) take one CTA each.
#ifndef DSA_TOPK_CLUSTER_MIN_LD
#define DSA_TOPK_CLUSTER_MIN_LD 8192
#endif

int launch_topk(const TopkArgs& a, cudaStream_t stream) {
  const int rows = a.B * a.T;
  if (a.ld > DSA_TOPK_CLUSTER_MIN_LD && a.ld <= 131072)
    return rows >= 4 ? launch_cluster<4>(a, stream) : launch_cluster<8>(a, stream);
  if (a.ld <= kRowMaxLen) {
    // rows of up to 4096 positions: 16 keys per thread, so every thread has work
    const cudaError_t e = launch_pdl(a.ld <= kRowThreads * 16 ? topk_rows_kernel<kRowThreads, 16>
                                                              : topk_rows_kernel<kRowThreads, 32>,
                                     dim3(rows), dim3(kRowThreads), 0, stream,
                                     a.scores, a.ld, a.offsets, a.B, a.T, a.k, a.indices, a.status);
    return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
  }
  static PerDeviceOnce attr;
  if (attr.run([] { return cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes); }) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  const cudaError_t e = launch_pdl(topk_kernel, dim3(rows), dim3(kThreads), kSmemBytes, stream, a.scores,
                                   a.ld, a.offsets, a.B, a.T, a.k, a.indices, a.status);
  return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
