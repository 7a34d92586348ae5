// indexer.cu -- stage 1: lightning-indexer scores on the tcgen05 tensor core.
//
// I[t,s] = sum_h w[t,h] * ReLU(q_I[t,h,:] . k_I[s,:])  (+ causal mask)
// ("DeepSeek-V3.2-Exp - Keep top-k positions", Indexer.forward: the fp8_index
// call and "index_score += mask"; the sum over heads is the fix of
// "[WIP] deepseek v32", mlx-lm PR #512.)
//
// Orientation: keys on the MMA's M (128 TMEM lanes), (query, head) pairs on N.
// One tile = 128 keys x NQ queries x 64 heads, K = 128:
//     D[key, q*64+h] = k_I[key,:] . q_I[q,h,:]
// so every epilogue thread owns one key (one TMEM lane) and forms
// sum_h w * max(0, D) from its own registers -- no cross-lane reduction.
//
// Roles (persistent CTAs, each over a balanced range of a flat list of
// (sequence, query block, key tile) items):
//   epilogue warps  TMEM -> registers, ReLU, weight, head sum, mask, store
//                   (4 warps for decode; 8 for prefill, two per TMEM lane
//                   quarter, each taking half of the block's queries)
//   producer warp   TMA: key tiles into a ring of stages, query blocks into
//                   two slots (reloaded only when the query block changes)
//   MMA warp        TMEM allocator + MMA issuer (one thread)
//   fill warp       prefill only: -inf past each row's causal frontier, where
//                   no tile is multiplied (its stores would otherwise delay
//                   the producer's next load)
// Key tiles and query blocks land in shared memory in the 128-byte-swizzled
// K-major layout the MMA descriptors describe; accumulators are double
// buffered in TMEM so the epilogue of tile i overlaps the MMA of tile i+1.
// The work split charges every query block one extra unit on top of its
// tiles (prefill), for its query reload and pipeline restart.
#include <cuda.h>

#include "dsa_internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace dsa {
namespace {

template <int NQ, bool FP8>
struct IdxCfg {
  static constexpr int N = 64 * NQ;                  // MMA N: (query, head) pairs
  static constexpr int ROWB = FP8 ? 128 : 256;       // bytes of one 128-dim vector
  static constexpr int BOXES = ROWB / 128;           // 128-byte swizzle columns per vector
  static constexpr int KT_BYTES = 128 * ROWB;        // one 128-key tile
  static constexpr int Q_BYTES = N * ROWB;           // one query block
  static constexpr int KSTEPS = ROWB / 32;           // MMAs per tile (K = 32 bytes each)
  // Decode (NQ = 1) runs two CTAs per SM with a short ring each, so a 32K-key
  // row spreads over 2x148 CTAs; prefill keeps one CTA per SM.
  static constexpr int CTAS_PER_SM = NQ == 1 ? 2 : 1;
  static constexpr int KSTAGES = NQ == 1 ? (FP8 ? 4 : 2) : (FP8 ? 8 : 2);
  static constexpr int QSLOTS = 2;
  static constexpr int EPI_WARPS = NQ == 1 ? 4 : 8;
  static constexpr int QPW = NQ * 4 / EPI_WARPS;     // queries per epilogue warp
  static constexpr int SEG_COST = NQ == 1 ? 0 : 1;   // balance units per query block
  static constexpr int PRODUCER = EPI_WARPS;         // warp indices of the other roles
  static constexpr int MMA_WARP = EPI_WARPS + 1;
  static constexpr int FILL_WARP = EPI_WARPS + 2;    // prefill only: -inf past the causal frontier
  static constexpr int ROLE_WARPS = NQ == 1 ? 2 : 3;
  // TMEM accumulators: two for decode (two CTAs share an SM), else as many as
  // 512 columns hold, so the epilogue's TMEM reads have slack behind the MMA.
  static constexpr int NACC = NQ == 1 ? 2 : 512 / N;
  static constexpr int TMEM_COLS = NACC * N;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_Q = OFF_K + KSTAGES * KT_BYTES;
  static constexpr int OFF_W = OFF_Q + QSLOTS * Q_BYTES;
  // e4m3: a ring of key scales per epilogue thread, fetched KSC_AHEAD tiles
  // ahead by cp.async
  static constexpr int KSC_AHEAD = 4;
  static constexpr int OFF_KSC = OFF_W + 2 * N * 4;
  static constexpr int KSC_BYTES = FP8 ? KSC_AHEAD * EPI_WARPS * 32 * 4 : 0;
  static constexpr int OFF_BAR = OFF_KSC + KSC_BYTES;
  static constexpr int NBAR = 2 * KSTAGES + 2 * QSLOTS + 2 * NACC;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // The swizzled tiles need 1 KiB alignment.  Where the budget allows, 1 KiB
  // of slack lets the kernel align the base itself; otherwise (the bf16
  // prefill ring) it relies on the dynamic shared memory base being 1 KiB
  // aligned and reports DSA_ERR_UNSUPPORTED, without touching memory, if not.
  static constexpr int USED_BYTES = OFF_MISC + 64;
  static constexpr bool SLACK = USED_BYTES + 1024 <= 232448;
  static constexpr int SMEM_BYTES = USED_BYTES + (SLACK ? 1024 : 0);
  static constexpr int THREADS = 32 * (EPI_WARPS + ROLE_WARPS);
  static_assert(NQ % (EPI_WARPS / 4) == 0, "queries split evenly over the warps of a lane quarter");
  static_assert(N <= 256, "MMA N limit");
  static_assert(OFF_Q % 1024 == 0 && OFF_W % 1024 == 0, "swizzle atoms need 1 KiB alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(CTAS_PER_SM == 1 || SMEM_BYTES * CTAS_PER_SM <= 228 * 1024 - 2048, "two CTAs per SM");
};

// Number of 128-key tiles the query block `qb` of sequence b must score: the
// block's last query sees keys [0, start + t_last].
template <int NQ>
__device__ __forceinline__ int seg_len(const int32_t* __restrict__ off, int T, int QB, int seg) {
  const int b = seg / QB, qb = seg - (seg / QB) * QB;
  const int E = off[b + 1] - off[b];
  const int t_last = min(T, (qb + 1) * NQ) - 1;
  const int L = E - T + t_last + 1;
  return (L + 127) >> 7;
}

struct SmemMisc {
  int abort, tmem_base, pad[14];
};

// 64-head weighted ReLU sum of one key for one query: sum_h w[h]*max(0, d[h]),
// d[0..31] in v0 and d[32..63] in v1, on packed two-lane fp32 arithmetic.
// The weights are staged halved (exact), and d + |d| is exactly 2*max(0, d)
// (+0 for d <= 0), so each product (d + |d|) * (w/2) equals max(0, d) * w
// bit for bit: one packed add and one packed FMA per pair of heads.
__device__ __forceinline__ float head_sum64(const uint32_t (&v0)[32], const uint32_t (&v1)[32],
                                            const float* __restrict__ whalf) {
  float2 a[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                 make_float2(0.f, 0.f)};
#pragma unroll
  for (int c = 0; c < 64; c += 4) {
    const float4 w4 = *reinterpret_cast<const float4*>(whalf + c);
    const uint32_t* v = c < 32 ? v0 : v1;
    const int cc = c & 31;
    const float2 d01 = make_float2(__uint_as_float(v[cc + 0]), __uint_as_float(v[cc + 1]));
    const float2 d23 = make_float2(__uint_as_float(v[cc + 2]), __uint_as_float(v[cc + 3]));
    const float2 x01 = __fadd2_rn(d01, make_float2(fabsf(d01.x), fabsf(d01.y)));
    const float2 x23 = __fadd2_rn(d23, make_float2(fabsf(d23.x), fabsf(d23.y)));
    const int j = (c >> 2) & 1;
    a[2 * j] = __ffma2_rn(x01, make_float2(w4.x, w4.y), a[2 * j]);
    a[2 * j + 1] = __ffma2_rn(x23, make_float2(w4.z, w4.w), a[2 * j + 1]);
  }
  return ((a[0].x + a[0].y) + (a[1].x + a[1].y)) + ((a[2].x + a[2].y) + (a[3].x + a[3].y));
}

// Two queries' head sums of one key at once (the same arithmetic as
// head_sum64, per query), interleaved so that eight independent packed
// accumulators keep the FMA pipe busy.
__device__ __forceinline__ void head_sum64x2(const uint32_t (&va)[2][32], const uint32_t (&vb)[2][32],
                                             const float* __restrict__ wa, const float* __restrict__ wb,
                                             float& sa, float& sb) {
  float2 a[4], c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a[i] = make_float2(0.f, 0.f);
    c[i] = make_float2(0.f, 0.f);
  }
#pragma unroll
  for (int h = 0; h < 64; h += 4) {
    const float4 wa4 = *reinterpret_cast<const float4*>(wa + h);
    const float4 wb4 = *reinterpret_cast<const float4*>(wb + h);
    const int hi = h >> 5, hh = h & 31;
    const int j = (h >> 2) & 1;
    const float2 da01 = make_float2(__uint_as_float(va[hi][hh]), __uint_as_float(va[hi][hh + 1]));
    const float2 da23 = make_float2(__uint_as_float(va[hi][hh + 2]), __uint_as_float(va[hi][hh + 3]));
    const float2 db01 = make_float2(__uint_as_float(vb[hi][hh]), __uint_as_float(vb[hi][hh + 1]));
    const float2 db23 = make_float2(__uint_as_float(vb[hi][hh + 2]), __uint_as_float(vb[hi][hh + 3]));
    a[2 * j] = __ffma2_rn(__fadd2_rn(da01, make_float2(fabsf(da01.x), fabsf(da01.y))), make_float2(wa4.x, wa4.y), a[2 * j]);
    a[2 * j + 1] = __ffma2_rn(__fadd2_rn(da23, make_float2(fabsf(da23.x), fabsf(da23.y))), make_float2(wa4.z, wa4.w), a[2 * j + 1]);
    c[2 * j] = __ffma2_rn(__fadd2_rn(db01, make_float2(fabsf(db01.x), fabsf(db01.y))), make_float2(wb4.x, wb4.y), c[2 * j]);
    c[2 * j + 1] = __ffma2_rn(__fadd2_rn(db23, make_float2(fabsf(db23.x), fabsf(db23.y))), make_float2(wb4.z, wb4.w), c[2 * j + 1]);
  }
  sa = ((a[0].x + a[0].y) + (a[1].x + a[1].y)) + ((a[2].x + a[2].y) + (a[3].x + a[3].y));
  sb = ((c[0].x + c[0].y) + (c[1].x + c[1].y)) + ((c[2].x + c[2].y) + (c[3].x + c[3].y));
}

// This CTA's range of work (warp-collective; every lane gets the result).
// The offsets are validated first.  Segment (query block) s costs
// SEG_COST + len_s units, its tiles being the last len_s of them; the CTA
// takes units [lo, hi) of the total and scores the tiles among them, which
// are contiguous in the flat tile list.
struct Split {
  int seg0, kt0, count;
  bool bad;
};

template <int NQ, int SEG_COST>
__device__ Split find_split(const int32_t* __restrict__ off, int B, int T, int64_t kv_rows, int64_t ld, int QB,
                            int nseg, int lane) {
  bool bad = false;
  for (int b = lane; b < B; b += 32) {
    const int E = off[b + 1] - off[b];
    bad |= (off[b] < 0) || (E < T) || ((int64_t)E > ld);
  }
  if (lane == 0) bad |= ((int64_t)off[B] > kv_rows);
  bad = __any_sync(0xffffffffu, bad);
  Split r{0, 0, 0, bad};
  if (bad) return r;
  if (nseg == 1) {  // one sequence, one query block: the range in closed form
    const int len = seg_len<NQ>(off, T, QB, 0);
    const int64_t total = len + SEG_COST;
    const int64_t lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;
    const int64_t t_lo = max(lo, (int64_t)SEG_COST), t_hi = hi;
    if (t_hi > t_lo) {
      r.kt0 = (int)(t_lo - SEG_COST);
      r.count = (int)(t_hi - t_lo);
    }
    return r;
  }
  int64_t total = 0;
  for (int base = 0; base < nseg; base += 32) {
    const int seg = base + lane;
    int64_t u = seg < nseg ? seg_len<NQ>(off, T, QB, seg) + SEG_COST : 0;
    for (int o = 16; o; o >>= 1) u += __shfl_xor_sync(0xffffffffu, u, o);
    total += u;
  }
  const int64_t lo = total * blockIdx.x / gridDim.x;
  const int64_t hi = total * (blockIdx.x + 1) / gridDim.x;
  int64_t count = 0, acc = 0;
  bool found = false;
  for (int base = 0; base < nseg && acc < hi; base += 32) {
    const int seg = base + lane;
    const int len = seg < nseg ? seg_len<NQ>(off, T, QB, seg) : 0;
    const int64_t u = seg < nseg ? len + SEG_COST : 0;
    int64_t incl = u;
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int64_t tile_lo = acc + incl - len, tile_hi = acc + incl;  // this segment's tile units
    const int64_t ov_lo = max(tile_lo, lo), ov_hi = min(tile_hi, hi);
    int64_t ov = ov_hi > ov_lo ? ov_hi - ov_lo : 0;
    const unsigned m = __ballot_sync(0xffffffffu, ov > 0);
    if (!found && m) {
      const int src = __ffs(m) - 1;
      r.seg0 = __shfl_sync(0xffffffffu, seg, src);
      r.kt0 = (int)__shfl_sync(0xffffffffu, ov_lo - tile_lo, src);
      found = true;
    }
    for (int o = 16; o; o >>= 1) ov += __shfl_xor_sync(0xffffffffu, ov, o);
    count += ov;
    acc += __shfl_sync(0xffffffffu, incl, 31);
  }
  r.count = found ? (int)count : 0;
  return r;
}

template <int NQ, bool FP8>
__global__ void __launch_bounds__(IdxCfg<NQ, FP8>::THREADS, IdxCfg<NQ, FP8>::CTAS_PER_SM)
    indexer_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const float* __restrict__ w, const float* __restrict__ k_scale,
                   const int32_t* __restrict__ off, int B, int T, int64_t kv_rows,
                   float* __restrict__ scores, int64_t ld, int32_t* status) {
  using C = IdxCfg<NQ, FP8>;
  extern __shared__ uint8_t smem_raw[];
  if (!C::SLACK && (smem_u32(smem_raw) & 1023u) != 0) {  // uniform over the CTA
    if (threadIdx.x == 0) report(status, DSA_ERR_UNSUPPORTED);
    return;
  }
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* w_s = reinterpret_cast<float*>(smem + C::OFF_W);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto k_full = [&](int i) { return bar0 + 8u * i; };
  auto k_empty = [&](int i) { return bar0 + 8u * (C::KSTAGES + i); };
  auto q_full = [&](int i) { return bar0 + 8u * (2 * C::KSTAGES + i); };
  auto q_empty = [&](int i) { return bar0 + 8u * (2 * C::KSTAGES + 2 + i); };
  auto acc_full = [&](int i) { return bar0 + 8u * (2 * C::KSTAGES + 4 + i); };
  auto acc_empty = [&](int i) { return bar0 + 8u * (2 * C::KSTAGES + 4 + C::NACC + i); };
  SmemMisc* misc = reinterpret_cast<SmemMisc*>(smem + C::OFF_MISC);
  volatile int* abort = &misc->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int QB = (T + NQ - 1) / NQ;
  const int nseg = B * QB;

  // ---- prologue that touches no memory an earlier kernel may still write:
  // barriers, TMEM, descriptor prefetch.  Overlaps the previous kernel's tail.
  if (warp == C::PRODUCER && lane == 0) {
    for (int i = 0; i < C::KSTAGES; ++i) {
      mbar_init(k_full(i), 1);
      mbar_init(k_empty(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full(i), 2);                  // expect-tx arrival + "weights staged" arrival
      mbar_init(q_empty(i), 1 + C::EPI_WARPS);  // MMA commit + every epilogue warp
    }
    for (int i = 0; i < C::NACC; ++i) {
      mbar_init(acc_full(i), 1);
      mbar_init(acc_empty(i), C::EPI_WARPS);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(sbase + C::OFF_MISC + offsetof(SmemMisc, tmem_base), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) misc->abort = 0;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc->tmem_base);
  grid_dependency_wait();
  allow_dependents_launch();

  // Every role warp finds the CTA's work range itself (no block-wide sync).
  const Split sp = find_split<NQ, C::SEG_COST>(off, B, T, kv_rows, ld, QB, nseg, lane);
  if (sp.bad && blockIdx.x == 0 && threadIdx.x == 0) report(status, DSA_ERR_BAD_OFFSETS);
  const int count = sp.count;

  // Walk of the CTA's items, identical in every role.
  int seg = sp.seg0, kt = sp.kt0;
  int len = count > 0 ? seg_len<NQ>(off, T, QB, seg) : 0;

  if (NQ > 1 && warp == C::FILL_WARP) {
    // ------------------------------------------------------------ causal fill (whole warp)
    // -inf past the causal frontier of the rows r = blockIdx.x (mod gridDim.x):
    // keys beyond the last tile of a row's query block are never multiplied.
    // A warp of its own, 512 bytes per store instruction: kept off the
    // producer, whose next key-tile load must not wait behind these stores.
    if (!sp.bad) {
      const int64_t n_rows = (int64_t)B * T;
      for (int64_t f_r = blockIdx.x; f_r < n_rows; f_r += gridDim.x) {
        const int fb = (int)(f_r / T), ft = (int)(f_r - (int64_t)fb * T);
        const int64_t f_end = off[fb + 1] - off[fb];
        float* f_row = scores + f_r * ld;
        // the frontier is a multiple of 128 keys: 16-byte aligned
        for (int64_t s0 = (int64_t)seg_len<NQ>(off, T, QB, fb * QB + ft / NQ) * 128 + 4 * lane; s0 < f_end;
             s0 += 128) {
          if (s0 + 4 <= f_end) {
            *reinterpret_cast<float4*>(f_row + s0) = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
          } else {
            for (int j = 0; j < 4; ++j)
              if (s0 + j < f_end) f_row[s0 + j] = -INFINITY;
          }
        }
      }
    }
  } else if (warp == C::PRODUCER) {
    // ------------------------------------------------------------ producer (whole warp)
    int qord = -1;
    int issued = 0;
    for (int item = 0; item < count; ++item) {
      const int b = seg / QB, qb = seg - b * QB;
      if (item == 0 || kt == 0) {
        ++qord;
        const int qs = qord & 1;
        bool ok = mbar_wait(q_empty(qs), ((qord >> 1) & 1) ^ 1, abort, kWaitLimitNs);
        if (!__all_sync(0xffffffffu, ok)) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(q_full(qs), C::Q_BYTES);
          const int y = (b * T + qb * NQ) * kHI;
          for (int bx = 0; bx < C::BOXES; ++bx)
            tma_load_2d(sbase + C::OFF_Q + qs * C::Q_BYTES + bx * (C::N * 128), &tm_q,
                        bx * (FP8 ? 128 : 64), y, q_full(qs));
        }
      }
      const int st = item % C::KSTAGES;
      bool ok = mbar_wait(k_empty(st), ((item / C::KSTAGES) & 1) ^ 1, abort, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, ok)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(k_full(st), C::KT_BYTES);
        const int y = off[b] + kt * 128;
        for (int bx = 0; bx < C::BOXES; ++bx)
          tma_load_2d(sbase + C::OFF_K + st * C::KT_BYTES + bx * 16384, &tm_k,
                      bx * (FP8 ? 128 : 64), y, k_full(st));
      }
      if (item == 0 || kt == 0) {
        // per-head weights of this query block, for the epilogue, staged while
        // both copies fly; the second arrival on q_full publishes them
        const int qs = qord & 1;
        float* wd = w_s + qs * C::N;
        for (int i = lane; i < C::N; i += 32) {
          const int t = qb * NQ + i / kHI;
          // halved (exact for |w| >= 2^-125), see head_sum64
          wd[i] = t < T ? 0.5f * w[((int64_t)b * T + t) * kHI + (i % kHI)] : 0.f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(q_full(qs));
      }
      issued = item + 1;
      if (++kt == len && item + 1 < count) {
        ++seg;
        kt = 0;
        len = seg_len<NQ>(off, T, QB, seg);
      }
    }
    if (*abort && lane == 0) {  // let copies already in flight land before the CTA exits
      volatile int never = 0;
      for (int item = max(0, issued - C::KSTAGES); item < issued; ++item)
        mbar_wait(k_full(item % C::KSTAGES), (item / C::KSTAGES) & 1, &never, 10000000ull);
      if (qord >= 0) mbar_wait(q_full(qord & 1), (qord >> 1) & 1, &never, 10000000ull);
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = FP8 ? idesc_e4m3(128, C::N) : idesc_bf16(128, C::N);
      int qord = -1;
      int issued = 0;
      for (int item = 0; item < count; ++item) {
        if (item == 0 || kt == 0) {
          ++qord;
          if (!mbar_wait(q_full(qord & 1), (qord >> 1) & 1, abort, kWaitLimitNs)) break;
        }
        const int ab = item % C::NACC;
        if (!mbar_wait(acc_empty(ab), ((item / C::NACC) & 1) ^ 1, abort, kWaitLimitNs)) break;
        const int st = item % C::KSTAGES;
        if (!mbar_wait(k_full(st), (item / C::KSTAGES) & 1, abort, kWaitLimitNs)) break;
        tc_fence_after();
        const uint32_t a0 = sbase + C::OFF_K + st * C::KT_BYTES;
        const uint32_t b0 = sbase + C::OFF_Q + (qord & 1) * C::Q_BYTES;
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS; ++ks) {
          const uint32_t within = (ks & 3) * 32;
          const uint64_t ad = smem_desc(a0 + (ks >> 2) * 16384 + within, 16, 1024, kSwizzle128B);
          const uint64_t bd = smem_desc(b0 + (ks >> 2) * (C::N * 128) + within, 16, 1024, kSwizzle128B);
          if (FP8)
            mma_f8_ss(tmem + ab * C::N, ad, bd, idesc, ks > 0);
          else
            mma_f16_ss(tmem + ab * C::N, ad, bd, idesc, ks > 0);
        }
        tc_commit(k_empty(st));
        tc_commit(acc_full(ab));
        issued = item + 1;
        const bool seg_end = (kt + 1 == len) || (item + 1 == count);
        if (seg_end) tc_commit(q_empty(qord & 1));
        if (++kt == len && item + 1 < count) {
          ++seg;
          kt = 0;
          len = seg_len<NQ>(off, T, QB, seg);
        }
      }
      if (*abort && issued > 0) {  // MMAs must finish before TMEM is released
        volatile int never = 0;
        const int last = issued - 1;
        mbar_wait(acc_full(last % C::NACC), (last / C::NACC) & 1, &never, 10000000ull);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue warps
    const int qd = warp & 3;                    // TMEM lane quarter of this warp
    const int q_lo = (warp >> 2) * C::QPW;      // its share of the block's queries
    const int row = qd * 32 + lane;             // TMEM lane == key within the tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    int qord = -1;
    int cur_b = -1, E = 0, start = 0;
    int32_t base_row = 0;
    float* ksc_ring = reinterpret_cast<float*>(smem + C::OFF_KSC) + threadIdx.x;  // slot i at [i * EPI_WARPS * 32]
    for (int item = 0; item < count; ++item) {
      const int b = seg / QB, qb = seg - b * QB;
      if (item == 0 || kt == 0) {
        ++qord;  // the producer has staged this block's weights with the query tile
        bool ok = mbar_wait(q_full(qord & 1), (qord >> 1) & 1, abort, kWaitLimitNs);
        if (!__all_sync(0xffffffffu, ok)) break;
      }
      if (b != cur_b) {
        cur_b = b;
        base_row = off[b];
        E = off[b + 1] - base_row;
        start = E - T;
      }
      const int s = kt * 128 + row;
      if constexpr (FP8) {
        // This thread's key scale for tile item + j goes into ring slot
        // (item + j) % KSC_AHEAD, one commit group per tile (empty past the
        // run or the sequence); a run's first tile fetches the slots ahead of
        // it too.  The HBM latency of the scales then runs behind the tiles
        // in between instead of after each accumulator.
        auto fetch = [&](int j) {
          if (kt + j < len && item + j < count && s + 128 * j < E)
            cp_async_4(smem_u32(ksc_ring + ((item + j) % C::KSC_AHEAD) * (C::EPI_WARPS * 32)),
                       k_scale + base_row + s + 128 * j);
          cp_async_commit();
        };
        if (item == 0 || kt == 0) {
#pragma unroll
          for (int j = 0; j < C::KSC_AHEAD - 1; ++j) fetch(j);
        }
        fetch(C::KSC_AHEAD - 1);
      }
      const int ab = item % C::NACC;
      bool ok = mbar_wait(acc_full(ab), (item / C::NACC) & 1, abort, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      // every TMEM load of the warp's queries first, then one wait
      uint32_t v[C::QPW][2][32];
#pragma unroll
      for (int qq = 0; qq < C::QPW; ++qq) {
        tmem_ld32(lane_addr + ab * C::N + (q_lo + qq) * 64, v[qq][0]);
        tmem_ld32(lane_addr + ab * C::N + (q_lo + qq) * 64 + 32, v[qq][1]);
      }
      tc_wait_ld();
      // the accumulator is in registers: hand its TMEM buffer back to the MMA now
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty(ab));
      float ksc = 1.f;
      if constexpr (FP8) {
        cp_async_wait<C::KSC_AHEAD - 1>();  // this tile's group is the oldest still open
        ksc = ksc_ring[(item % C::KSC_AHEAD) * (C::EPI_WARPS * 32)];
      }
      float sc[C::QPW];
      if constexpr (C::QPW == 2) {
        const float* wq = w_s + (qord & 1) * C::N + q_lo * 64;
        head_sum64x2(v[0], v[1], wq, wq + 64, sc[0], sc[1]);
      } else {
#pragma unroll
        for (int qq = 0; qq < C::QPW; ++qq)
          sc[qq] = head_sum64(v[qq][0], v[qq][1], w_s + (qord & 1) * C::N + (q_lo + qq) * 64);
      }
#pragma unroll
      for (int qq = 0; qq < C::QPW; ++qq) {
        const int q = q_lo + qq;
        const float score = sc[qq] * ksc;
        const int t = qb * NQ + q;
        if (t < T && s < E)
          scores[((int64_t)b * T + t) * ld + s] = (s <= start + t) ? score : -INFINITY;
      }
      __syncwarp();
      if (lane == 0 && (kt + 1 == len || item + 1 == count)) mbar_arrive(q_empty(qord & 1));  // block done
      if (++kt == len && item + 1 < count) {
        ++seg;
        kt = 0;
        len = seg_len<NQ>(off, T, QB, seg);
      }
    }
    if constexpr (FP8) cp_async_wait<0>();  // scale fetches past the CTA's last tile
  }

  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort) report(status, DSA_ERR_TIMEOUT);
}

template <int NQ, bool FP8>
int launch_cfg(const IndexerArgs& a, cudaStream_t stream) {
  using C = IdxCfg<NQ, FP8>;
  CUtensorMap tq, tk;
  const CUtensorMapDataType dt = FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint32_t box_inner = FP8 ? 128 : 64;
  const uint64_t q_rows = (uint64_t)a.B * a.T * kHI;
  if (!make_tmap_2d(&tq, a.q_idx, dt, kDI, q_rows, C::ROWB, box_inner, C::N,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  if (!make_tmap_2d(&tk, a.k_idx, dt, kDI, (uint64_t)a.kv_rows, C::ROWB, box_inner, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  auto kern = indexer_kernel<NQ, FP8>;
  static PerDeviceOnce attr;  // per template instance
  if (attr.run([&] { return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES); }) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  const int grid = device_info().sm_count * C::CTAS_PER_SM;
  const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, stream, tq, tk,
                                   a.w, a.k_scale, a.offsets, a.B, a.T, a.kv_rows, a.scores, a.ld,
                                   a.status);
  return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// Queries per prefill block (bf16): N = 64 * kPrefillNQ.
constexpr int kPrefillNQ = 4;

}  // namespace

int launch_indexer(const IndexerArgs& a, cudaStream_t stream) {
  const bool fp8 = a.idx_dtype == DSA_E4M3;
  if (a.T == 1) return fp8 ? launch_cfg<1, true>(a, stream) : launch_cfg<1, false>(a, stream);
  return fp8 ? launch_cfg<4, true>(a, stream) : launch_cfg<kPrefillNQ, false>(a, stream);
}

}  // namespace dsa
