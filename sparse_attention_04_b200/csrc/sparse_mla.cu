// sparse_mla.cu -- stage 3: absorbed MLA over the selected latent rows.
//
// "DeepSeek-V3.2-Exp - Apply sparse mask", MQA decode listing:
//   scores = (q_nope.kv + q_pe.pe) * softmax_scale,   S~ = S' + M^sel,
//   p = softmax(S~),   x = p . kv
// With the cache row stored as one 576-wide vector (512 latent || 64 rope) the
// two score einsums are one dot product, and only the selected rows carry a
// finite score, so the kernel gathers exactly those rows and never touches
// the rest of the cache.
//
// Work unit (one CTA, one per SM): query row r, value half v (latent columns
// [256v, 256v+256)), split sp (a contiguous range of 32-key chunks of the
// row's index list).  Per chunk i:
//   S_i = Q . Kv_i^T          M=128 heads, N=32 keys, K=576  (tcgen05, TMEM)
//   P_i = exp2(S_i*scale*log2e - m)  in bf16                  (CUDA cores)
//   O  += P_i . Kv_i[:, half] M=128, N=256, K=32              (tcgen05, TMEM)
// The running max m is only raised when a chunk exceeds it by more than
// 2^8 (then O and the running sum are rescaled), so P <= 256 and the
// final O / l is exact softmax.  With more than one split, the unnormalised
// O (bf16) and (m, l) go to the workspace and the combine kernel merges them.
//
// TMEM: O half in columns [0,256), S in two 32-column buffers at 256 and 288.
// Shared memory: Q (128 x 576 bf16, 9 swizzled 64-column blocks, by TMA), two
// stages of 32 gathered rows (cp.async, same swizzled layout), and P.
// The gathered stage is K-major for Q.K^T and, read as MN-major, the B
// operand of P.V: one copy of each row serves both products.
//
// Roles: warps 0-3 softmax + epilogue (thread = head = TMEM lane),
//        warps 4-7 row gather, warp 8 TMEM allocator + MMA issuer.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>

#include "dsa_internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace dsa {
namespace {

constexpr int kChunk = 32;
constexpr int kKB = kDQK / 64;                   // 9 column blocks of 64
constexpr int kQBytes = kKB * 128 * 128;         // 147456
constexpr int kKvBytes = kKB * kChunk * 128;     // 36864
constexpr int kPBytes = 128 * kChunk * 2;        // 8192
constexpr int kOffQ = 0;
constexpr int kOffKv = kOffQ + kQBytes;
constexpr int kOffP = kOffKv + 2 * kKvBytes;
constexpr int kOffBar = kOffP + kPBytes;
constexpr int kNumBar = 9;
constexpr int kOffMisc = kOffBar + kNumBar * 8;
constexpr int kStageBlock = 128 * 128;           // epilogue staging: one box, 128 rows x 128 B
static_assert(8 * kStageBlock <= kQBytes, "the staged output fits where the query tile was");
constexpr int kMiscBytes = 64 + 4 * ((DSA_MAX_TOPK + kChunk - 1) / kChunk);  // MlaMisc
constexpr int kSmemBytes = kOffMisc + kMiscBytes + 1024;
constexpr int kThreads = 288;
constexpr int kTmemCols = 512;
constexpr uint32_t kIdescQK = idesc_bf16(128, kChunk);
constexpr uint32_t kIdescPV = idesc_bf16(128, 256, /*b_mn_major=*/true);
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffKv % 1024 == 0 && kOffP % 1024 == 0, "alignment");

constexpr int kMaxChunks = (DSA_MAX_TOPK + kChunk - 1) / kChunk;
struct MlaMisc {
  int tmem_base, abort, n_chunks, last_valid, pad[12];
  uint32_t vmask[kMaxChunks];  // per chunk of this split: bit j = position valid
};
static_assert(sizeof(MlaMisc) == kMiscBytes, "shared-memory budget of the bookkeeping block");


// Position selected at slot j of row r: the index list's entry, or (dense
// mode, every prefix shorter than k) slot j itself while j < the prefix length.
__device__ __forceinline__ int32_t selected_pos(const int32_t* __restrict__ idx_row, bool dense, int j, int L) {
  return dense ? (j < L ? j : -1) : idx_row[j];
}

__device__ __forceinline__ bool index_ok(int32_t idx, int E) { return idx >= 0 && idx < E; }

__global__ void __launch_bounds__(kThreads, 1)
    sparse_mla_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_out,
                      const MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kOffBar;
  const uint32_t q_full = bar0;
  auto kv_full = [&](int i) { return bar0 + 8u * (1 + i); };
  auto kv_empty = [&](int i) { return bar0 + 8u * (3 + i); };
  auto s_full = [&](int i) { return bar0 + 8u * (5 + i); };
  const uint32_t p_full = bar0 + 8u * 7;
  const uint32_t pv_done = bar0 + 8u * 8;
  MlaMisc* misc = reinterpret_cast<MlaMisc*>(smem + kOffMisc);
  volatile int* abort = &misc->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (!p.early_inputs) grid_dependency_wait();  // q and the offsets may come from the previous kernel
  const int v = blockIdx.x & 1;
  const int sp = (blockIdx.x >> 1) % p.n_splits;
  const int r = (blockIdx.x >> 1) / p.n_splits;
  const int b = r / p.T;
  const int32_t base_row = p.off[b];
  const int E = p.off[b + 1] - base_row;
  const bool geo_ok = base_row >= 0 && E >= p.T && (int64_t)base_row + E <= p.kv_rows;
  const int32_t* idx_row = p.dense ? nullptr : p.idx + (int64_t)r * p.k;
  const bool dense = p.dense != 0;
  const int L_row = E - p.T + (r - b * p.T) + 1;  // causal prefix of the row
  const int c_begin = sp * p.cps;
  const int n_chunks_total = (p.k + kChunk - 1) / kChunk;
  const int c_end = min(c_begin + p.cps, n_chunks_total);

  // ---- prologue: barriers, TMEM, and the query tile, overlapping the
  // previous kernel's tail when the inputs are known to be complete.
  if (threadIdx.x == 0) {
    misc->last_valid = -1;
    misc->abort = 0;
  }
  if (threadIdx.x < kMaxChunks) misc->vmask[threadIdx.x] = 0u;
  if (warp == 8) {
    if (lane == 0) {
      mbar_init(q_full, 1 + p.debug_stall);  // + the test hook's missing arrival
      for (int i = 0; i < 2; ++i) {
        mbar_init(kv_full(i), 64);  // one arrival per gather thread
        mbar_init(kv_empty(i), 1);
        mbar_init(s_full(i), 1);
      }
      mbar_init(p_full, 128);
      mbar_init(pv_done, 1);
      fence_mbar_init();
      if (geo_ok) {
        mbar_arrive_expect_tx(q_full, kQBytes);
        for (int kb = 0; kb < kKB; ++kb)
          tma_load_2d(sbase + kOffQ + kb * 16384, &tm_q, kb * 64, r * p.H, q_full);
      }
    }
    __syncwarp();
    tmem_alloc(sbase + kOffMisc + offsetof(MlaMisc, tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc->tmem_base);
  grid_dependency_wait();  // the indices come from the previous kernel
  allow_dependents_launch();

  // ---- how many chunks of this split hold a selected row.  Each warp owns
  // whole chunks: it loads all their indices first (one L2 round trip), then
  // builds each chunk's validity mask with ballots, so no shared-memory
  // atomics contend on a chunk's mask word.
  if (geo_ok) {
    constexpr int kWarps = kThreads / 32, kPerWarp = (kMaxChunks + kWarps - 1) / kWarps;
    const int n_ch = c_end - c_begin;
    int32_t ids[kPerWarp][kChunk / 32];
#pragma unroll
    for (int u = 0; u < kPerWarp; ++u)
#pragma unroll
      for (int hh = 0; hh < kChunk / 32; ++hh) {
        const int c = warp + kWarps * u, j = (c_begin + c) * kChunk + 32 * hh + lane;
        ids[u][hh] = (c < n_ch && j < p.k) ? selected_pos(idx_row, dense, j, L_row) : -1;
      }
    int lv = -1;
#pragma unroll
    for (int u = 0; u < kPerWarp; ++u) {
      const int c = warp + kWarps * u;
      if (c >= n_ch) break;  // uniform over the warp
      uint32_t m = 0;
#pragma unroll
      for (int hh = 0; hh < kChunk / 32; ++hh) {
        const bool valid = index_ok(ids[u][hh], E);
        if (!valid && ids[u][hh] != -1) report(p.status, DSA_ERR_BAD_INDEX);
        m |= static_cast<uint32_t>(__ballot_sync(0xffffffffu, valid)) << (32 * hh);
      }
      if (lane == 0) misc->vmask[c] = m;
      if (m) lv = (c_begin + c) * kChunk + 31 - __clz((int)m);
    }
    if (lane == 0 && lv >= 0) atomicMax(&misc->last_valid, lv);
  } else if (threadIdx.x == 0) {
    report(p.status, DSA_ERR_BAD_OFFSETS);
  }
  __syncthreads();
  const int n_my = misc->last_valid < 0 ? 0 : misc->last_valid / kChunk - c_begin + 1;

  const int h = threadIdx.x;  // softmax / epilogue threads: head = TMEM lane
  if (n_my == 0) {
    // nothing selected in this split: empty partial, or zero output
    if (warp < 4 && h < p.H) {
      const int64_t rh = (int64_t)r * p.H + h;
      if (p.n_splits == 1) {
        if (p.out_bf16) {
          __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out) + rh * kDV + 256 * v;
          for (int c = 0; c < 256; ++c) o[c] = __float2bfloat16(0.f);
        } else {
          float* o = reinterpret_cast<float*>(p.out) + rh * kDV + 256 * v;
          for (int c = 0; c < 256; ++c) o[c] = 0.f;
        }
        if (v == 0 && p.lse) p.lse[rh] = -INFINITY;
      } else {
        const int64_t slot = ((int64_t)r * p.n_splits + sp) * p.H + h;
        __nv_bfloat16* o = p.ws_o + slot * kDV + 256 * v;
        for (int c = 0; c < 256; ++c) o[c] = __float2bfloat16(0.f);
        if (v == 0) {
          p.ws_ml[2 * slot] = -INFINITY;
          p.ws_ml[2 * slot + 1] = 0.f;
        }
      }
    }
    if (warp == 8 && lane == 0 && geo_ok) {  // the query tile must land before the CTA exits
      volatile int never = 0;
      mbar_wait(q_full, 0, &never, 10000000ull);
    }
  } else if (warp == 8) {
    // -------------------------------------------------------------- MMA issuer
    // QK of chunk i and PV of chunk j < i touch different TMEM (S buffer,
    // O) and shared memory (stage i; stage j and P), so they are issued in
    // whichever order their inputs arrive: QK(i) once chunk i has landed and
    // its S buffer is free (PV(i-2) issued, so softmax(i-2) is done with it);
    // PV(j) once softmax(j) has written P.  An early PV(j) frees its stage for
    // the load of chunk j+2 without waiting for chunk j+1 to land.
    if (lane == 0) {
      int n_qk = 0, n_pv = 0;
      bool ok = mbar_wait(q_full, 0, abort, p.wait_limit_ns);
      // Descriptors differ only in the start-address field (address >> 4 in
      // the low 14 bits, no carry below 256 KiB): built once, offset per MMA.
      const uint64_t qk_a0 = smem_desc(sbase + kOffQ, 16, 1024, kSwizzle128B);
      const uint64_t qk_b0 = smem_desc(sbase + kOffKv, 16, 1024, kSwizzle128B);
      const uint64_t pv_a0 = smem_desc(sbase + kOffP, 128, 512, kSwizzleNone);
      const uint64_t pv_b0 = smem_desc(sbase + kOffKv + (4 * v) * (kChunk * 128), kChunk * 128, 1024, kSwizzle128B);
      // PV of chunk n_pv (its P is in shared memory; p_full has been seen)
      auto issue_pv = [&]() {
        const int j = n_pv;
        tc_fence_after();
        const uint64_t bd0 = pv_b0 + (uint64_t)(((j & 1) * kKvBytes) >> 4);
#pragma unroll
        for (int ks = 0; ks < kChunk / 16; ++ks)
          mma_f16_ss(tmem, pv_a0 + (uint64_t)((ks * 256) >> 4), bd0 + (uint64_t)((ks * 2048) >> 4), kIdescPV,
                     (j > 0 || ks > 0) ? 1u : 0u);
        tc_commit(pv_done);
        tc_commit(kv_empty(j & 1));
        ++n_pv;
      };
      const uint64_t t0 = globaltimer_ns();
      uint32_t spins = 0;
      while (ok && n_pv < n_my) {
        bool progressed = false;
        if (n_qk < n_my && n_qk <= n_pv + 1 && mbar_try_wait(kv_full(n_qk & 1), (n_qk >> 1) & 1)) {
          const int st = n_qk & 1;
          tc_fence_after();
          const uint64_t bst = qk_b0 + (uint64_t)((st * kKvBytes) >> 4);
#pragma unroll 1
          for (int kb = 0; kb < kKB; ++kb) {
            const uint64_t akb = qk_a0 + (uint64_t)((kb * 16384) >> 4);
            const uint64_t bkb = bst + (uint64_t)((kb * (kChunk * 128)) >> 4);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_f16_ss(tmem + 256 + 32 * st, akb + (uint64_t)ks * 2, bkb + (uint64_t)ks * 2, kIdescQK,
                         (kb | ks) ? 1u : 0u);
            // a PV whose P is ready is slotted in between the groups of QK
            // MMAs, instead of waiting for the whole (slow, N = 32) QK
            if (n_pv < n_qk && mbar_try_wait(p_full, n_pv & 1)) issue_pv();
          }
          tc_commit(s_full(st));
          ++n_qk;
          progressed = true;
        }
        if (n_pv < n_qk && mbar_try_wait(p_full, n_pv & 1)) {
          issue_pv();
          progressed = true;
        }
        if (!progressed && (++spins & 63u) == 0) {  // bounded, like every other wait here
          if (*abort) ok = false;
          else if (globaltimer_ns() - t0 > p.wait_limit_ns) {
            *abort = 1;
            ok = false;
          }
        }
      }
      if (*abort && n_pv > 0) {  // tensor-core work must finish before TMEM is released
        volatile int never = 0;
        mbar_wait(pv_done, (n_pv - 1) & 1, &never, 10000000ull);
      }
      if (*abort) {
        volatile int never = 0;
        mbar_wait(q_full, 0, &never, 10000000ull);
      }
    }
  } else if (warp >= 4) {
    // -------------------------------------------------------------- row gather
    // Warps 4-5 fill stage 0 (even chunks), warps 6-7 stage 1 (odd chunks):
    // the two groups run independently, so both stages are in flight from
    // the start and a group waits only for its own copies before it signals.
    // Each warp copies 16 whole rows, one row at a time, so every copy
    // instruction reads 512 contiguous bytes of a row.
    const int pt = threadIdx.x - 128;
    const int grp = pt >> 6, gw = (pt >> 5) & 1;
    const __nv_bfloat16* kv = p.kv;
    for (int i = grp; i < n_my; i += 2) {
      const int st = i & 1;
      if (!mbar_wait(kv_empty(st), ((i >> 1) & 1) ^ 1, abort, p.wait_limit_ns)) break;
      int32_t my_id = -1;
      if (lane < 16) {
        const int pos = (c_begin + i) * kChunk + gw * 16 + lane;
        my_id = pos < p.k ? selected_pos(idx_row, dense, pos, L_row) : -1;
      }
#pragma unroll 2
      for (int rr = 0; rr < 16; ++rr) {
        const int jr = gw * 16 + rr;
        const int32_t id = __shfl_sync(0xffffffffu, my_id, rr);
        const bool valid = index_ok(id, E);
        const __nv_bfloat16* src = valid ? kv + ((int64_t)base_row + id) * kDQK : kv;
        const uint32_t dst_row = sbase + kOffKv + st * kKvBytes + (jr >> 3) * 1024 + (jr & 7) * 128;
#pragma unroll
        for (int u = 0; u < 3; ++u) {
          const int c = lane + 32 * u;  // 16-byte piece of the 72 in a row
          if (c < kDQK / 8) {
            const int kb = c >> 3, cc = c & 7;
            cp_async_16(dst_row + kb * (kChunk * 128) + ((cc ^ (jr & 7)) << 4), src + c * 8, valid ? 16u : 0u);
          }
        }
      }
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async_smem();
      mbar_arrive(kv_full(st));
    }
    cp_async_wait<0>();
  } else {
    // -------------------------------------------------------------- softmax + epilogue
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int i = 0; i < n_my; ++i) {
      const int st = i & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(s_full(st), (i >> 1) & 1, abort, p.wait_limit_ns));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[32];
      tmem_ld32(lane_addr + 256 + 32 * st, sv);
      tc_wait_ld();
      float x[32];
      float mc = -INFINITY;
      const uint32_t vm = misc->vmask[i];  // validity of the chunk's 32 positions
      if (vm == ~0u) {  // every position valid (the common case): scale in pairs
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float2 x2 = __fmul2_rn(make_float2(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])),
                                       make_float2(p.scale_log2, p.scale_log2));
          x[j] = x2.x;
          x[j + 1] = x2.y;
          mc = fmaxf(mc, fmaxf(x2.x, x2.y));
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          x[j] = ((vm >> j) & 1u) ? __uint_as_float(sv[j]) * p.scale_log2 : -INFINITY;
          mc = fmaxf(mc, x[j]);
        }
      }
      float m_new = m_run;
      bool resc = false;
      if (mc > m_run + 8.f) {
        resc = m_run != -INFINITY;
        m_new = mc;
      }
      const float alpha = resc ? exp2f(m_run - m_new) : 1.f;
      // p = 2^(x - m) (masked positions carry x = -inf, so p = +0), rounded
      // to bf16 for P.V; the running sum adds the same rounded values
      uint32_t pk[16];
      float2 l2 = make_float2(0.f, 0.f);
      const float m_sub = m_new == -INFINITY ? 0.f : m_new;  // nothing valid yet: every x is -inf
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float2 d = __fadd2_rn(make_float2(x[j], x[j + 1]), make_float2(-m_sub, -m_sub));
        const __nv_bfloat162 pb = __floats2bfloat162_rn(ex2_approx(d.x), ex2_approx(d.y));
        l2 = __fadd2_rn(l2, __bfloat1622float2(pb));
        pk[j / 2] = *reinterpret_cast<const uint32_t*>(&pb);
      }
      const float l_chunk = l2.x + l2.y;
      if (i > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(pv_done, (i - 1) & 1, abort, p.wait_limit_ns));
        if (!ok) break;
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
        for (int cb = 0; cb < 8; ++cb) {
          uint32_t ov[32];
          tmem_ld32(lane_addr + 32 * cb, ov);
          tc_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
          tmem_st32(lane_addr + 32 * cb, ov);
        }
        tc_wait_st();
      }
      l_run = l_run * alpha + l_chunk;
      m_run = m_new;
      // P row h, K-major without swizzle: 8-row x 16-byte core matrices,
      // 128 bytes apart along K, 512 bytes apart along M.
      uint8_t* prow = smem + kOffP + (h >> 3) * 512 + (h & 7) * 16;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4*>(prow + c * 128) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(pv_done, (n_my - 1) & 1, abort, p.wait_limit_ns));
    // Every MMA has completed, so the query tile's shared memory is free: the
    // 128 x 256 result is staged there as 128-byte-swizzled boxes of 32 fp32
    // (or 64 bf16) columns, one thread per head row, and written by a few
    // TMA tensor stores (the output's tensor map has one box per such block).
    const bool final_out = p.n_splits == 1;
    const bool as_bf16 = !final_out || p.out_bf16;  // partials are bf16 too
    if (ok) {
      tc_fence_after();
      const float mul = final_out ? (l_run > 0.f ? 1.f / l_run : 0.f) : 1.f;
      uint8_t* stage = smem + kOffQ;
      const int sw = h & 7;
#pragma unroll 1
      for (int cb2 = 0; cb2 < 8; cb2 += 2) {
        uint32_t ovp[2][32];
        tmem_ld32(lane_addr + 32 * cb2, ovp[0]);
        tmem_ld32(lane_addr + 32 * cb2 + 32, ovp[1]);
        tc_wait_ld();
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int cb = cb2 + hf;
          const uint32_t (&ov)[32] = ovp[hf];
          if (as_bf16) {
            uint8_t* rowp = stage + (cb >> 1) * kStageBlock + h * 128;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint32_t w4[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 t2 = __floats2bfloat162_rn(__uint_as_float(ov[8 * q4 + 2 * e]) * mul,
                                                                 __uint_as_float(ov[8 * q4 + 2 * e + 1]) * mul);
                w4[e] = *reinterpret_cast<const uint32_t*>(&t2);
              }
              const int ci = (cb & 1) * 4 + q4;
              *reinterpret_cast<uint4*>(rowp + ((ci ^ sw) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
          } else {
            uint8_t* rowp = stage + cb * kStageBlock + h * 128;
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              *reinterpret_cast<float4*>(rowp + ((q4 ^ sw) << 4)) =
                  make_float4(__uint_as_float(ov[4 * q4]) * mul, __uint_as_float(ov[4 * q4 + 1]) * mul,
                              __uint_as_float(ov[4 * q4 + 2]) * mul, __uint_as_float(ov[4 * q4 + 3]) * mul);
          }
        }
      }
      fence_proxy_async_smem();
    }
    named_barrier_sync(1, 128);  // every epilogue warp, whatever its wait outcome
    if (threadIdx.x == 0 && !*abort) {
      const int nblk = as_bf16 ? 4 : 8, colw = as_bf16 ? 64 : 32;
      const int y = final_out ? r * p.H : (r * p.n_splits + sp) * p.H;
      for (int bk = 0; bk < nblk; ++bk) tma_store_2d(&tm_out, sbase + kOffQ + bk * kStageBlock, 256 * v + colw * bk, y);
      bulk_commit();
    }
    if (ok && h < p.H && v == 0) {
      const int64_t rh = (int64_t)r * p.H + h;
      if (final_out) {
        if (p.lse) p.lse[rh] = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
      } else {
        const int64_t slot = ((int64_t)r * p.n_splits + sp) * p.H + h;
        p.ws_ml[2 * slot] = l_run > 0.f ? m_run : -INFINITY;
        p.ws_ml[2 * slot + 1] = l_run;
      }
    }
    if (threadIdx.x == 0) bulk_wait_read();  // the staged boxes stay valid until read
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort) report(p.status, DSA_ERR_TIMEOUT);
}

// Merges the per-split partials of one (row, head): O = sum_s 2^(m_s-M) O_s /
// sum_s 2^(m_s-M) l_s (the same log-sum-exp merge a single pass would do).
// G heads of one row per CTA, 64 * SP threads per head: thread (part, c)
// owns eight columns c and the splits part, part + SP, ...; with SP > 1 the
// parts' sums meet in shared memory.  Launch shapes:
//   - many (row, head) pairs: G > 1, SP = 1.  One CTA per pair would be so
//     short that the rate at which CTAs are dispatched sets the time (32 rows
//     x 128 heads, two splits: 19 us with one head per CTA, measured on B200);
//   - few pairs with many splits (a decode row): G = 1, SP = 4, so that four
//     times the warps share each head's dependent load-and-add chain.
constexpr int kMaxSplits = 64;
__device__ __forceinline__ void acc_bf16x8(float (&acc)[8], const uint4 v, float f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
    acc[2 * e] = fmaf(t.x, f, acc[2 * e]);
    acc[2 * e + 1] = fmaf(t.y, f, acc[2 * e + 1]);
  }
}

template <int G, int SP>
__global__ void __launch_bounds__(64 * G * SP)
    mla_combine_kernel(const __nv_bfloat16* __restrict__ ws_o, const float* __restrict__ ws_ml, int H,
                       int n_splits, void* out, int out_bf16, float* lse) {
  static_assert(G == 1 || SP == 1, "several heads or several parts per head, not both");
  __shared__ float s_w[G][kMaxSplits];
  __shared__ float s_ml[G][2];
  __shared__ float4 s_part[SP > 1 ? (SP - 1) * 64 * 2 : 1];  // parts 1.. of each column group
  grid_dependency_wait();  // partials come from the previous kernel
  allow_dependents_launch();
  const int groups = (H + G - 1) / G;  // head groups per row
  const int64_t r = blockIdx.x / groups;
  const int g = SP > 1 ? 0 : threadIdx.x >> 6;   // head of the group
  const int part = SP > 1 ? threadIdx.x >> 6 : 0;  // this thread's splits: part, part + SP, ...
  const int64_t h = (int64_t)(blockIdx.x % groups) * G + g;
  const bool live = h < H;             // uniform over the head's warps
  const int64_t rh = r * H + h;
  const int c8 = threadIdx.x & 63;  // eight columns: 8*c8 .. 8*c8+7
  const uint4* base = reinterpret_cast<const uint4*>(ws_o + (r * n_splits * H + (live ? h : 0)) * kDV) + c8;
  const int64_t stride = (int64_t)H * kDV / 8 * SP;  // uint4 between this thread's consecutive splits
  const int n_mine = (n_splits - part + SP - 1) / SP;
  // splits whose loads are in flight at once (registers: 512 threads at G = 8)
  constexpr int NB = G == 1 && SP == 1 ? 32 : 16;
  uint4 o[NB];
  const uint4* mine = base + (int64_t)part * (stride / SP);
#pragma unroll
  for (int s = 0; s < NB; ++s)
    if (live && s < n_mine) o[s] = __ldg(mine + s * stride);
  if (live && part == 0 && c8 < 32) {
    const int s0 = c8, s1 = c8 + 32;
    float m0 = -INFINITY, l0 = 0.f, m1 = -INFINITY, l1 = 0.f;
    if (s0 < n_splits) {
      const int64_t slot = (r * n_splits + s0) * H + h;
      m0 = ws_ml[2 * slot];
      l0 = ws_ml[2 * slot + 1];
    }
    if (s1 < n_splits) {
      const int64_t slot = (r * n_splits + s1) * H + h;
      m1 = ws_ml[2 * slot];
      l1 = ws_ml[2 * slot + 1];
    }
    float M = fmaxf(m0, m1);
#pragma unroll
    for (int d = 16; d; d >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, d));
    const float f0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - M);
    const float f1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - M);
    float L = l0 * f0 + l1 * f1;
#pragma unroll
    for (int d = 16; d; d >>= 1) L += __shfl_xor_sync(0xffffffffu, L, d);
    s_w[g][s0] = f0;
    s_w[g][s1] = f1;
    if (s0 == 0) {
      s_ml[g][0] = M;
      s_ml[g][1] = L;
    }
  }
  __syncthreads();
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (live) {
    for (int sb = 0; sb < n_mine; sb += NB) {
      if (sb > 0) {  // the next group of this thread's splits
#pragma unroll
        for (int s = 0; s < NB; ++s)
          if (sb + s < n_mine) o[s] = __ldg(mine + (sb + s) * stride);
      }
#pragma unroll
      for (int s = 0; s < NB; ++s)
        if (sb + s < n_mine) acc_bf16x8(acc, o[s], s_w[g][part + SP * (sb + s)]);
    }
  }
  if constexpr (SP > 1) {
    if (part > 0) {
      s_part[((part - 1) * 64 + c8) * 2] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      s_part[((part - 1) * 64 + c8) * 2 + 1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
    __syncthreads();
    if (part > 0) return;  // no barrier below
#pragma unroll
    for (int q = 0; q < SP - 1; ++q) {
      const float4 a = s_part[(q * 64 + c8) * 2], b = s_part[(q * 64 + c8) * 2 + 1];
      acc[0] += a.x;
      acc[1] += a.y;
      acc[2] += a.z;
      acc[3] += a.w;
      acc[4] += b.x;
      acc[5] += b.y;
      acc[6] += b.z;
      acc[7] += b.w;
    }
  }
  if (!live) return;
  const float M = s_ml[g][0], L = s_ml[g][1];
  const float inv = L > 0.f ? 1.f / L : 0.f;
  if (out_bf16) {
    uint32_t w4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 t2 = __floats2bfloat162_rn(acc[2 * e] * inv, acc[2 * e + 1] * inv);
      w4[e] = *reinterpret_cast<const uint32_t*>(&t2);
    }
    reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out) + rh * kDV)[c8] =
        make_uint4(w4[0], w4[1], w4[2], w4[3]);
  } else {
    float4* o4 = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + rh * kDV) + 2 * c8;
    o4[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    o4[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
  }
  if (c8 == 0 && lse) lse[rh] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
}

// Heads per combine CTA: one while that leaves at least two CTAs per SM,
// else up to eight.
int combine_heads_per_cta(int64_t n_rows, int H, int sms) {
  int G = 1;
  while (G < 8 && n_rows * ((H + 2 * G - 1) / (2 * G)) >= 2 * (int64_t)sms) G *= 2;
  return G;
}

cudaError_t launch_combine(const MlaParams& p, int64_t n_rows, int H, cudaStream_t stream) {
  const int G = combine_heads_per_cta(n_rows, H, device_info().sm_count);
  const dim3 grid((unsigned)(n_rows * ((H + G - 1) / G)));
  const __nv_bfloat16* o = p.ws_o;
  const float* ml = p.ws_ml;
  const int ns = p.n_splits;
  switch (G) {
    case 1:
      // one head per CTA: with eight or more splits, four parts per head
      if (ns >= 8)
        return launch_pdl(mla_combine_kernel<1, 4>, grid, dim3(256), 0, stream, o, ml, H, ns, p.out, p.out_bf16, p.lse);
      return launch_pdl(mla_combine_kernel<1, 1>, grid, dim3(64), 0, stream, o, ml, H, ns, p.out, p.out_bf16, p.lse);
    case 2: return launch_pdl(mla_combine_kernel<2, 1>, grid, dim3(128), 0, stream, o, ml, H, ns, p.out, p.out_bf16, p.lse);
    case 4: return launch_pdl(mla_combine_kernel<4, 1>, grid, dim3(256), 0, stream, o, ml, H, ns, p.out, p.out_bf16, p.lse);
    default: return launch_pdl(mla_combine_kernel<8, 1>, grid, dim3(512), 0, stream, o, ml, H, ns, p.out, p.out_bf16, p.lse);
  }
}

}  // namespace

// Which attention kernel a launch uses.
//
// The pair kernel (sparse_mla_pair.cu: a QK CTA and a PV CTA per (row,
// split), 128-key chunks, S computed once at N = 128) wherever the launch has
// at least kMlaPairMinChunksPerSlot 128-key chunks per cluster slot (two SMs):
// large decode batches and causal prefill.  Its per-unit prologue (128 KB of
// query into TMEM) and its 128-key chunks make it slower for a few long rows.
//
// Otherwise the 64-key kernel, which halves the QK issue cost per key of the
// 32-key kernel and after a selection stage is the faster one for any row
// count (decode 32K: 27.9 against 29.5 us per step; four 131K rows: 49.0
// against 52.1 us).  Its query prologue (blocks 0-5 into TMEM through
// registers) is slower than the 32-key kernel's single TMA load, and only a
// launch with no preceding stage to hide behind pays for it: the dense
// short-context attention with few chunks per SM (one 2K row: 14.6 against
// 13.9 us) keeps the 32-key kernel unless 2 * rows * 64-key chunks reaches
// kMlaWideMinChunksPerSm times the SM count.
//
// DSA_ATTENTION_KERNEL=pair|wide|narrow in the environment (read once per
// process) forces one of the three for every launch, for measurements.
constexpr int kMlaWideMinChunksPerSm = 8;
constexpr int kMlaPairMinChunksPerSlot = 4;

namespace {
int forced_kernel() {  // 0: automatic, else the forced chunk size
  static const int forced = [] {
    const char* e = std::getenv("DSA_ATTENTION_KERNEL");
    if (!e) return 0;
    if (!std::strcmp(e, "pair")) return kMlaPairChunk;
    if (!std::strcmp(e, "wide")) return kMlaWideChunk;
    if (!std::strcmp(e, "narrow")) return kChunk;
    return 0;
  }();
  return forced;
}
}  // namespace

int mla_chunk(int n_rows, int k, bool dense) {
  if (const int f = forced_kernel()) return f;
  const int64_t sms = device_info().sm_count;
  const int64_t n128 = (k + kMlaPairChunk - 1) / kMlaPairChunk;
  if ((int64_t)n_rows * n128 >= kMlaPairMinChunksPerSlot * (sms / 2)) return kMlaPairChunk;
  if (!dense) return kMlaWideChunk;
  const int64_t n64 = (k + kMlaWideChunk - 1) / kMlaWideChunk;
  return 2 * (int64_t)n_rows * n64 >= kMlaWideMinChunksPerSm * sms ? kMlaWideChunk : kChunk;
}

// Splits of a row's index list.  Every split is a pair of CTAs (one per value
// half, or the QK and PV sides of the pair kernel; one CTA per SM for shared
// memory), so n_rows x splits x 2 CTAs run in ceil(that / SMs) waves, each
// costing its chunks (1000 per 32 keys for the 32- and 64-key kernels, 1000
// per 64 keys for the pair kernel) plus about 1500 of fixed work (query tile,
// epilogue; 2500 for the pair kernel); every (row, split) partial costs the
// combine about 17 at H = 128 (measured on B200).  The split count minimises
// that estimate, ties going to fewer splits, with at least 64 keys per split
// (fewer keys per split double the partials' traffic for too little gain).
static_assert(DSA_MAX_TOPK / 64 <= kMaxSplits, "the combine holds every split of a row in registers");

int mla_num_splits(int n_rows, int k, int H, bool dense) {
  const int chunk = mla_chunk(n_rows, k, dense);
  const bool pair = chunk == kMlaPairChunk;
  const int n_chunks = (k + chunk - 1) / chunk;
  const int64_t sms = device_info().sm_count;
  int max_splits = n_chunks * chunk / 64;
  if (max_splits > n_chunks) max_splits = n_chunks;
  if (max_splits < 1) max_splits = 1;
  const int64_t per_chunk = pair ? 2000 : 1000 * (int64_t)chunk / 32;
  const int64_t fixed = pair ? 2500 : 1500;
  int best = 1;
  int64_t best_cost = -1;
  for (int ns = 1; ns <= max_splits; ++ns) {
    const int cps = (n_chunks + ns - 1) / ns;
    if ((n_chunks + cps - 1) / cps != ns) continue;  // same chunks per split as a smaller count
    const int64_t waves = ((int64_t)n_rows * ns * 2 + sms - 1) / sms;
    const int64_t cost = waves * (per_chunk * cps + fixed) + (ns > 1 ? (int64_t)n_rows * ns * 17 * H / 128 : 0);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = ns;
    }
  }
  return best;
}

namespace {
inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }
// Workspace: [split partials bf16][(max, sum) fp32], sized for whichever of
// the index-list and dense launches splits more
size_t mla_partials_bytes(int n_rows, int H, int k) {
  const int ns = std::max(mla_num_splits(n_rows, k, H, false), mla_num_splits(n_rows, k, H, true));
  if (ns <= 1) return 0;
  return align256((size_t)n_rows * ns * H * (kDV * sizeof(__nv_bfloat16) + 2 * sizeof(float)));
}
}  // namespace

size_t mla_workspace_bytes(int n_rows, int H, int k) {
  return mla_partials_bytes(n_rows, H, k);
}

namespace {
std::atomic<int> g_stall_left{0};
std::atomic<uint64_t> g_stall_limit_ns{0};
}  // namespace

void take_attention_debug(MlaParams& p) {
  p.debug_stall = 0;
  p.wait_limit_ns = kWaitLimitNs;
  int left = g_stall_left.load();
  while (left > 0 && !g_stall_left.compare_exchange_weak(left, left - 1)) {
  }
  if (left > 0) {
    p.debug_stall = 1;
    p.wait_limit_ns = g_stall_limit_ns.load();
  }
}

int launch_sparse_mla(const MlaArgs& a, cudaStream_t stream) {
  const int n_rows = a.B * a.T;
  const bool dense = a.indices == nullptr;
  const int ns = mla_num_splits(n_rows, a.k, a.H, dense);
  const int chunk = mla_chunk(n_rows, a.k, dense);
  const int n_chunks = (a.k + chunk - 1) / chunk;
  MlaParams p;
  p.q = reinterpret_cast<const __nv_bfloat16*>(a.q);
  p.kv = reinterpret_cast<const __nv_bfloat16*>(a.kv);
  p.off = a.offsets;
  p.idx = a.indices;
  p.T = a.T;
  p.H = a.H;
  p.k = a.k;
  p.n_splits = ns;
  p.cps = (n_chunks + ns - 1) / ns;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.kv_rows = a.kv_rows;
  p.out = a.out;
  p.out_bf16 = a.out_dtype == DSA_BF16;
  p.lse = a.lse;
  p.ws_o = nullptr;
  p.ws_ml = nullptr;
  p.status = a.status;
  p.early_inputs = a.early_inputs ? 1 : 0;
  p.dense = a.indices == nullptr ? 1 : 0;
  take_attention_debug(p);
  if (ns > 1) {
    p.ws_o = reinterpret_cast<__nv_bfloat16*>(a.workspace);  // partials first
    p.ws_ml = reinterpret_cast<float*>(p.ws_o + (size_t)n_rows * ns * a.H * kDV);
  }
  CUtensorMap tq, tout;
  if (!make_tmap_2d(&tq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kDQK, (uint64_t)n_rows * a.H,
                    kDQK * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  // where the epilogue's boxes go: the split partials (bf16), or the output
  bool tm_ok;
  if (ns > 1)
    tm_ok = make_tmap_2d(&tout, p.ws_o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kDV, (uint64_t)n_rows * ns * a.H,
                         kDV * 2, 64, (uint32_t)a.H, CU_TENSOR_MAP_SWIZZLE_128B);
  else if (p.out_bf16)
    tm_ok = make_tmap_2d(&tout, a.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kDV, (uint64_t)n_rows * a.H, kDV * 2, 64,
                         (uint32_t)a.H, CU_TENSOR_MAP_SWIZZLE_128B);
  else
    tm_ok = make_tmap_2d(&tout, a.out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, kDV, (uint64_t)n_rows * a.H, kDV * 4, 32,
                         (uint32_t)a.H, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!tm_ok) return DSA_ERR_CUDA;
  static PerDeviceOnce attr;
  if (attr.run([] { return cudaFuncSetAttribute(sparse_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                kSmemBytes); }) != cudaSuccess)
    return DSA_ERR_CUDA;
  const int64_t grid = (int64_t)n_rows * ns * 2;
  const cudaError_t e =
      chunk == kMlaPairChunk   ? launch_sparse_mla_pair(tq, tout, p, (unsigned)(grid / 2), stream)
      : chunk == kMlaWideChunk ? launch_sparse_mla_wide(tq, tout, p, (unsigned)grid, stream)
                               : launch_pdl(sparse_mla_kernel, dim3((unsigned)grid), dim3(kThreads), kSmemBytes,
                                            stream, tq, tout, p);
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  if (ns > 1 && launch_combine(p, n_rows, a.H, stream) != cudaSuccess) return DSA_ERR_CUDA;
  return DSA_OK;
}

}  // namespace dsa

extern "C" int dsa_debug_stall_attention(int n_launches, uint64_t wait_limit_ns) {
  if (n_launches < 0) return DSA_ERR_INVALID_ARG;
  if (n_launches > 0 && (wait_limit_ns < 1000000ull || wait_limit_ns > 1000000000ull)) return DSA_ERR_INVALID_ARG;
  dsa::g_stall_limit_ns.store(wait_limit_ns);
  dsa::g_stall_left.store(n_launches);
  return DSA_OK;
}
