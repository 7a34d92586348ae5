// sparse_mla_wide.cu -- stage 3 for long index lists: absorbed MLA over the
// selected latent rows in 64-key chunks.
//
// "DeepSeek-V3.2-Exp - Apply sparse mask", MQA decode listing (the same
// computation as sparse_mla.cu; see there for the formulas).  This kernel
// serves every launch with an index list (after a selection stage: decode
// at any batch, causal prefill), where 64-key chunks halve the QK issue cost
// per key.  The dense short-context launch (no index list) uses it too once
// 2 x rows x 64-key chunks reach 8 per SM; below that the 32-key kernel,
// whose query prologue is a single TMA load, stays ahead.
//
// Work unit (one CTA, one per SM): query row r, value half v (latent columns
// [256v, 256v+256)), split sp (a contiguous range of 64-key chunks of the
// row's index list).  Per chunk i:
//   S_i = Q . Kv_i^T          M=128 heads, N=64 keys, K=576  (tcgen05, TMEM)
//   P_i = exp2(S_i*scale*log2e - m)  in bf16                  (CUDA cores)
//   O  += P_i . Kv_i[:, half] M=128, N=256, K=64              (tcgen05, TMEM)
// with the lazy running max of the 32-key kernel (rescale above 2^8).
//
// A tcgen05.mma of M = 128, K = 16 costs about 46 cycles to issue for any N
// up to 64.  A 64-key chunk is 72 KB, so shared memory keeps only what must
// be there and TMEM takes the rest of the query:
//   TMEM (512 columns): O half [0,256), one 64-column S buffer [256,320)
//     (released as soon as softmax has it in registers), query blocks 0-5
//     (latent 0-383) as the A operand of QK [320,512), written by the
//     softmax threads (row h in lane h, two bf16 per column).
//   Shared memory: query blocks 6-8 (latent 384-511, rope; TMA), two stages
//     of 64 gathered rows (swizzled 64-column blocks), two P buffers.
// The gathered stage is K-major for Q.K^T and, read as MN-major, the B
// operand of P.V: one copy of each row serves both products.
//
// Roles: warps 0-3 softmax + epilogue (thread = head = TMEM lane),
//        warps 4-7 row gather, warp 8 TMEM allocator + MMA issuer.
#include <cuda.h>
#include <cuda_bf16.h>

#include "dsa_internal.h"
#include "sm100.cuh"

namespace dsa {
namespace {

constexpr int kChunk = kMlaWideChunk;               // keys per chunk: the QK MMA's N
constexpr int kKB = kDQK / 64;                      // 9 column blocks of 64
constexpr int kQTmemBlocks = 6;                     // query blocks 0-5: TMEM (tensor-core A operand)
constexpr int kQSmemBlocks = kKB - kQTmemBlocks;    // query blocks 6-8: shared memory
constexpr int kQBytes = kQSmemBlocks * 128 * 128;   // 49152
constexpr int kStages = 2;
constexpr int kBlockBytes = kChunk * 128;           // one 64-column block of a chunk: 8192
constexpr int kKvBytes = kKB * kBlockBytes;         // 73728
constexpr int kPBytes = 128 * kChunk * 2;           // 16384
constexpr int kOffQ = 0;
constexpr int kOffKv = kOffQ + kQBytes;
constexpr int kOffP = kOffKv + kStages * kKvBytes;  // two P buffers
constexpr int kOffBar = kOffP + 2 * kPBytes;
// q_full, kv_full[2], kv_empty[2], s_full, s_empty, p_full[2], pv_done[2], drain, kv_first
constexpr int kNumBar = 13;
constexpr int kOffMisc = kOffBar + kNumBar * 8;
constexpr int kStageBlock = 128 * 128;              // epilogue staging: one box, 128 rows x 128 B
static_assert(8 * kStageBlock <= kOffP, "the staged output fits where the query blocks and key stages were");
constexpr int kMaxChunks = (DSA_MAX_TOPK + kChunk - 1) / kChunk;
constexpr int kMiscBytes = 64 + 8 * kMaxChunks;     // MlaMisc
constexpr int kSmemBytes = kOffMisc + kMiscBytes + 1024;
constexpr int kThreads = 288;
constexpr int kTmemCols = 512;
constexpr uint32_t kTmemS = 256;                    // the 64-column S buffer
constexpr uint32_t kTmemQ = 320;                    // query blocks 0-5, 32 columns each
static_assert(kTmemQ + 32 * kQTmemBlocks == kTmemCols, "TMEM budget: O half, S, query blocks");
constexpr uint32_t kIdescQK = idesc_bf16(128, kChunk);
constexpr uint32_t kIdescPV = idesc_bf16(128, 256, /*b_mn_major=*/true);
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffKv % 1024 == 0 && kOffP % 1024 == 0, "alignment");

struct MlaMisc {
  int tmem_base, abort, n_chunks, last_valid, pad[12];
  unsigned long long vmask[kMaxChunks];  // per chunk of this split: bit j = position valid
};
static_assert(sizeof(MlaMisc) == kMiscBytes, "shared-memory budget of the bookkeeping block");


// Position selected at slot j of row r: the index list's entry, or (dense
// mode, every prefix shorter than k) slot j itself while j < the prefix length.
__device__ __forceinline__ int32_t selected_pos(const int32_t* __restrict__ idx_row, bool dense, int j, int L) {
  return dense ? (j < L ? j : -1) : idx_row[j];
}

__device__ __forceinline__ bool index_ok(int32_t idx, int E) { return idx >= 0 && idx < E; }

__global__ void __launch_bounds__(kThreads, 1)
    sparse_mla_wide_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_out,
                      const MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kOffBar;
  const uint32_t q_full = bar0;
  auto kv_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (3 + s); };
  const uint32_t s_full = bar0 + 8u * 5;
  const uint32_t s_empty = bar0 + 8u * 6;
  auto p_full = [&](int b) { return bar0 + 8u * (7 + b); };
  auto pv_done = [&](int b) { return bar0 + 8u * (9 + b); };
  const uint32_t drain = bar0 + 8u * 11;
  // The split's first chunk is gathered into stage 0 by warps 0-7 together
  // (the softmax warps are idle until its scores exist), with its own
  // barrier; stage 0's kv_full phases then start at chunk 2.
  const uint32_t kv_first = bar0 + 8u * 12;
  MlaMisc* misc = reinterpret_cast<MlaMisc*>(smem + kOffMisc);
  volatile int* abort = &misc->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (!p.early_inputs) grid_dependency_wait();  // q and the offsets may come from the previous kernel
  const int v = blockIdx.x & 1;
  const int sp = (blockIdx.x >> 1) % p.n_splits;
  // rows in reverse launch order: a causal prefill's late rows keep the most
  // keys, and launching them first leaves the short rows to fill the last
  // wave (prefill 4K attention 4.27 -> 4.20 ms)
  const int r = (int)(gridDim.x / (2 * p.n_splits)) - 1 - (int)((blockIdx.x >> 1) / p.n_splits);
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
  if (threadIdx.x < kMaxChunks) misc->vmask[threadIdx.x] = 0ull;
  if (warp == 8) {
    if (lane == 0) {
      // TMA bytes of blocks 6-8, the 128 threads writing blocks 0-5 (+ the test
      // hook's missing arrival)
      mbar_init(q_full, 1 + 128 + p.debug_stall);
      for (int s = 0; s < kStages; ++s) {
        mbar_init(kv_full(s), 128);  // one cp.async arrival per gather thread
        mbar_init(kv_empty(s), 1);
      }
      mbar_init(s_full, 1);
      mbar_init(s_empty, 128);
      for (int i = 0; i < 2; ++i) {
        mbar_init(p_full(i), 128);
        mbar_init(pv_done(i), 1);
      }
      mbar_init(drain, 1);
      mbar_init(kv_first, 256);
      fence_mbar_init();
      if (geo_ok) {
        mbar_arrive_expect_tx(q_full, kQBytes);
        for (int j = 0; j < kQSmemBlocks; ++j)
          tma_load_2d(sbase + kOffQ + j * 16384, &tm_q, (kQTmemBlocks + j) * 64, r * p.H, q_full);
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
  const int h = threadIdx.x;  // softmax / epilogue threads: head = TMEM lane
  if (warp < 4 && geo_ok) {
    // Query blocks 0-5 of head h go to TMEM lane h, two bf16 per column: the
    // A operand of the first 24 QK MMAs of every chunk.  Rows past H are zero.
    const uint32_t lane_q = tmem + (static_cast<uint32_t>(warp * 32) << 16) + kTmemQ;
    const bool live = h < p.H;
    const uint4* qrow = reinterpret_cast<const uint4*>(p.q + ((int64_t)r * p.H + (live ? h : 0)) * kDQK);
#pragma unroll
    for (int half = 0; half < 2; ++half) {  // three blocks' loads in flight at a time
      uint4 qv[24];
#pragma unroll
      for (int u = 0; u < 24; ++u) qv[u] = live ? __ldg(qrow + 24 * half + u) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int g = 0; g < 3; ++g) {
        uint32_t w[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          w[4 * u] = qv[8 * g + u].x;
          w[4 * u + 1] = qv[8 * g + u].y;
          w[4 * u + 2] = qv[8 * g + u].z;
          w[4 * u + 3] = qv[8 * g + u].w;
        }
        tmem_st32(lane_q + 96 * half + 32 * g, w);
      }
    }
    tc_wait_st();
    tc_fence_before();
    mbar_arrive(q_full);
  }
  grid_dependency_wait();  // the indices come from the previous kernel
  allow_dependents_launch();

  // ---- the split's first chunk: warps 0-7 copy 8 rows each into stage 0
  // right away, before the validity pass below (a single SM's gather rate
  // grows with the threads issuing it; a decode row's split often has just
  // this one chunk).  Invalid positions are zero-filled.
  if (geo_ok && warp < 8) {
    const int pos0 = c_begin * kChunk + 8 * warp + lane;
    const int32_t my_id = (lane < 8 && pos0 < p.k) ? selected_pos(idx_row, dense, pos0, L_row) : -1;
#pragma unroll 2
    for (int rr = 0; rr < 8; ++rr) {
      const int jr = 8 * warp + rr;
      const int32_t id = __shfl_sync(0xffffffffu, my_id, rr);
      const bool valid = index_ok(id, E);
      const __nv_bfloat16* src = valid ? p.kv + ((int64_t)base_row + id) * kDQK : p.kv;
      const uint32_t dst_row = sbase + kOffKv + (jr >> 3) * 1024 + (jr & 7) * 128;
#pragma unroll
      for (int u = 0; u < 3; ++u) {
        const int c = lane + 32 * u;  // 16-byte piece of the 72 in a row
        if (c < kDQK / 8) {
          const int kb = c >> 3, cc = c & 7;
          cp_async_16(dst_row + kb * kBlockBytes + ((cc ^ (jr & 7)) << 4), src + c * 8, valid ? 16u : 0u);
        }
      }
    }
    cp_async_mbar_arrive(kv_first);
  }

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
      unsigned long long m = 0;
#pragma unroll
      for (int hh = 0; hh < kChunk / 32; ++hh) {
        const bool valid = index_ok(ids[u][hh], E);
        if (!valid && ids[u][hh] != -1) report(p.status, DSA_ERR_BAD_INDEX);
        m |= static_cast<unsigned long long>(__ballot_sync(0xffffffffu, valid)) << (32 * hh);
      }
      if (lane == 0) misc->vmask[c] = m;
      if (m) lv = (c_begin + c) * kChunk + 63 - __clzll((long long)m);
    }
    if (lane == 0 && lv >= 0) atomicMax(&misc->last_valid, lv);
  } else if (threadIdx.x == 0) {
    report(p.status, DSA_ERR_BAD_OFFSETS);
  }
  __syncthreads();
  const int n_my = misc->last_valid < 0 ? 0 : misc->last_valid / kChunk - c_begin + 1;

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
    if (warp == 8 && lane == 0 && geo_ok) {  // the query tile and the first chunk must land before the CTA exits
      volatile int never = 0;
      mbar_wait(q_full, 0, &never, 10000000ull);
      mbar_wait(kv_first, 0, &never, 10000000ull);
    }
  } else if (warp == 8) {
    // -------------------------------------------------------------- MMA issuer
    // QK of chunk i and PV of chunk j < i touch different TMEM (S, O) and
    // shared memory (stage i; stage j and P buffer j), so they are issued in
    // whichever order their inputs arrive: QK(i) once chunk i has landed and
    // softmax(i-1) has read S into registers; PV(j) once softmax(j) has
    // written P(j).  Each PV frees its stage for the load of chunk j + 2.
    // A QK's 36 MMAs go out in two branch-free runs (query blocks in TMEM,
    // then in shared memory).  Between the two, a PV whose P has meanwhile
    // been written goes in, so its stage is freed for the next load about
    // half a QK sooner (polling between single MMAs measured slower).
    if (lane == 0) {
      int n_qk = 0, n_pv = 0;
      bool ok = mbar_wait(q_full, 0, abort, p.wait_limit_ns);
      // Descriptors differ only in the start-address field (address >> 4 in
      // the low 14 bits, no carry below 256 KiB): built once, offset per MMA.
      const uint64_t qk_a0 = smem_desc(sbase + kOffQ, 16, 1024, kSwizzle128B);
      const uint64_t qk_b0 = smem_desc(sbase + kOffKv, 16, 1024, kSwizzle128B);
      const uint64_t pv_a0 = smem_desc(sbase + kOffP, 128, 1024, kSwizzleNone);
      const uint64_t pv_b0 = smem_desc(sbase + kOffKv + (4 * v) * kBlockBytes, kBlockBytes, 1024, kSwizzle128B);
      // chunk i has landed: the first chunk on its own barrier, stage 0's
      // later chunks (2, 4, ...) on kv_full(0) phases 0, 1, ...
      auto kv_ready = [&](int i) -> bool {
        if (i == 0) return mbar_try_wait(kv_first, 0);
        const int st = i % kStages;
        return mbar_try_wait(kv_full(st), (i / kStages - (st == 0 ? 1 : 0)) & 1);
      };
      // PV of chunk n_pv (its P is in shared memory; p_full has been seen)
      auto issue_pv = [&]() {
        const int j = n_pv;
        tc_fence_after();
        const uint64_t ad0 = pv_a0 + (uint64_t)(((j & 1) * kPBytes) >> 4);
        const uint64_t bd0 = pv_b0 + (uint64_t)(((j % kStages) * kKvBytes) >> 4);
#pragma unroll
        for (int ks = 0; ks < kChunk / 16; ++ks)
          mma_f16_ss(tmem, ad0 + (uint64_t)((ks * 256) >> 4), bd0 + (uint64_t)((ks * 2048) >> 4), kIdescPV,
                     (j > 0 || ks > 0) ? 1u : 0u);
        tc_commit(pv_done(j & 1));
        tc_commit(kv_empty(j % kStages));
        ++n_pv;
      };
      const uint64_t t0 = globaltimer_ns();
      uint32_t spins = 0;
      while (ok && n_pv < n_my) {
        bool progressed = false;
        if (n_qk < n_my && (n_qk == 0 || mbar_try_wait(s_empty, (n_qk - 1) & 1)) && kv_ready(n_qk)) {
          const int st = n_qk % kStages;
          fence_proxy_async_smem();  // rows written by cp.async, read by the tensor core
          tc_fence_after();
          const uint64_t bst = qk_b0 + (uint64_t)((st * kKvBytes) >> 4);
          const uint32_t d = tmem + kTmemS;
          // Two branch-free loops (a branch between the MMA forms inside one
          // unrolled loop slowed the issue): query blocks in TMEM, then in
          // shared memory.
#pragma unroll 1
          for (int kb = 0; kb < kQTmemBlocks; ++kb) {
            const uint64_t bkb = bst + (uint64_t)((kb * kBlockBytes) >> 4);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_f16_ts(d, tmem + kTmemQ + kb * 32 + ks * 8, bkb + (uint64_t)ks * 2, kIdescQK,
                         (kb | ks) ? 1u : 0u);
          }
          if (n_pv < n_qk && mbar_try_wait(p_full(n_pv & 1), (n_pv >> 1) & 1)) issue_pv();
#pragma unroll 1
          for (int kb = kQTmemBlocks; kb < kKB; ++kb) {
            const uint64_t akb = qk_a0 + (uint64_t)(((kb - kQTmemBlocks) * 16384) >> 4);
            const uint64_t bkb = bst + (uint64_t)((kb * kBlockBytes) >> 4);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_f16_ss(d, akb + (uint64_t)ks * 2, bkb + (uint64_t)ks * 2, kIdescQK, 1u);
          }
          tc_commit(s_full);
          ++n_qk;
          progressed = true;
        }
        if (n_pv < n_qk && mbar_try_wait(p_full(n_pv & 1), (n_pv >> 1) & 1)) {
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
      if (*abort) {
        // tensor-core work must finish before TMEM is released, and the
        // query tile must have landed before the CTA exits
        volatile int never = 0;
        tc_commit(drain);
        mbar_wait(drain, 0, &never, 10000000ull);
        mbar_wait(q_full, 0, &never, 10000000ull);
        mbar_wait(kv_first, 0, &never, 10000000ull);
      }
    }
  } else if (warp >= 4) {
    // -------------------------------------------------------------- row gather
    // From the second chunk on (the first was copied above), warp 4 + gw
    // copies rows 16gw .. 16gw+15 of every chunk, one row at a time, so each
    // copy instruction reads 512 contiguous bytes of a row.  Completion is
    // signalled by the copies themselves (cp.async arrival on the stage's
    // barrier), so both stages are in flight from the start; the next
    // chunk's indices are read while the current one is issued.
    const int gw = warp - 4;
    const __nv_bfloat16* kv = p.kv;
    auto row_id = [&](int i) -> int32_t {
      if (lane >= 16) return -1;
      const int pos = (c_begin + i) * kChunk + gw * 16 + lane;
      return pos < p.k ? selected_pos(idx_row, dense, pos, L_row) : -1;
    };
    int32_t next_id = n_my > 1 ? row_id(1) : -1;
    for (int i = 1; i < n_my; ++i) {
      const int st = i % kStages;
      const int32_t my_id = next_id;
      if (i + 1 < n_my) next_id = row_id(i + 1);
      if (!__all_sync(0xffffffffu, mbar_wait(kv_empty(st), ((i / kStages) & 1) ^ 1, abort, p.wait_limit_ns)))
        break;
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
            cp_async_16(dst_row + kb * kBlockBytes + ((cc ^ (jr & 7)) << 4), src + c * 8, valid ? 16u : 0u);
          }
        }
      }
      cp_async_mbar_arrive(kv_full(st));
    }
    cp_async_wait<0>();
  } else {
    // -------------------------------------------------------------- softmax + epilogue
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int i = 0; i < n_my; ++i) {
      const int pb = i & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(s_full, i & 1, abort, p.wait_limit_ns));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[64];
      tmem_ld32(lane_addr + kTmemS, *reinterpret_cast<uint32_t(*)[32]>(sv));
      tmem_ld32(lane_addr + kTmemS + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive(s_empty);  // S is in registers: the next chunk's QK may overwrite it
      const unsigned long long vm = misc->vmask[i];  // validity of the chunk's 64 positions
      float mc = -INFINITY;
      if (vm == ~0ull) {  // every position valid (the common case): scale in pairs
#pragma unroll
        for (int j = 0; j < 64; j += 2) {
          const float2 x2 = __fmul2_rn(make_float2(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])),
                                       make_float2(p.scale_log2, p.scale_log2));
          sv[j] = __float_as_uint(x2.x);
          sv[j + 1] = __float_as_uint(x2.y);
          mc = fmaxf(mc, fmaxf(x2.x, x2.y));
        }
      } else {
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const float xj = ((vm >> j) & 1ull) ? __uint_as_float(sv[j]) * p.scale_log2 : -INFINITY;
          sv[j] = __float_as_uint(xj);
          mc = fmaxf(mc, xj);
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
      uint32_t pk[32];
      float2 l2 = make_float2(0.f, 0.f);
      const float m_sub = m_new == -INFINITY ? 0.f : m_new;  // nothing valid yet: every x is -inf
#pragma unroll
      for (int j = 0; j < 64; j += 2) {
        const float2 d = __fadd2_rn(make_float2(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])),
                                    make_float2(-m_sub, -m_sub));
        const __nv_bfloat162 pbf = __floats2bfloat162_rn(ex2_approx(d.x), ex2_approx(d.y));
        l2 = __fadd2_rn(l2, __bfloat1622float2(pbf));
        pk[j / 2] = *reinterpret_cast<const uint32_t*>(&pbf);
      }
      const float l_chunk = l2.x + l2.y;
      if (__any_sync(0xffffffffu, resc)) {
        // O is rescaled in TMEM: every earlier PV must have completed (the
        // last one, PV(i-1), completes after all the others)
        ok = __all_sync(0xffffffffu, mbar_wait(pv_done((i - 1) & 1), ((i - 1) >> 1) & 1, abort, p.wait_limit_ns));
        if (!ok) break;
        tc_fence_after();
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
      if (i >= 2) {  // P buffer pb was last read by PV(i-2)
        ok = __all_sync(0xffffffffu, mbar_wait(pv_done(pb), ((i - 2) >> 1) & 1, abort, p.wait_limit_ns));
        if (!ok) break;
      }
      l_run = l_run * alpha + l_chunk;
      m_run = m_new;
      // P row h, K-major without swizzle: 8-row x 16-byte core matrices,
      // 128 bytes apart along K, 1024 bytes apart along M.
      uint8_t* prow = smem + kOffP + pb * kPBytes + (h >> 3) * 1024 + (h & 7) * 16;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(prow + c * 128) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full(pb));
    }
    if (ok)
      ok = __all_sync(0xffffffffu,
                      mbar_wait(pv_done((n_my - 1) & 1), ((n_my - 1) >> 1) & 1, abort, p.wait_limit_ns));
    // Every MMA has completed, so the query blocks and key stages are free:
    // the 128 x 256 result is staged there as 128-byte-swizzled boxes of 32
    // fp32 (or 64 bf16) columns, one thread per head row, and written by TMA
    // tensor stores (the output's tensor map has one box per block).  Each
    // 64-column slice is stored as soon as it is staged, so the copy of one
    // overlaps the staging of the next.
    const bool final_out = p.n_splits == 1;
    const bool as_bf16 = !final_out || p.out_bf16;  // partials are bf16 too
    const int y_out = final_out ? r * p.H : (r * p.n_splits + sp) * p.H;
    if (ok) tc_fence_after();
    const float mul = final_out ? (l_run > 0.f ? 1.f / l_run : 0.f) : 1.f;
    uint8_t* stage = smem;
    const int sw = h & 7;
#pragma unroll 1
    for (int cb2 = 0; cb2 < 8; cb2 += 2) {
      if (ok) {
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
        fence_proxy_async_smem();
      }
      named_barrier_sync(1, 128);  // every epilogue warp, whatever its wait outcome
      if (threadIdx.x == 0 && !*abort) {
        if (as_bf16) {
          tma_store_2d(&tm_out, sbase + (cb2 >> 1) * kStageBlock, 256 * v + 32 * cb2, y_out);
        } else {
          tma_store_2d(&tm_out, sbase + cb2 * kStageBlock, 256 * v + 32 * cb2, y_out);
          tma_store_2d(&tm_out, sbase + (cb2 + 1) * kStageBlock, 256 * v + 32 * (cb2 + 1), y_out);
        }
        bulk_commit();
      }
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

  cp_async_wait<0>();  // the first chunk's copies of warps 0-7
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort) report(p.status, DSA_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_sparse_mla_wide(const CUtensorMap& tq, const CUtensorMap& tout,
                                   const MlaParams& p, unsigned grid, cudaStream_t stream) {
  static PerDeviceOnce attr;
  const cudaError_t e = attr.run(
      [] { return cudaFuncSetAttribute(sparse_mla_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes); });
  if (e != cudaSuccess) return e;
  return launch_pdl(sparse_mla_wide_kernel, dim3(grid), dim3(kThreads), kSmemBytes, stream, tq, tout, p);
}

}  // namespace dsa
