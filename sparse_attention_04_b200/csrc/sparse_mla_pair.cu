// sparse_mla_pair.cu -- stage 3 for launches with many 128-key chunks per SM
// (causal prefill, large decode batches): absorbed MLA over the selected
// latent rows, with the work of one (row, split) divided by role between the
// two CTAs of a thread-block cluster.
//
// "DeepSeek-V3.2-Exp - Apply sparse mask", MQA decode listing (the same
// computation as sparse_mla.cu; see there for the formulas).
//
// Why a pair.  A tcgen05.mma of M = 128, K = 16 issues in about 46 cycles for
// any N up to 64 and in N/2 cycles above, so the score tile S = Q.Kv^T runs
// at the tensor core's full rate only from N = 128 keys per chunk.  One SM
// cannot hold the query (147 KB), a 128-key chunk of latent rows (147 KB), S
// and the 128 x 512 fp32 output together; the 64-key kernel therefore splits
// the value columns over two CTAs, each of which computes the same S.  Here
// the two CTAs split by role instead, and S is computed once:
//
//   CTA 0 (QK side).  Query blocks 0-7 (latent 0-511) sit in TMEM as the A
//     operand of S, block 8 (rope) in shared memory.  The chunk's rows stream
//     through a ring of three 48 KB slots, each three 64-column blocks of the
//     128 rows (swizzled, K-major); every slot is read once by the QK MMAs.
//     S goes to one of two 128-column TMEM buffers.  Softmax runs in
//     registers, thread = head = TMEM lane, with the lazy running max of
//     sparse_mla.cu (raised only when a chunk exceeds it by more than 2^8).
//     Each thread writes its bf16 P row and its rescale factor into one of
//     two local staging buffers and moves on to the next chunk; warp 15 sends
//     each staged message to CTA 1 with one bulk copy (shared::cta to
//     shared::cluster), whose bytes complete on CTA 1's barrier.
//   CTA 1 (PV side).  O (128 heads x 512 latent, fp32) fills all 512 TMEM
//     columns.  The chunk's latent columns 0-511 stream through a ring of
//     four 32 KB slots (two 64-column blocks each).  Before P.V of a chunk
//     whose max was raised, each thread rescales its O row; then
//     O += P.V runs as four N = 128 quarters.  The epilogue normalises O
//     (or keeps the split's unnormalised partial) and writes it with TMA.
//   The completion of P.V(i) arrives on a barrier at the same offset in both
//     CTAs (tcgen05.commit multicast): CTA 0 may then overwrite P buffer
//     i & 1.
//
// Each latent row is read by both CTAs (576 + 512 columns), about what the
// 64-key kernel's two value-half CTAs read (2 x 576); the QK MMAs are issued
// once per key instead of twice, at N = 128 instead of 64.
//
// Roles in each CTA: warps 0-3 softmax (CTA 0) or rescale + epilogue (CTA 1),
// warp 12 TMEM allocator + MMA issuer, warp 15 message sender (CTA 0), the
// other warps (4-11, 13-14; and 15 in CTA 1) row gather.
#include <cuda.h>
#include <cuda_bf16.h>

#include "dsa_internal.h"
#include "sm100.cuh"

namespace dsa {
namespace {

constexpr int kChunk = kMlaPairChunk;               // keys per chunk: the QK MMA's N
constexpr int kKB = kDQK / 64;                      // 9 column blocks of 64
constexpr int kBlockBytes = kChunk * 128;           // one 64-column block of a chunk: 16384
constexpr int kMaxChunks = (DSA_MAX_TOPK + kChunk - 1) / kChunk;  // 16

constexpr int kPBytes = 128 * kChunk * 2;           // 32768: P, 128 heads x 128 keys bf16
constexpr uint32_t kPMsgBytes = kPBytes + 128 * 4;  // one chunk's message to CTA 1: P, then alpha per head
// ---- CTA 0 shared memory
constexpr int kQ8Off = 0;                           // query block 8 (rope), TMA
constexpr int kKSlotBlocks = 3;
constexpr int kKSlotsPerChunk = kKB / kKSlotBlocks;  // 3
constexpr int kKSlotBytes = kKSlotBlocks * kBlockBytes;  // 49152
constexpr int kKSlots = 3;
constexpr int kKRingOff = kBlockBytes;
constexpr int kStageOff = kKRingOff + kKSlots * kKSlotBytes;  // 163840: two messages, staged for the copy
constexpr int kKEnd = kStageOff + 2 * (int)kPMsgBytes;        // 230400
// ---- CTA 1 shared memory
constexpr int kVSlotBlocks = 2;
constexpr int kVSlotBytes = kVSlotBlocks * kBlockBytes;  // 32768
constexpr int kVSlots = 4;                          // = quarters per chunk: slot q holds quarter q
constexpr int kVRingOff = 0;
constexpr int kPOff = kVRingOff + kVSlots * kVSlotBytes;  // 131072: two message buffers (P, alpha)
constexpr int kMLOff = kPOff + 2 * (int)kPMsgBytes;  // 197632: (m, l) per head from CTA 0
constexpr int kVEnd = kMLOff + 128 * 8;             // 198656
// ---- both
constexpr int kOffBar = kKEnd > kVEnd ? kKEnd : kVEnd;
enum Bar : int {
  kQFull = 0,
  kKFull = 1,        // [kKSlots]   CTA 0
  kKEmpty = 5,       // [kKSlots]   CTA 0
  kSFull = 9,        // [2]         CTA 0
  kSEmpty = 11,      // [2]         CTA 0
  kPvDone = 13,      // [2]         both: P.V(i) complete (multicast commit)
  kVFull = 15,       // [kVSlots]   CTA 1
  kVEmpty = 19,      // [kVSlots]   CTA 1
  kPFull = 23,       // [2]         CTA 1: P(i) written by CTA 0
  kReady = 25,       // [2]         CTA 1: O rescaled for chunk i
  kMLFull = 27,      //             CTA 1: CTA 0's (m, l)
  kDrain = 28,
  kStageFree = 29,   // [2]         CTA 0: the copy of message i has landed in CTA 1 (staging i & 1 free)
  kStaged = 31,      // [2]         CTA 0: message i is staged (128 softmax arrivals)
  kNumBar = 33
};
constexpr int kStageBlock = 128 * 128;              // epilogue staging: one box, 128 rows x 128 B
constexpr int kOffMisc = kOffBar + kNumBar * 8;
struct PairMisc {
  int tmem_base, abort, last_valid, pad;
  uint32_t vmask[kMaxChunks][kChunk / 32];  // per chunk of this split: bit = position valid
};
constexpr int kSmemBytes = kOffMisc + (int)sizeof(PairMisc) + 1024;
// Warps: 0-3 softmax (CTA 0) or rescale + epilogue (CTA 1), warp 12 TMEM
// allocator + MMA issuer, warp 15 message sender (CTA 0), the other ten (or
// eleven, in CTA 1) gather rows.  A single SM's
// cp.async gather rate grows with the number of threads issuing it (about 35,
// 55 and 75 GB/s with 128, 256 and 384 threads, measured on B200), so most of
// the CTA gathers.  512 threads leave 128 registers per thread; the softmax
// therefore holds one 64-column half of a row's scores at a time.
constexpr int kThreads = 512;
constexpr int kMmaWarp = 12;
constexpr int kSendWarp = 15;  // CTA 0 only; a gather warp in CTA 1
constexpr int kGatherWarpsK = 10, kGatherWarpsV = 11;
constexpr int kTmemCols = 512;
constexpr uint32_t kTmemS = 256;                    // CTA 0: query blocks 0-7 in [0, 256), S buffers at 256, 384
constexpr uint32_t kIdescQK = idesc_bf16(128, kChunk);
constexpr uint32_t kIdescPV = idesc_bf16(128, 128, /*b_mn_major=*/true);
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kKRingOff % 1024 == 0 && kPOff % 1024 == 0 && kOffBar % 8 == 0 && kPMsgBytes % 16 == 0, "alignment");
static_assert(8 * kStageBlock <= kPOff, "the staged output fits where the value ring was");
static_assert(kVSlots == 4, "one value slot per quarter of the 512 latent columns");

__device__ __forceinline__ int32_t selected_pos(const int32_t* __restrict__ idx_row, bool dense, int j, int L) {
  return dense ? (j < L ? j : -1) : idx_row[j];
}

__device__ __forceinline__ bool index_ok(int32_t idx, int E) { return idx >= 0 && idx < E; }

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    sparse_mla_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_out,
                           const MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  PairMisc* misc = reinterpret_cast<PairMisc*>(smem + kOffMisc);
  volatile int* abort = &misc->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: QK side, 1: PV side
  const uint32_t peer = rank ^ 1u;
  // the partner's abort flag: a CTA that gives up makes its partner give up too
  const uint32_t peer_abort = mapa_shared(sbase + kOffMisc + (uint32_t)offsetof(PairMisc, abort), peer);
  auto give_up = [&]() {
    *abort = 1;
    st_cluster_u32(peer_abort, 1u);
  };

  if (!p.early_inputs) grid_dependency_wait();  // q and the offsets may come from the previous kernel
  const int unit = blockIdx.x >> 1;
  const int sp = unit % p.n_splits;
  // rows in reverse launch order: a causal prefill's late rows keep the most keys
  const int r = (int)(gridDim.x / (2 * p.n_splits)) - 1 - unit / p.n_splits;
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

  // ---- prologue: barriers, TMEM, the query (CTA 0)
  if (threadIdx.x == 0) {
    misc->last_valid = -1;
    misc->abort = 0;
  }
  if (threadIdx.x < kMaxChunks * (kChunk / 32)) (&misc->vmask[0][0])[threadIdx.x] = 0u;
  if (warp == kMmaWarp) {
    if (lane == 0) {
      // TMA bytes of block 8, 128 TMEM writers (+ the test hook's missing arrival)
      mbar_init(bar(kQFull), 1 + 128 + p.debug_stall);
      for (int s = 0; s < kKSlots; ++s) {
        mbar_init(bar(kKFull + s), 32 * kGatherWarpsK);
        mbar_init(bar(kKEmpty + s), 1);
      }
      for (int s = 0; s < kVSlots; ++s) {
        mbar_init(bar(kVFull + s), 32 * kGatherWarpsV);
        mbar_init(bar(kVEmpty + s), 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(bar(kSFull + i), 1);
        mbar_init(bar(kSEmpty + i), 128);
        mbar_init(bar(kPvDone + i), 1);
        mbar_init(bar(kPFull + i), 1);  // CTA 0's expect-tx arrival; the bytes come by st.async
        mbar_init(bar(kReady + i), 128);
      }
      mbar_init(bar(kMLFull), 128);
      mbar_init(bar(kDrain), 1);
      for (int i = 0; i < 2; ++i) {
        mbar_init(bar(kStageFree + i), 1);
        mbar_init(bar(kStaged + i), 128);
      }
      fence_mbar_init();
      if (rank == 0 && geo_ok) {
        mbar_arrive_expect_tx(bar(kQFull), kBlockBytes);
        tma_load_2d(sbase + kQ8Off, &tm_q, 8 * 64, r * p.H, bar(kQFull));
      }
    }
    __syncwarp();
    tmem_alloc(sbase + kOffMisc + (uint32_t)offsetof(PairMisc, tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc->tmem_base);
  const int h = threadIdx.x;  // warps 0-3: head = TMEM lane
  if (rank == 0 && warp < 4 && geo_ok) {
    // Query blocks 0-7 of head h into TMEM lane h, two bf16 per column: the
    // A operand of 32 of the 36 QK MMAs of every chunk.  Rows past H are zero.
    const uint32_t lane_q = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const bool live = h < p.H;
    const uint4* qrow = reinterpret_cast<const uint4*>(p.q + ((int64_t)r * p.H + (live ? h : 0)) * kDQK);
#pragma unroll 2
    for (int g = 0; g < kKB - 1; ++g) {  // one block (8 x 16 bytes) per round
      uint32_t w[32];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint4 v = live ? __ldg(qrow + 8 * g + u) : make_uint4(0u, 0u, 0u, 0u);
        w[4 * u] = v.x;
        w[4 * u + 1] = v.y;
        w[4 * u + 2] = v.z;
        w[4 * u + 3] = v.w;
      }
      tmem_st32(lane_q + 32 * g, w);
    }
    tc_wait_st();
    tc_fence_before();
    mbar_arrive(bar(kQFull));
  }
  grid_dependency_wait();  // the indices come from the previous kernel
  allow_dependents_launch();

  // ---- which chunks of this split hold a selected row (both CTAs, the same
  // answer): each warp loads all its chunks' indices, then builds their
  // validity masks with ballots
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
#pragma unroll
      for (int hh = 0; hh < kChunk / 32; ++hh) {
        const bool valid = index_ok(ids[u][hh], E);
        if (!valid && ids[u][hh] != -1 && rank == 0) report(p.status, DSA_ERR_BAD_INDEX);
        const uint32_t m = __ballot_sync(0xffffffffu, valid);
        if (lane == 0) misc->vmask[c][hh] = m;
        if (m) lv = max(lv, (c_begin + c) * kChunk + 32 * hh + 31 - __clz((int)m));
      }
    }
    if (lane == 0 && lv >= 0) atomicMax(&misc->last_valid, lv);
  } else if (threadIdx.x == 0 && rank == 0) {
    report(p.status, DSA_ERR_BAD_OFFSETS);
  }
  __syncthreads();
  // every barrier of both CTAs is initialised before either touches the other
  cluster_sync_all();
  const int n_my = misc->last_valid < 0 ? 0 : misc->last_valid / kChunk - c_begin + 1;
  const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);

  if (n_my == 0) {
    // nothing selected in this split: empty partial, or zero output (CTA 1)
    if (rank == 1 && warp < 4 && h < p.H) {
      const int64_t rh = (int64_t)r * p.H + h;
      if (p.n_splits == 1) {
        if (p.out_bf16) {
          __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out) + rh * kDV;
          for (int c = 0; c < kDV; ++c) o[c] = __float2bfloat16(0.f);
        } else {
          float* o = reinterpret_cast<float*>(p.out) + rh * kDV;
          for (int c = 0; c < kDV; ++c) o[c] = 0.f;
        }
        if (p.lse) p.lse[rh] = -INFINITY;
      } else {
        const int64_t slot = ((int64_t)r * p.n_splits + sp) * p.H + h;
        __nv_bfloat16* o = p.ws_o + slot * kDV;
        for (int c = 0; c < kDV; ++c) o[c] = __float2bfloat16(0.f);
        p.ws_ml[2 * slot] = -INFINITY;
        p.ws_ml[2 * slot + 1] = 0.f;
      }
    }
    if (rank == 0 && warp == kMmaWarp && lane == 0 && geo_ok) {  // the query tile must land before the CTA exits
      volatile int never = 0;
      mbar_wait(bar(kQFull), 0, &never, 10000000ull);
    }
  }
  // gather warps: 4-11 and 13-15 are gather warps 0-10
  const int gw = warp < kMmaWarp ? warp - 4 : warp - 5;
  if (n_my > 0 && rank == 0) {
    // ================================================================ QK side
    if (warp == kMmaWarp) {
      if (lane == 0) {
        // ---- MMA issuer: S(i) = Q . Kv(i)^T into buffer i & 1, once
        // softmax(i-2) has read that buffer; the three slots of chunk i in
        // order, each released for the next load as soon as its MMAs
        // complete.  Query blocks 0-7 come from TMEM, block 8 from shared
        // memory: two branch-free runs.
        bool ok = mbar_wait(bar(kQFull), 0, abort, p.wait_limit_ns);
        const uint64_t q8 = smem_desc(sbase + kQ8Off, 16, 1024, kSwizzle128B);
        const uint64_t kb0 = smem_desc(sbase + kKRingOff, 16, 1024, kSwizzle128B);
        for (int i = 0; ok && i < n_my; ++i) {
          const int sb = i & 1;
          if (i >= 2 && !(ok = mbar_wait(bar(kSEmpty + sb), ((i - 2) >> 1) & 1, abort, p.wait_limit_ns))) break;
          const uint32_t d = tmem + kTmemS + 128 * sb;
#pragma unroll 1
          for (int j = 0; j < kKSlotsPerChunk; ++j) {
            const int g = i * kKSlotsPerChunk + j, slot = g % kKSlots;
            if (!(ok = mbar_wait(bar(kKFull + slot), (g / kKSlots) & 1, abort, p.wait_limit_ns))) break;
            fence_proxy_async_smem();  // rows written by cp.async, read by the tensor core
            tc_fence_after();
            const uint64_t bs = kb0 + (uint64_t)((slot * kKSlotBytes) >> 4);
            const int n_tmem_blocks = j < kKSlotsPerChunk - 1 ? kKSlotBlocks : kKSlotBlocks - 1;
#pragma unroll 1
            for (int bb = 0; bb < n_tmem_blocks; ++bb) {
              const int kb = kKSlotBlocks * j + bb;
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                mma_f16_ts(d, tmem + kb * 32 + ks * 8, bs + (uint64_t)((bb * kBlockBytes) >> 4) + (uint64_t)ks * 2,
                           kIdescQK, (kb | ks) ? 1u : 0u);
            }
            if (j == kKSlotsPerChunk - 1) {
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                mma_f16_ss(d, q8 + (uint64_t)ks * 2,
                           bs + (uint64_t)(((kKSlotBlocks - 1) * kBlockBytes) >> 4) + (uint64_t)ks * 2, kIdescQK, 1u);
            }
            tc_commit(bar(kKEmpty + slot));
          }
          if (!ok) break;
          tc_commit(bar(kSFull + sb));
        }
        if (*abort) {
          give_up();
          // tensor-core work must finish before TMEM is released, and the
          // query tile must have landed before the CTA exits
          volatile int never = 0;
          tc_commit(bar(kDrain));
          mbar_wait(bar(kDrain), 0, &never, 10000000ull);
          mbar_wait(bar(kQFull), 0, &never, 10000000ull);
        }
      }
    } else if (warp == kSendWarp) {
      if (lane == 0) {
        // ---- message sender: once message i is staged and CTA 1's buffer
        // i & 1 is free (P.V(i-2) complete), the copy engine moves it into
        // CTA 1, completing on CTA 1's barrier
        const uint32_t rem_msg = mapa_shared(sbase + kPOff, 1);
        const uint32_t rem_pfull = mapa_shared(bar(kPFull), 1);
        int n_sent = 0;
        for (int i = 0; i < n_my; ++i) {
          const int sb = i & 1;
          if (!mbar_wait(bar(kStaged + sb), (i >> 1) & 1, abort, p.wait_limit_ns)) break;
          if (i >= 2 && !mbar_wait_cluster(bar(kPvDone + sb), ((i - 2) >> 1) & 1, abort, p.wait_limit_ns)) break;
          const uint32_t pfull = rem_pfull + 8u * (uint32_t)sb;
          mbar_arrive_expect_tx_cluster(pfull, kPMsgBytes);
          bulk_copy_s2c(rem_msg + (uint32_t)sb * kPMsgBytes, sbase + kStageOff + (uint32_t)sb * kPMsgBytes, kPMsgBytes,
                        pfull);
          ++n_sent;
        }
        if (*abort) {
          give_up();
          // a copy may still be reading the staging buffers: wait (bounded)
          // for CTA 1's acknowledgements of the last ones
          volatile int never = 0;
          for (int j = max(0, n_sent - 2); j < n_sent; ++j)
            mbar_wait_cluster(bar(kStageFree + (j & 1)), (j >> 1) & 1, &never, 10000000ull);
        }
      }
    } else if (warp >= 4) {
      // ---- row gather into the 48 KB slots: gather warp gw copies the row
      // groups gw, gw + 10, gw + 20, gw + 30 (four rows each) of the chunk,
      // one group (96 pieces of 16 bytes, rows contiguous) per three copy
      // instructions.  Lane 4t + r holds the position of row r of the warp's
      // group t.
      const __nv_bfloat16* kv = p.kv;
      auto row_id = [&](int i) -> int32_t {
        const int gi = gw + kGatherWarpsK * (lane >> 2);
        if (lane >= 16 || gi >= kChunk / 4) return -1;
        const int pos = (c_begin + i) * kChunk + 4 * gi + (lane & 3);
        return pos < p.k ? selected_pos(idx_row, dense, pos, L_row) : -1;
      };
      int32_t my_id = row_id(0), next_id = -1;
      for (int i = 0; i < n_my; ++i) {
        if (i + 1 < n_my) next_id = row_id(i + 1);
        bool ok = true;
#pragma unroll 1
        for (int j = 0; j < kKSlotsPerChunk; ++j) {
          const int g = i * kKSlotsPerChunk + j, slot = g % kKSlots;
          if (!(ok = __all_sync(0xffffffffu,
                                mbar_wait(bar(kKEmpty + slot), ((g / kKSlots) & 1) ^ 1, abort, p.wait_limit_ns))))
            break;
          const uint32_t dst0 = sbase + kKRingOff + slot * kKSlotBytes;
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int gi = gw + kGatherWarpsK * t;
            if (gi >= kChunk / 4) break;  // uniform over the warp
#pragma unroll
            for (int u = 0; u < 3; ++u) {
              const int pc = 32 * u + lane;          // piece 0..95 of the group's four rows
              const int rr = pc / 24;
              const int c24 = pc % 24, bb = c24 >> 3, cc = c24 & 7;
              const int32_t id = __shfl_sync(0xffffffffu, my_id, 4 * t + rr);
              const bool valid = index_ok(id, E);
              const int row = 4 * gi + rr;           // row of the chunk, 0..127
              const __nv_bfloat16* src =
                  valid ? kv + ((int64_t)base_row + id) * kDQK + (kKSlotBlocks * j + bb) * 64 + cc * 8 : kv;
              const uint32_t dst = dst0 + bb * kBlockBytes + (row >> 3) * 1024 + (row & 7) * 128 + ((cc ^ (row & 7)) << 4);
              cp_async_16(dst, src, valid ? 16u : 0u);
            }
          }
          cp_async_mbar_arrive(bar(kKFull + slot));
        }
        if (!ok) break;
        my_id = next_id;
      }
      cp_async_wait<0>();
      if (*abort) give_up();
    } else {
      // ---- softmax: thread h owns head h (TMEM lane h).  P(i) and the
      // rescale factors are staged in this CTA's shared memory as message i
      // (two staging buffers); the sender warp has the copy engine move it
      // into CTA 1, which acknowledges each landed message.
      const uint32_t rem_ml = mapa_shared(sbase + kMLOff, 1);
      const uint32_t rem_mlfull = mapa_shared(bar(kMLFull), 1);
      float m_run = -INFINITY, l_run = 0.f;
      bool ok = true;
      // masked positions score -inf; the others x = s * scale * log2(e)
      auto scaled = [&](uint32_t (&sv)[64], int i, int half) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint32_t vm = misc->vmask[i][2 * half + c];  // validity of 32 positions
          if (vm == ~0u) {
#pragma unroll
            for (int j = 32 * c; j < 32 * c + 32; j += 2) {
              const float2 x2 = __fmul2_rn(make_float2(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])),
                                           make_float2(p.scale_log2, p.scale_log2));
              sv[j] = __float_as_uint(x2.x);
              sv[j + 1] = __float_as_uint(x2.y);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              sv[32 * c + j] =
                  __float_as_uint(((vm >> j) & 1u) ? __uint_as_float(sv[32 * c + j]) * p.scale_log2 : -INFINITY);
          }
        }
      };
      const int prow_off = (h >> 3) * 2048 + (h & 7) * 16;
      // p = 2^(x - m_sub) of 64 scores, rounded to bf16 and
      // staged as P row h (K-major without swizzle: 8-row x 16-byte core
      // matrices, 128 bytes apart along K, 2048 apart along M); returns the
      // sum of the rounded values.
      // (Four partial sums: one serial chain of 32 additions would bound
      // the loop by its latency.)
      auto emit = [&](const uint32_t (&sv)[64], uint8_t* prow, int half, float m_sub) -> float {
        float2 l2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        const float2 nm2 = make_float2(-m_sub, -m_sub);
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 8 * c8 + 2 * e;
            const float2 d = __fadd2_rn(make_float2(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])), nm2);
            const __nv_bfloat162 pb = __floats2bfloat162_rn(ex2_approx(d.x), ex2_approx(d.y));
            l2[e] = __fadd2_rn(l2[e], __bfloat1622float2(pb));
            w4[e] = *reinterpret_cast<const uint32_t*>(&pb);
          }
          *reinterpret_cast<uint4*>(prow + (8 * half + c8) * 128) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        const float2 a = __fadd2_rn(l2[0], l2[1]), b = __fadd2_rn(l2[2], l2[3]);
        return (a.x + b.x) + (a.y + b.y);
      };
      // max of 64 values as a tree (a serial chain of 64 would bound the loop)
      auto max64 = [](const uint32_t (&sv)[64]) -> float {
        float m8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          m8[q] = __uint_as_float(sv[q]);
#pragma unroll
          for (int j = 8 + q; j < 64; j += 8) m8[q] = fmaxf(m8[q], __uint_as_float(sv[j]));
        }
        return fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      };
      for (int i = 0; i < n_my; ++i) {
        const int sb = i & 1;  // S buffer, staging buffer and CTA 1's message buffer
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kSFull + sb), (i >> 1) & 1, abort, p.wait_limit_ns));
        // staging buffer sb is free once the copy of message i-2 has landed
        if (ok && i >= 2)
          ok = __all_sync(0xffffffffu,
                          mbar_wait_cluster(bar(kStageFree + sb), ((i - 2) >> 1) & 1, abort, p.wait_limit_ns));
        if (!ok) break;
        uint8_t* const stage = smem + kStageOff + sb * kPMsgBytes;
        uint8_t* const prow = stage + prow_off;
        const uint32_t s_addr = lane_addr + kTmemS + 128 * sb;
        tc_fence_after();
        // One pass over S, 64 columns per TMEM load, with the running max
        // m_run: p = 2^(x - m_run) stays below 2^8 unless a score exceeds
        // m_run + 8.  A thread that meets such a score (always in the first
        // chunk, rarely later) takes the chunk's max and emits its row again
        // with the raised max; O and l are rescaled by alpha.
        const float m_sub0 = m_run == -INFINITY ? 0.f : m_run;
        float l_chunk = 0.f, mc = -INFINITY;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          uint32_t sv[64];
          tmem_ld64(s_addr + 64 * half, sv);
          tc_wait_ld();
          scaled(sv, i, half);
          mc = fmaxf(mc, max64(sv));
          l_chunk += emit(sv, prow, half, m_sub0);
        }
        float alpha = 1.f;
        const bool raise = mc > m_run + 8.f;
        // the TMEM loads are warp-wide: the whole warp emits again if any
        // lane raises its max (a lane that does not raise recomputes the
        // same values)
        if (__any_sync(0xffffffffu, raise)) {
          const float m_new = raise ? mc : m_run;
          alpha = (raise && m_run != -INFINITY) ? exp2f(m_run - m_new) : 1.f;
          const float m_sub = m_new == -INFINITY ? 0.f : m_new;
          l_chunk = 0.f;
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            uint32_t sv[64];
            tmem_ld64(s_addr + 64 * half, sv);
            tc_wait_ld();
            scaled(sv, i, half);
            l_chunk += emit(sv, prow, half, m_sub);
          }
          m_run = m_new;
        }
        tc_fence_before();
        mbar_arrive(bar(kSEmpty + sb));  // S read: QK(i+2) may overwrite the buffer
        reinterpret_cast<float*>(stage + kPBytes)[h] = alpha;
        l_run = l_run * alpha + l_chunk;
        fence_proxy_async_smem();  // the message is read by the copy engine
        mbar_arrive(bar(kStaged + sb));
      }
      if (ok) {
        // the row's (max, sum) for CTA 1's epilogue
        const uint32_t a = rem_ml + (uint32_t)(h * 8);
        st_cluster_u32(a, __float_as_uint(l_run > 0.f ? m_run : -INFINITY));
        st_cluster_u32(a + 4, __float_as_uint(l_run));
        mbar_arrive_cluster(rem_mlfull);
        // the last two P.V completions arrive here too (multicast commit):
        // they must have landed before this CTA exits
        for (int j = max(0, n_my - 2); j < n_my; ++j)
          mbar_wait_cluster(bar(kPvDone + (j & 1)), (j >> 1) & 1, abort, p.wait_limit_ns);
      }
      if (*abort) give_up();
    }
  } else if (n_my > 0) {
    // ================================================================ PV side
    if (warp == kMmaWarp) {
      if (lane == 0) {
        // ---- MMA issuer: O[:, 128q .. 128q+127] += P(i) . V(i)[:, quarter q]
        const uint64_t pa0 = smem_desc(sbase + kPOff, 128, 2048, kSwizzleNone);  // message buffer 0's P
        const uint64_t vb0 = smem_desc(sbase + kVRingOff, kBlockBytes, 1024, kSwizzle128B);
        bool ok = true;
        for (int i = 0; ok && i < n_my; ++i) {
          const int pb = i & 1;
          if (!(ok = mbar_wait(bar(kReady + pb), (i >> 1) & 1, abort, p.wait_limit_ns))) break;
          tc_fence_after();
          const uint64_t ad = pa0 + (uint64_t)((pb * kPMsgBytes) >> 4);
#pragma unroll 1
          for (int q = 0; q < kVSlots; ++q) {
            if (!(ok = mbar_wait(bar(kVFull + q), i & 1, abort, p.wait_limit_ns))) break;
            fence_proxy_async_smem();
            tc_fence_after();
            const uint64_t bd = vb0 + (uint64_t)((q * kVSlotBytes) >> 4);
#pragma unroll
            for (int s = 0; s < kChunk / 16; ++s)
              mma_f16_ss(tmem + 128 * q, ad + (uint64_t)((s * 256) >> 4), bd + (uint64_t)((s * 2048) >> 4), kIdescPV,
                         (i > 0 || s > 0) ? 1u : 0u);
            tc_commit(bar(kVEmpty + q));
          }
          if (!ok) break;
          tc_commit_mc(bar(kPvDone + pb), 0x3);  // here, and CTA 0's "P buffer free"
        }
        if (*abort) {
          give_up();
          volatile int never = 0;
          tc_commit(bar(kDrain));
          mbar_wait(bar(kDrain), 0, &never, 10000000ull);
        }
      }
    } else if (warp >= 4) {
      // ---- value gather: slot q holds latent columns 128q .. 128q+127 of the
      // chunk's 128 rows; gather warp gw copies the row pairs gw, gw + 11, ...
      // (256 contiguous bytes per row, one pair per copy instruction).  Lane
      // 2t + r holds the position of row r of the warp's pair t.
      const __nv_bfloat16* kv = p.kv;
      auto row_id = [&](int i) -> int32_t {
        const int gi = gw + kGatherWarpsV * (lane >> 1);
        if (lane >= 12 || gi >= kChunk / 2) return -1;
        const int pos = (c_begin + i) * kChunk + 2 * gi + (lane & 1);
        return pos < p.k ? selected_pos(idx_row, dense, pos, L_row) : -1;
      };
      int32_t my_id = row_id(0), next_id = -1;
      for (int i = 0; i < n_my; ++i) {
        if (i + 1 < n_my) next_id = row_id(i + 1);
        bool ok = true;
#pragma unroll 1
        for (int q = 0; q < kVSlots; ++q) {
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar(kVEmpty + q), (i & 1) ^ 1, abort, p.wait_limit_ns))))
            break;
          const uint32_t dst0 = sbase + kVRingOff + q * kVSlotBytes;
#pragma unroll
          for (int t = 0; t < 6; ++t) {
            const int gi = gw + kGatherWarpsV * t;
            if (gi >= kChunk / 2) break;  // uniform over the warp
            const int rr = lane >> 4;
            const int pc = lane & 15, bb = pc >> 3, cc = pc & 7;
            const int32_t id = __shfl_sync(0xffffffffu, my_id, 2 * t + rr);
            const bool valid = index_ok(id, E);
            const int row = 2 * gi + rr;
            const __nv_bfloat16* src = valid ? kv + ((int64_t)base_row + id) * kDQK + 128 * q + pc * 8 : kv;
            const uint32_t dst = dst0 + bb * kBlockBytes + (row >> 3) * 1024 + (row & 7) * 128 + ((cc ^ (row & 7)) << 4);
            cp_async_16(dst, src, valid ? 16u : 0u);
          }
          cp_async_mbar_arrive(bar(kVFull + q));
        }
        if (!ok) break;
        my_id = next_id;
      }
      cp_async_wait<0>();
      if (*abort) give_up();
    } else {
      // ---- rescale, then the epilogue: thread h owns O row h (TMEM lane h).
      // Each landed message is acknowledged to CTA 0 (its staging buffer is
      // free again).
      const uint32_t rem_stage_free = mapa_shared(bar(kStageFree), 0);
      bool ok = true;
      for (int i = 0; i < n_my; ++i) {
        const int pb = i & 1;
        ok = __all_sync(0xffffffffu, mbar_wait_cluster(bar(kPFull + pb), (i >> 1) & 1, abort, p.wait_limit_ns));
        if (!ok) break;
        const float alpha = reinterpret_cast<const float*>(smem + kPOff + pb * kPMsgBytes + kPBytes)[h];
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
          // O is rescaled in TMEM once every earlier P.V has completed (the
          // last one, P.V(i-1), completes after all the others)
          if (i > 0) {
            ok = __all_sync(0xffffffffu,
                            mbar_wait(bar(kPvDone + ((i - 1) & 1)), ((i - 1) >> 1) & 1, abort, p.wait_limit_ns));
            if (!ok) break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int cb = 0; cb < kDV / 32; ++cb) {
            uint32_t ov[32];
            tmem_ld32(lane_addr + 32 * cb, ov);
            tc_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
            tmem_st32(lane_addr + 32 * cb, ov);
          }
          tc_wait_st();
        }
        fence_proxy_async_smem();  // P, stored by CTA 0, is read by this CTA's tensor core
        tc_fence_before();
        mbar_arrive(bar(kReady + pb));
        if (h == 0) mbar_arrive_cluster(rem_stage_free + 8u * (uint32_t)pb);  // CTA 0 may restage buffer pb
      }
      if (ok)
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kPvDone + ((n_my - 1) & 1)), ((n_my - 1) >> 1) & 1, abort,
                                              p.wait_limit_ns));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait_cluster(bar(kMLFull), 0, abort, p.wait_limit_ns));
      float m_row = -INFINITY, l_row = 0.f;
      if (ok) {
        const float* ml = reinterpret_cast<const float*>(smem + kMLOff);
        m_row = ml[2 * h];
        l_row = ml[2 * h + 1];
      }
      // Every MMA has completed, so the value ring is free: the 128 x 512
      // result is staged there as 128-byte-swizzled boxes of 32 fp32 (or 64
      // bf16) columns, one thread per head row, and written by TMA tensor
      // stores (the output's tensor map has one box per block), each 64
      // columns as soon as they are staged.  fp32 output goes in two halves
      // of 256 columns.
      const bool final_out = p.n_splits == 1;
      const bool as_bf16 = !final_out || p.out_bf16;  // partials are bf16 too
      const float mul = final_out ? (l_row > 0.f ? 1.f / l_row : 0.f) : 1.f;
      const int sw = h & 7;
      const int y = final_out ? r * p.H : (r * p.n_splits + sp) * p.H;
      const int n_pass = as_bf16 ? 1 : 2;
      for (int pass = 0; pass < n_pass; ++pass) {
        if (ok) tc_fence_after();
        const int cb_lo = as_bf16 ? 0 : 8 * pass, cb_hi = as_bf16 ? 16 : 8 * pass + 8;
#pragma unroll 1
        for (int cb2 = cb_lo; cb2 < cb_hi; cb2 += 2) {
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
                uint8_t* rowp = smem + (cb >> 1) * kStageBlock + h * 128;
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
                uint8_t* rowp = smem + (cb - cb_lo) * kStageBlock + h * 128;
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
              tma_store_2d(&tm_out, sbase + (cb2 >> 1) * kStageBlock, 32 * cb2, y);
            } else {
              tma_store_2d(&tm_out, sbase + (cb2 - cb_lo) * kStageBlock, 32 * cb2, y);
              tma_store_2d(&tm_out, sbase + (cb2 + 1 - cb_lo) * kStageBlock, 32 * (cb2 + 1), y);
            }
            bulk_commit();
          }
        }
        if (threadIdx.x == 0 && !*abort) bulk_wait_read();  // the staged boxes stay valid until read
        named_barrier_sync(1, 128);
      }
      if (ok && h < p.H) {
        const int64_t rh = (int64_t)r * p.H + h;
        if (final_out) {
          if (p.lse) p.lse[rh] = l_row > 0.f ? (m_row + __log2f(l_row)) * 0.69314718055994531f : -INFINITY;
        } else {
          const int64_t slot = ((int64_t)r * p.n_splits + sp) * p.H + h;
          p.ws_ml[2 * slot] = l_row > 0.f ? m_row : -INFINITY;
          p.ws_ml[2 * slot + 1] = l_row;
        }
      }
      if (*abort) give_up();
    }
  }

  tc_fence_before();
  __syncthreads();
  // neither CTA leaves while the other may still write into its shared memory
  cluster_sync_all();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort) report(p.status, DSA_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_sparse_mla_pair(const CUtensorMap& tq, const CUtensorMap& tout, const MlaParams& p,
                                   unsigned n_units, cudaStream_t stream) {
  static PerDeviceOnce attr;
  const cudaError_t e = attr.run(
      [] { return cudaFuncSetAttribute(sparse_mla_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes); });
  if (e != cudaSuccess) return e;
  return launch_pdl(sparse_mla_pair_kernel, dim3(2 * n_units), dim3(kThreads), kSmemBytes, stream, tq, tout, p);
}

}  // namespace dsa
