// dsa_internal.h -- constants and launcher declarations shared by the kernel
// translation units and the C-ABI layer (dsa_api.cu).  Not installed.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/dsa.h"

namespace dsa {

constexpr int kHI = 64;    // indexer heads
constexpr int kDI = 128;   // indexer head dim
constexpr int kDQK = 576;  // latent 512 || rope 64
constexpr int kDV = 512;   // value width (the latent)
constexpr int kMaxTopk = DSA_MAX_TOPK;
constexpr int kMaxHeads = DSA_MAX_HEADS;

// Every pipeline wait in the kernels gives up after this long and reports
// DSA_ERR_TIMEOUT.  Normal waits last microseconds.
constexpr uint64_t kWaitLimitNs = 200ull * 1000ull * 1000ull;

// Per-device facts the launchers need (cached after the first query).
struct DeviceInfo {
  int sm_count;
  int max_smem_optin;
};
const DeviceInfo& device_info();

// Runs `set` (kernel attribute calls) once per device, under a lock.  CUDA
// keeps a kernel's attributes (dynamic shared-memory limit, cluster size
// permission) per device context, so a process that calls the library on
// several GPUs must set them on each before its first launch there.
class PerDeviceOnce {
 public:
  template <class Fn>
  cudaError_t run(Fn&& set) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool cached = dev >= 0 && dev < kMaxDevices;
    std::lock_guard<std::mutex> lock(mu_);
    if (cached && done_[dev]) return cudaSuccess;
    e = set();
    if (e == cudaSuccess && cached) done_[dev] = true;
    return e;
  }

 private:
  static constexpr int kMaxDevices = 64;
  std::mutex mu_;
  bool done_[kMaxDevices] = {};
};

// ---- stage 1: indexer ------------------------------------------------------
struct IndexerArgs {
  const void* q_idx;
  const float* w;
  const void* k_idx;
  const float* k_scale;
  int idx_dtype;
  const int32_t* offsets;
  int B, T;
  int64_t kv_rows;
  float* scores;
  int64_t ld;
  int32_t* status;
};
int launch_indexer(const IndexerArgs& a, cudaStream_t stream);

// ---- stage 2: top-k ---------------------------------------------------------
struct TopkArgs {
  const float* scores;
  int64_t ld;
  const int32_t* offsets;
  int B, T, k;
  int32_t* indices;
  int32_t* status;
};
int launch_topk(const TopkArgs& a, cudaStream_t stream);

// ---- stage 3: sparse MLA ----------------------------------------------------
struct MlaArgs {
  const void* q;
  const void* kv;
  const int32_t* offsets;
  const int32_t* indices;
  int B, T, H, k;
  float scale;
  int64_t kv_rows;
  void* out;
  int out_dtype;
  float* lse;
  void* workspace;
  size_t ws_bytes;
  int32_t* status;
  // The step's inputs (q, offsets) were complete before the preceding kernel
  // in the stream started (true inside dsa_decode_step, whose first kernel
  // waited for them): the kernel may then read them before its dependency
  // wait.  Standalone calls wait first.
  bool early_inputs;
};
// Kernel parameters of the attention stage (both attention kernels).
struct MlaParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* kv;
  const int32_t* off;
  const int32_t* idx;
  int T, H, k;
  int n_splits, cps;  // splits per row, chunks per split
  float scale_log2;
  int64_t kv_rows;
  void* out;
  int out_bf16;
  float* lse;
  __nv_bfloat16* ws_o;  // [rows][splits][H][512] unnormalised partials (n_splits > 1)
  float* ws_ml;          // [rows][splits][H][2]   their (max, sum)
  int32_t* status;
  int early_inputs;  // q and offsets may be read before the dependency wait
  int dense;         // no index list: row r attends to its whole causal prefix
  // Test hook (dsa_debug_stall_attention): 1 makes the query barrier expect
  // one arrival more than will ever come, so its wait runs out and the
  // kernel takes its timeout path.  0 in normal use.
  int debug_stall;
  uint64_t wait_limit_ns;  // limit of every pipeline wait (kWaitLimitNs in normal use)
};
// Settings of the next attention launch: normal, or stalled by the test hook.
void take_attention_debug(MlaParams& p);

// The attention kernel for long index lists (sparse_mla_wide.cu): 64-key
// chunks, grid of 2 CTAs per (row, split) as the 32-key kernel.
constexpr int kMlaWideChunk = 64;
cudaError_t launch_sparse_mla_wide(const CUtensorMap& tq, const CUtensorMap& tout,
                                   const MlaParams& p, unsigned grid, cudaStream_t stream);

// The attention kernel for launches with many 128-key chunks per SM
// (sparse_mla_pair.cu): a cluster of two CTAs per (row, split), the QK side
// and the PV side; grid of 2 CTAs per unit.
constexpr int kMlaPairChunk = 128;
cudaError_t launch_sparse_mla_pair(const CUtensorMap& tq, const CUtensorMap& tout, const MlaParams& p,
                                   unsigned n_units, cudaStream_t stream);

int mla_num_splits(int n_rows, int k, int H, bool dense);  // dense: no index list (short context)
int mla_chunk(int n_rows, int k, bool dense);
size_t mla_workspace_bytes(int n_rows, int H, int k);
int launch_sparse_mla(const MlaArgs& a, cudaStream_t stream);

// Launches `kernel` on `stream` with programmatic stream serialisation, so
// that its prologue overlaps the tail of the previous kernel in the stream.
// The kernel must call grid_dependency_wait() before reading its inputs.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace dsa
