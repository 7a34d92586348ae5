// noalloc.cu -- dsa_sparse_mla_noalloc: the sparse-MLA stage for callers that
// cannot hand the library a workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// attention step: a plugin inside another runtime that owns every byte of
// device memory and exposes no allocator, a serving loop whose memory budget
// is fixed at start-up and forbids cudaMalloc afterwards, or code whose
// allocator cannot be called from where the step is issued.  For them this
// entry point keeps the split partials of the sparse-MLA stage in a fixed
// scratch array that is part of the library image itself.
//
// The scratch is a file-scope device array of kScratchBytes (32 MiB).  Every
// GPU that loads the library holds it until the process exits.  Its device
// address is looked up once per device with cudaGetSymbolAddress (the host
// side name of the array is only a stand-in, not a device address).
#include <cstdint>
#include <mutex>

#include "dsa_internal.h"

namespace {

constexpr size_t kScratchBytes = DSA_NOALLOC_SCRATCH_BYTES;
static_assert(kScratchBytes == (32ull << 20), "the header states 32 MiB");

static __device__ __align__(256) unsigned char g_mla_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch on the current device (looked up on first use).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mla_scratch) != cudaSuccess || !p) return DSA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return DSA_OK;
}

}  // namespace

extern "C" {

int dsa_sparse_mla_noalloc(const void* q, const void* kv, const int32_t* offsets, const int32_t* indices,
                           int B, int T, int H, int k, float scale, int64_t kv_rows, void* out, int out_dtype,
                           float* lse, int32_t* dev_status, void* stream) {
  if (B <= 0 || T <= 0 || H < 1 || H > DSA_MAX_HEADS || k < 1 || k > DSA_MAX_TOPK)
    return dsa_sparse_mla(q, kv, offsets, indices, B, T, H, k, scale, kv_rows, out, out_dtype, lse, nullptr,
                          0, dev_status, stream);  // same argument errors as the allocating entry point
  const size_t need = dsa_sparse_mla_workspace_size(B, T, H, k);
  if (need > kScratchBytes) return DSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (need > 0) {
    const int rc = scratch_address(&scratch);
    if (rc != DSA_OK) return rc;
  }
  return dsa_sparse_mla(q, kv, offsets, indices, B, T, H, k, scale, kv_rows, out, out_dtype, lse, scratch,
                        need > 0 ? kScratchBytes : 0, dev_status, stream);
}

}  // extern "C"
