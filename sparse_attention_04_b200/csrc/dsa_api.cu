// dsa_api.cu -- the C ABI declared in include/dsa.h: argument validation,
// workspace sizing and the launch sequence of each call.  Validation happens
// on the host before anything is launched; nothing here allocates memory.
#include <cstdint>
#include <mutex>

#include "dsa_internal.h"

namespace dsa {

const DeviceInfo& device_info() {
  static DeviceInfo info[64];
  static bool have[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!have[dev]) {
    int sms = 148, smem = 232448;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    info[dev].sm_count = sms > 0 ? sms : 148;
    info[dev].max_smem_optin = smem;
    have[dev] = true;
  }
  return info[dev];
}

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shared argument checks of the three stages.
int check_rows(int B, int T) {
  if (B <= 0 || T <= 0) return DSA_ERR_INVALID_ARG;
  if ((int64_t)B * T > (int64_t)1 << 24) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

const char* dsa_status_string(int status) {
  switch (status) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG: bad pointer, size, alignment or enum";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED: valid but not implemented";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE: workspace missing or too small";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA: a CUDA call failed";
    case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT: a device pipeline wait ran out of time";
    case DSA_ERR_BAD_INDEX: return "DSA_ERR_BAD_INDEX: an index outside [0, end_pos)";
    case DSA_ERR_BAD_OFFSETS: return "DSA_ERR_BAD_OFFSETS: offsets exceed kv_rows, ld or T";
    default: return "DSA_ERR_UNKNOWN";
  }
}

int dsa_version(void) { return 100; }

int dsa_indexer_scores(const void* q_idx, const float* w, const void* k_idx, const float* k_scale,
                       int idx_dtype, const int32_t* offsets, int B, int T, int64_t kv_rows,
                       float* scores, int64_t ld_scores, int32_t* dev_status, void* stream) {
  if (int rc = check_rows(B, T)) return rc;
  if (!q_idx || !w || !k_idx || !offsets || !scores) return DSA_ERR_INVALID_ARG;
  if (idx_dtype != DSA_BF16 && idx_dtype != DSA_E4M3) return DSA_ERR_INVALID_ARG;
  if (idx_dtype == DSA_E4M3 && !k_scale) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) || !aligned16(scores))
    return DSA_ERR_INVALID_ARG;
  if (ld_scores < T || (ld_scores & 3) != 0) return DSA_ERR_INVALID_ARG;
  if (kv_rows < T || kv_rows > ((int64_t)1 << 31) - 1) return DSA_ERR_INVALID_ARG;
  IndexerArgs a{q_idx, w, k_idx, k_scale, idx_dtype, offsets, B, T, kv_rows, scores, ld_scores, dev_status};
  return launch_indexer(a, reinterpret_cast<cudaStream_t>(stream));
}

int dsa_topk(const float* scores, int64_t ld_scores, const int32_t* offsets, int B, int T, int k,
             int32_t* indices, int32_t* dev_status, void* stream) {
  if (int rc = check_rows(B, T)) return rc;
  if (!scores || !offsets || !indices) return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > DSA_MAX_TOPK) return DSA_ERR_INVALID_ARG;
  if (ld_scores < T || (ld_scores & 3) != 0 || ld_scores > ((int64_t)1 << 31) - 1)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(scores) || !aligned16(indices)) return DSA_ERR_INVALID_ARG;
  TopkArgs a{scores, ld_scores, offsets, B, T, k, indices, dev_status};
  return launch_topk(a, reinterpret_cast<cudaStream_t>(stream));
}

size_t dsa_sparse_mla_workspace_size(int B, int T, int H, int k) {
  if (check_rows(B, T) || H < 1 || H > DSA_MAX_HEADS || k < 1 || k > DSA_MAX_TOPK) return 0;
  return mla_workspace_bytes(B * T, H, k);
}

namespace {
int sparse_mla_call(const void* q, const void* kv, const int32_t* offsets, const int32_t* indices, int B, int T,
                    int H, int k, float scale, int64_t kv_rows, void* out, int out_dtype, float* lse,
                    void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream, bool early_inputs,
                    bool dense = false) {
  if (int rc = check_rows(B, T)) return rc;
  // dense: no index list, the decode step's short-context path (every prefix <= k)
  if (!q || !kv || !offsets || (!indices && !dense) || !out) return DSA_ERR_INVALID_ARG;
  if (dense) indices = nullptr;
  if (H < 1 || k < 1 || k > DSA_MAX_TOPK) return DSA_ERR_INVALID_ARG;
  if (H > DSA_MAX_HEADS) return DSA_ERR_UNSUPPORTED;
  if (out_dtype != DSA_BF16 && out_dtype != DSA_F32) return DSA_ERR_INVALID_ARG;
  if (!(scale == scale) || kv_rows < 1 || kv_rows > ((int64_t)1 << 31) - 1) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv) || !aligned16(out) || (indices && !aligned16(indices)))
    return DSA_ERR_INVALID_ARG;
  const size_t need = mla_workspace_bytes(B * T, H, k);
  if (need > 0 && (!workspace || ws_bytes < need || !aligned16(workspace))) return DSA_ERR_WORKSPACE;
  MlaArgs a{q, kv, offsets, indices, B, T, H, k, scale, kv_rows, out, out_dtype, lse, workspace, ws_bytes, dev_status,
            early_inputs};
  return launch_sparse_mla(a, reinterpret_cast<cudaStream_t>(stream));
}
}  // namespace

int dsa_sparse_mla(const void* q, const void* kv, const int32_t* offsets, const int32_t* indices,
                   int B, int T, int H, int k, float scale, int64_t kv_rows, void* out,
                   int out_dtype, float* lse, void* workspace, size_t ws_bytes,
                   int32_t* dev_status, void* stream) {
  return sparse_mla_call(q, kv, offsets, indices, B, T, H, k, scale, kv_rows, out, out_dtype, lse, workspace,
                         ws_bytes, dev_status, stream, false);
}

int dsa_decode_step_workspace_layout(int B, int max_end_pos, int k, int H, size_t* scores_off,
                                     int64_t* ld_scores, size_t* indices_off, size_t* mla_off) {
  if (B <= 0 || max_end_pos <= 0 || k < 1 || k > DSA_MAX_TOPK || H < 1 || H > DSA_MAX_HEADS)
    return DSA_ERR_INVALID_ARG;
  const int64_t ld = (int64_t)align_up((size_t)max_end_pos, 4);
  const size_t s_off = 0;
  const size_t i_off = align_up(s_off + (size_t)B * ld * sizeof(float), 256);
  const size_t m_off = align_up(i_off + (size_t)B * k * sizeof(int32_t), 256);
  if (scores_off) *scores_off = s_off;
  if (ld_scores) *ld_scores = ld;
  if (indices_off) *indices_off = i_off;
  if (mla_off) *mla_off = m_off;
  return DSA_OK;
}

int dsa_decode_step_launches(int B, int max_end_pos, int k, int H) {
  if (B <= 0 || max_end_pos <= 0 || k < 1 || k > DSA_MAX_TOPK || H < 1 || H > DSA_MAX_HEADS) return -1;
  int n = max_end_pos <= k ? 0 : 2;           // indexer + selection (skipped for short contexts)
  n += 1;                                      // attention
  n += mla_num_splits(B, k, H, max_end_pos <= k) > 1 ? 1 : 0;  // combine of the split partials
  return n;
}

size_t dsa_decode_step_workspace_size(int B, int max_end_pos, int k, int H) {
  size_t m_off = 0;
  if (dsa_decode_step_workspace_layout(B, max_end_pos, k, H, nullptr, nullptr, nullptr, &m_off))
    return 0;
  return m_off + mla_workspace_bytes(B, H, k);
}

int dsa_decode_step(const void* q_idx, const float* w, const void* k_idx, const float* k_scale,
                    int idx_dtype, const void* q, const void* kv, const int32_t* offsets, int B,
                    int max_end_pos, int64_t kv_rows, int k, int H, float scale, void* out,
                    int out_dtype, float* lse, void* workspace, size_t ws_bytes,
                    int32_t* dev_status, void* stream) {
  size_t s_off, i_off, m_off;
  int64_t ld;
  if (dsa_decode_step_workspace_layout(B, max_end_pos, k, H, &s_off, &ld, &i_off, &m_off))
    return DSA_ERR_INVALID_ARG;
  const size_t need = m_off + mla_workspace_bytes(B, H, k);
  if (!workspace || ws_bytes < need || !aligned16(workspace)) return DSA_ERR_WORKSPACE;
  if (!q || !kv || !out) return DSA_ERR_INVALID_ARG;
  if (out_dtype != DSA_BF16 && out_dtype != DSA_F32) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* scores = reinterpret_cast<float*>(ws + s_off);
  int32_t* indices = reinterpret_cast<int32_t*>(ws + i_off);
  if (max_end_pos <= k) {
    // Every sequence keeps all of its positions whatever the scores
    // (k_eff = end_pos): the indexer and the selection are skipped and the
    // attention runs over each whole prefix.  Scores and indices in the
    // workspace are left unwritten.
    if (!q_idx || !w || !k_idx || !offsets) return DSA_ERR_INVALID_ARG;
    if (idx_dtype != DSA_BF16 && idx_dtype != DSA_E4M3) return DSA_ERR_INVALID_ARG;
    // The attention is this call's first kernel here: nothing launched by
    // the library has waited for the work before it in the stream (a copy
    // kernel that may still be writing q, say), so it reads its inputs only
    // after its own dependency wait.
    return sparse_mla_call(q, kv, offsets, nullptr, B, 1, H, k, scale, kv_rows, out, out_dtype, lse, ws + m_off,
                           ws_bytes - m_off, dev_status, stream, /*early_inputs=*/false, /*dense=*/true);
  }
  int rc = dsa_indexer_scores(q_idx, w, k_idx, k_scale, idx_dtype, offsets, B, 1, kv_rows, scores,
                              ld, dev_status, stream);
  if (rc) return rc;
  rc = dsa_topk(scores, ld, offsets, B, 1, k, indices, dev_status, stream);
  if (rc) return rc;
  return sparse_mla_call(q, kv, offsets, indices, B, 1, H, k, scale, kv_rows, out, out_dtype, lse, ws + m_off,
                         ws_bytes - m_off, dev_status, stream, true);
}

}  // extern "C"
