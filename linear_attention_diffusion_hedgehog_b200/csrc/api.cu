// C-ABI entry points of libbha: argument validation on the host, then dispatch to the
// tensor-core kernels when the dims match their specialisation, else to the generic
// CUDA-core kernels.  Declarations and the full contract are in include/bha.h.
#include <cstdint>

#include "../../include/bha.h"
#include "kernels.h"

namespace {

constexpr int kVersion = 101;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_dims(const bha_dims* dm) {
  if (dm == nullptr) return BHA_ERR_INVALID;
  if (dm->num_requests < 0 || dm->num_q_heads < 1 || dm->num_kv_heads < 1 ||
      dm->total_tokens < 0 || dm->num_slots < 0 || dm->head_dim < 1 || dm->feature_dim < 2 ||
      dm->max_block < 1)
    return BHA_ERR_INVALID;
  if (dm->num_q_heads % dm->num_kv_heads != 0) return BHA_ERR_INVALID;
  if (dm->feature_dim % 2 != 0) return BHA_ERR_INVALID;
  if (dm->act_dtype != BHA_BF16 && dm->act_dtype != BHA_F32) return BHA_ERR_INVALID;
  if (!bha::simt_supports(dm->head_dim, dm->feature_dim, dm->max_block))
    return BHA_ERR_UNSUPPORTED;
  return BHA_OK;
}

// A tensor pointer must be non-null and 16-byte aligned (tensor-memory-access rule).
bool tensor_ok(const void* p) { return p != nullptr && aligned(p, 16); }
bool index_ok(const void* p) { return p != nullptr && aligned(p, 4); }

bha::FullPrefixArgs full_args(const bha_dims* dims, int64_t kv_capacity) {
  bha::FullPrefixArgs a{};
  a.kv_capacity = kv_capacity;
  a.R = dims->num_requests;
  a.Hq = dims->num_q_heads;
  a.Hkv = dims->num_kv_heads;
  a.d = dims->head_dim;
  a.Bmax = dims->max_block;
  a.T = dims->total_tokens;
  return a;
}

int launch_status(cudaError_t e) {
  if (e == cudaSuccess) return BHA_OK;
  return BHA_ERR_CUDA;
}

}  // namespace

extern "C" {

int bha_version(void) { return kVersion; }

const char* bha_status_string(int status) {
  switch (status) {
    case BHA_OK: return "BHA_OK";
    case BHA_ERR_INVALID: return "BHA_ERR_INVALID: invalid argument";
    case BHA_ERR_UNSUPPORTED: return "BHA_ERR_UNSUPPORTED: dims outside the implemented range";
    case BHA_ERR_CUDA: return "BHA_ERR_CUDA: CUDA runtime or launch failure";
    case BHA_ERR_TIMEOUT: return "BHA_ERR_TIMEOUT: a bounded device wait gave up";
    default: return "unknown bha_status";
  }
}

int bha_kernel_variant(const bha_dims* dims, int32_t which) {
  const int s = check_dims(dims);
  if (s != BHA_OK) return s;
  if (which < 0 || which > 4) return BHA_ERR_INVALID;
  const bool bf16 = dims->act_dtype == BHA_BF16;
  if (which == 0)
    return bha::featuremap_tc_supports(dims->total_tokens, dims->num_q_heads, dims->num_kv_heads,
                                       dims->head_dim, dims->feature_dim, bf16) ? 1 : 0;
  if (which == 1 || which == 4) {
    bha::HybridArgs a{};
    a.R = dims->num_requests;
    a.Hq = dims->num_q_heads;
    a.Hkv = dims->num_kv_heads;
    a.d = dims->head_dim;
    a.F = dims->feature_dim;
    a.Bmax = dims->max_block;
    a.T = dims->total_tokens;
    a.num_slots = dims->num_slots;
    return bha::hybrid_tc_supports(a, bf16) ? 1 : 0;
  }
  if (which == 2) {
    bha::CommitArgs c{};
    c.R = dims->num_requests;
    c.Hkv = dims->num_kv_heads;
    c.d = dims->head_dim;
    c.F = dims->feature_dim;
    c.Bmax = dims->max_block;
    c.T = dims->total_tokens;
    c.num_slots = dims->num_slots;
    return bha::commit_tc_supports(c, bf16) ? 1 : 0;
  }
  if (which == 3) return bha::full_prefix_tc_supports(full_args(dims, 0), bf16) ? 1 : 0;
  return 0;
}

int bha_featuremap(const bha_dims* dims, const void* x, int32_t x_heads, const void* W,
                   void* phi, int32_t out_dtype, void* stream) {
  return bha_featuremap_checked(dims, x, x_heads, W, phi, out_dtype, nullptr, stream);
}

int bha_featuremap_checked(const bha_dims* dims, const void* x, int32_t x_heads, const void* W,
                           void* phi, int32_t out_dtype, int32_t* dev_err, void* stream) {
  int s = check_dims(dims);
  if (s != BHA_OK) return s;
  if (x_heads < 1) return BHA_ERR_INVALID;
  if (out_dtype != BHA_BF16 && out_dtype != BHA_F32) return BHA_ERR_INVALID;
  if (dims->total_tokens == 0) return BHA_OK;
  if (!tensor_ok(x) || !tensor_ok(W) || !tensor_ok(phi)) return BHA_ERR_INVALID;
  if (x == phi || W == phi) return BHA_ERR_INVALID;
  if (dev_err != nullptr && !index_ok(dev_err)) return BHA_ERR_INVALID;
  if (bha::featuremap_tc_supports(dims->total_tokens, x_heads, dims->num_kv_heads, dims->head_dim,
                                  dims->feature_dim, dims->act_dtype == BHA_BF16))
    return launch_status(bha::launch_featuremap_tc(x, dims->total_tokens, x_heads, dims->num_kv_heads,
                                                   W, phi, out_dtype == BHA_BF16, dev_err,
                                                   static_cast<cudaStream_t>(stream)));
  return launch_status(bha::launch_featuremap_simt(
      x, dims->total_tokens, x_heads, dims->num_kv_heads, dims->head_dim, dims->feature_dim, W,
      phi, dims->act_dtype == BHA_BF16, out_dtype == BHA_BF16,
      static_cast<cudaStream_t>(stream)));
}

int bha_hybrid_attn(const bha_dims* dims, const int32_t* cu_blk, const int32_t* state_slot,
                    const void* Q, const void* K, const void* V, const float* S,
                    const float* Z, const void* W, const float* alpha, void* O,
                    int32_t* dev_err, void* stream) {
  int s = check_dims(dims);
  if (s != BHA_OK) return s;
  if (dims->num_requests == 0 || dims->total_tokens == 0) return BHA_OK;
  if (!index_ok(cu_blk)) return BHA_ERR_INVALID;
  if (state_slot != nullptr && !aligned(state_slot, 4)) return BHA_ERR_INVALID;
  if (state_slot == nullptr && dims->num_slots < dims->num_requests) return BHA_ERR_INVALID;
  if (!tensor_ok(Q) || !tensor_ok(K) || !tensor_ok(V) || !tensor_ok(S) || !tensor_ok(Z) ||
      !tensor_ok(W) || !tensor_ok(O))
    return BHA_ERR_INVALID;
  if (alpha != nullptr && !aligned(alpha, 4)) return BHA_ERR_INVALID;
  if (dev_err != nullptr && !aligned(dev_err, 4)) return BHA_ERR_INVALID;
  if (O == Q || O == K || O == V || O == W || O == (const void*)S || O == (const void*)Z)
    return BHA_ERR_INVALID;
  bha::HybridArgs a{cu_blk, state_slot, Q, K, V, S, Z, W, alpha, O, dev_err,
                    dims->num_requests, dims->num_q_heads, dims->num_kv_heads, dims->head_dim,
                    dims->feature_dim, dims->max_block, dims->total_tokens, dims->num_slots};
  const bool bf16 = dims->act_dtype == BHA_BF16;
  if (bha::hybrid_tc_supports(a, bf16))
    return launch_status(bha::launch_hybrid_tc(a, static_cast<cudaStream_t>(stream)));
  return launch_status(bha::launch_hybrid_simt(a, bf16, static_cast<cudaStream_t>(stream)));
}

int bha_hybrid_attn_commit(const bha_dims* dims, const int32_t* cu_blk, const int32_t* state_slot,
                           const void* Q, const void* K, const void* V, float* S, float* Z,
                           const void* W, const float* alpha, void* O, int32_t* dev_err,
                           void* stream) {
  int s = check_dims(dims);
  if (s != BHA_OK) return s;
  if (dims->num_requests == 0 || dims->total_tokens == 0) return BHA_OK;
  if (!index_ok(cu_blk)) return BHA_ERR_INVALID;
  if (state_slot != nullptr && !aligned(state_slot, 4)) return BHA_ERR_INVALID;
  if (state_slot == nullptr && dims->num_slots < dims->num_requests) return BHA_ERR_INVALID;
  if (!tensor_ok(Q) || !tensor_ok(K) || !tensor_ok(V) || !tensor_ok(S) || !tensor_ok(Z) ||
      !tensor_ok(W) || !tensor_ok(O))
    return BHA_ERR_INVALID;
  if (alpha != nullptr && !aligned(alpha, 4)) return BHA_ERR_INVALID;
  if (dev_err != nullptr && !aligned(dev_err, 4)) return BHA_ERR_INVALID;
  const void* outs[3] = {O, S, Z};
  const void* ins[6] = {Q, K, V, W, alpha, cu_blk};
  for (const void* o : outs)
    for (const void* i : ins)
      if (o == i) return BHA_ERR_INVALID;
  if (O == (void*)S || O == (void*)Z || (void*)S == (void*)Z) return BHA_ERR_INVALID;
  bha::HybridArgs a{cu_blk, state_slot, Q, K, V, S, Z, W, alpha, O, dev_err,
                    dims->num_requests, dims->num_q_heads, dims->num_kv_heads, dims->head_dim,
                    dims->feature_dim, dims->max_block, dims->total_tokens, dims->num_slots};
  const bool bf16 = dims->act_dtype == BHA_BF16;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (bha::hybrid_tc_supports(a, bf16)) return launch_status(bha::launch_hybrid_commit_tc(a, S, Z, st));
  // other dims: the decode step, then the commit, as two launches on the same stream
  const int r = launch_status(bha::launch_hybrid_simt(a, bf16, st));
  if (r != BHA_OK) return r;
  bha::CommitArgs c{cu_blk, state_slot, K, V, W, S, Z, dev_err, dims->num_requests,
                    dims->num_kv_heads, dims->head_dim, dims->feature_dim, dims->max_block,
                    dims->total_tokens, dims->num_slots};
  return launch_status(bha::launch_commit_simt(c, bf16, st));
}

int bha_commit_block(const bha_dims* dims, const int32_t* cu_blk, const int32_t* state_slot,
                     const void* K, const void* V, const void* W, float* S, float* Z,
                     int32_t* dev_err, void* stream) {
  int s = check_dims(dims);
  if (s != BHA_OK) return s;
  if (dims->num_requests == 0 || dims->total_tokens == 0) return BHA_OK;
  if (!index_ok(cu_blk)) return BHA_ERR_INVALID;
  if (state_slot != nullptr && !aligned(state_slot, 4)) return BHA_ERR_INVALID;
  if (state_slot == nullptr && dims->num_slots < dims->num_requests) return BHA_ERR_INVALID;
  if (!tensor_ok(K) || !tensor_ok(V) || !tensor_ok(W) || !tensor_ok(S) || !tensor_ok(Z))
    return BHA_ERR_INVALID;
  if (dev_err != nullptr && !aligned(dev_err, 4)) return BHA_ERR_INVALID;
  if ((const void*)S == K || (const void*)S == V || (const void*)Z == K || (const void*)Z == V ||
      (void*)S == (void*)Z)
    return BHA_ERR_INVALID;
  bha::CommitArgs a{cu_blk, state_slot, K, V, W, S, Z, dev_err, dims->num_requests,
                    dims->num_kv_heads, dims->head_dim, dims->feature_dim, dims->max_block,
                    dims->total_tokens, dims->num_slots};
  const bool bf16 = dims->act_dtype == BHA_BF16;
  if (bha::commit_tc_supports(a, bf16))
    return launch_status(bha::launch_commit_tc(a, static_cast<cudaStream_t>(stream)));
  return launch_status(bha::launch_commit_simt(a, bf16, static_cast<cudaStream_t>(stream)));
}


size_t bha_full_prefix_workspace_bytes(const bha_dims* dims, int64_t kv_capacity) {
  if (check_dims(dims) != BHA_OK || kv_capacity < 0 || kv_capacity > INT32_MAX) return 0;
  const bha::FullPrefixArgs a = full_args(dims, kv_capacity);
  if (!bha::full_prefix_tc_supports(a, dims->act_dtype == BHA_BF16)) return 0;
  return bha::full_prefix_tc_workspace(a);
}

int bha_full_prefix_attn(const bha_dims* dims, const int32_t* cu_blk, const int32_t* kv_len,
                         const void* Q, const void* Kc, const void* Vc, int64_t kv_capacity,
                         void* O, void* workspace, size_t workspace_bytes, int32_t* dev_err,
                         void* stream) {
  int s = check_dims(dims);
  if (s != BHA_OK) return s;
  if (kv_capacity < 0 || kv_capacity > INT32_MAX) return BHA_ERR_INVALID;
  if (dims->num_requests == 0 || dims->total_tokens == 0) return BHA_OK;
  if (!index_ok(cu_blk) || !index_ok(kv_len)) return BHA_ERR_INVALID;
  if (!tensor_ok(Q) || !tensor_ok(O)) return BHA_ERR_INVALID;
  if (kv_capacity > 0 && (!tensor_ok(Kc) || !tensor_ok(Vc))) return BHA_ERR_INVALID;
  if (dev_err != nullptr && !aligned(dev_err, 4)) return BHA_ERR_INVALID;
  const size_t need = bha_full_prefix_workspace_bytes(dims, kv_capacity);
  if (workspace_bytes < need || (need > 0 && !tensor_ok(workspace))) return BHA_ERR_INVALID;
  if (O == Q || O == Kc || O == Vc) return BHA_ERR_INVALID;
  bha::FullPrefixArgs a{cu_blk, kv_len, Q, Kc, Vc, O, workspace, dev_err, kv_capacity,
                        dims->num_requests, dims->num_q_heads, dims->num_kv_heads,
                        dims->head_dim, dims->max_block, dims->total_tokens};
  const bool bf16 = dims->act_dtype == BHA_BF16;
  if (bha::full_prefix_tc_supports(a, bf16))
    return launch_status(bha::launch_full_prefix_tc(a, workspace, static_cast<cudaStream_t>(stream)));
  return launch_status(bha::launch_full_prefix_simt(a, bf16, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
