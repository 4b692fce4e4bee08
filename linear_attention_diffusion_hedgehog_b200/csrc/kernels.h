// Internal kernel-argument structs and launcher declarations (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace bha {

struct HybridArgs {
  const int32_t* cu_blk;
  const int32_t* state_slot;
  const void* Q;
  const void* K;
  const void* V;
  const float* S;
  const float* Z;
  const void* W;
  const float* alpha;
  void* O;
  int32_t* dev_err;
  int R, Hq, Hkv, d, F, Bmax, T, num_slots;
};

struct CommitArgs {
  const int32_t* cu_blk;
  const int32_t* state_slot;
  const void* K;
  const void* V;
  const void* W;
  float* S;
  float* Z;
  int32_t* dev_err;
  int R, Hkv, d, F, Bmax, T, num_slots;
};

struct FullPrefixArgs {
  const int32_t* cu_blk;
  const int32_t* kv_len;
  const void* Q;
  const void* Kc;
  const void* Vc;
  void* O;
  void* workspace;
  int32_t* dev_err;
  int64_t kv_capacity;
  int R, Hq, Hkv, d, Bmax, T;
};

// Parameters of the tensor-core decode-step kernel (hybrid_tc.cu); the tensor maps describe
// Q, K, V, W and S for the Tensor Memory Accelerator.
struct TcHybridParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_w, tm_s;
  const int32_t* cu_blk;
  const int32_t* state_slot;
  const float* Z;
  const float* alpha;
  __nv_bfloat16* O;
  int32_t* dev_err;
  int R, Hq, Hkv, G, T, Bmax, num_slots;  // G = Hq / Hkv query heads per KV head
  int o32;               // O is 32-byte aligned: rows are written in whole 32-byte sectors
  long long wait_limit;  // SM cycles a bounded wait may spin before giving up
};

// Parameters of the decode step fused with the block commit (hybrid_commit_tc.cu): the decode
// step's, plus K in 8-row boxes for the commit, and S and Z for its atomic adds.
struct TcHybridCommitParams {
  TcHybridParams h;
  float* Sw;
  float* Zw;
};

// Parameters of the tensor-core block-commit kernel (commit_tc.cu).
struct TcCommitParams {
  CUtensorMap tm_k, tm_v, tm_w, tm_s;  // tm_s: S as [rows of F][d] fp32, the reduce-add target
  const int32_t* cu_blk;
  const int32_t* state_slot;
  float* S;
  float* Z;
  int32_t* dev_err;
  int R, Hkv, T, Bmax, num_slots;
  long long wait_limit;
};

// Parameters of the tensor-core softmax-teacher kernel (full_prefix_tc.cu).
struct TcFullParams {
  CUtensorMap tm_q, tm_k, tm_v;
  const int32_t* cu_blk;
  const int32_t* kv_len;
  __nv_bfloat16* O;
  float* opart;  // [nsplit][T * Hq][d] unnormalised partial outputs
  float* mpart;  // [nsplit][T * Hq] running max (log2 units)
  float* lpart;  // [nsplit][T * Hq] softmax sums
  int32_t* dev_err;
  int R, Hq, Hkv, T, Bmax, cap, nsplit, tiles_per_split;
  int o32;  // O is 32-byte aligned: rows are written in whole 32-byte sectors
  long long wait_limit;
};

// Parameters of the tensor-core feature-map kernel (featuremap_tc.cu).
struct TcFeatParams {
  CUtensorMap tm_x, tm_w, tm_o;
  void* phi;         // the output, for direct row stores when it is 32-byte aligned
  int32_t* dev_err;  // BHA_ERR_TIMEOUT if a bounded wait gave up; may be null
  int T, H, Hw, G, out_bf16, o32;
  long long wait_limit;
};

// host helpers shared by the tensor-core launchers (tc_host.cu)
enum TmaSwizzle { kTma128B, kTma128BAtom32, kTmaNone };
bool make_tensor_map(CUtensorMap* m, bool f32, int rank, const void* base, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box, TmaSwizzle swizzle);
int device_sm_count();
// Grid of a persistent kernel over `units` work units striding by the grid: the fewest CTAs
// (at most nsm, one per SM) that finish in the least number of rounds, rounded up to a
// multiple of stride_mult when that costs no extra round (each CTA then keeps one weight
// matrix resident; otherwise it reloads the weights when the head changes).
int persistent_grid(int units, int stride_mult, int nsm);

// tensor-core kernels
bool hybrid_tc_supports(const HybridArgs& a, bool act_bf16);
cudaError_t launch_hybrid_tc(const HybridArgs& a, cudaStream_t st);
// the decode step of a, then S += phi(K)^T V and Z += sum phi(K) for its blocks (same shapes)
cudaError_t launch_hybrid_commit_tc(const HybridArgs& a, float* S, float* Z, cudaStream_t st);
bool commit_tc_supports(const CommitArgs& a, bool act_bf16);
cudaError_t launch_commit_tc(const CommitArgs& a, cudaStream_t st);
bool full_prefix_tc_supports(const FullPrefixArgs& a, bool act_bf16);
int full_prefix_splits(int R, int Hkv, int64_t cap);
size_t full_prefix_tc_workspace(const FullPrefixArgs& a);
cudaError_t launch_full_prefix_tc(const FullPrefixArgs& a, void* workspace, cudaStream_t st);
bool featuremap_tc_supports(int T, int x_heads, int Hw, int d, int F, bool act_bf16);
cudaError_t launch_featuremap_tc(const void* x, int T, int x_heads, int Hw, const void* W, void* phi,
                                 bool out_bf16, int32_t* dev_err, cudaStream_t st);

// generic CUDA-core kernels (simt.cu)
bool simt_supports(int d, int F, int Bmax);
cudaError_t launch_featuremap_simt(const void* x, int T_rows, int H, int Hw, int d, int F,
                                   const void* W, void* phi, bool act_bf16, bool out_bf16,
                                   cudaStream_t st);
cudaError_t launch_hybrid_simt(const HybridArgs& a, bool act_bf16, cudaStream_t st);
cudaError_t launch_commit_simt(const CommitArgs& a, bool act_bf16, cudaStream_t st);
cudaError_t launch_full_prefix_simt(const FullPrefixArgs& a, bool act_bf16, cudaStream_t st);

}  // namespace bha
