// Internal kernel-argument structs and launcher declarations (not part of the C ABI).
#pragma once

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

// generic CUDA-core kernels (simt.cu)
bool simt_supports(int d, int F, int Bmax);
cudaError_t launch_featuremap_simt(const void* x, int T_rows, int H, int Hw, int d, int F,
                                   const void* W, void* phi, bool act_bf16, bool out_bf16,
                                   cudaStream_t st);
cudaError_t launch_hybrid_simt(const HybridArgs& a, bool act_bf16, cudaStream_t st);
cudaError_t launch_commit_simt(const CommitArgs& a, bool act_bf16, cudaStream_t st);
cudaError_t launch_full_prefix_simt(const FullPrefixArgs& a, bool act_bf16, cudaStream_t st);

}  // namespace bha
