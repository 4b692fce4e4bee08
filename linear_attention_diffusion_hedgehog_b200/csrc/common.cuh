// Shared device helpers for the libbha kernels: dtype loads/stores, warp reductions,
// request-range validation and the device error word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/bha.h"

namespace bha {

// ----------------------------------------------------------------- dtype helpers
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Two floats rounded to bf16 (nearest even) and packed low-first into 32 bits.
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// ----------------------------------------------------------------- warp reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ----------------------------------------------------------------- error word
// Records the first nonzero status; later ones are dropped.
__device__ __forceinline__ void set_error(int32_t* dev_err, int32_t code) {
  if (dev_err != nullptr) atomicCAS(dev_err, 0, code);
}

// Active-block row range of request r, validated against the call's dims.  Returns false
// (and records BHA_ERR_INVALID once per failing request) when cu_blk is malformed.
struct RowRange {
  int lo, n;
};
__device__ __forceinline__ bool request_rows(const int32_t* cu_blk, int r, int total_tokens,
                                             int max_block, int32_t* dev_err, bool report,
                                             RowRange* out) {
  const int lo = cu_blk[r], hi = cu_blk[r + 1];
  if (lo < 0 || hi < lo || hi > total_tokens || hi - lo > max_block) {
    if (report) set_error(dev_err, BHA_ERR_INVALID);
    return false;
  }
  out->lo = lo;
  out->n = hi - lo;
  return true;
}

// Slot of request r (identity when no map is given), validated.
__device__ __forceinline__ bool request_slot(const int32_t* state_slot, int r, int num_slots,
                                             int32_t* dev_err, bool report, int* slot) {
  const int s = state_slot ? state_slot[r] : r;
  if (s < 0 || s >= num_slots) {
    if (report) set_error(dev_err, BHA_ERR_INVALID);
    return false;
  }
  *slot = s;
  return true;
}

}  // namespace bha
