// Host helpers shared by the tensor-core launchers: tensor-map encoding (through the
// driver entry point the runtime exposes, so the library needs no link to libcuda) and the
// SM count of the current device.
#include <cuda.h>

#include "kernels.h"

namespace bha {
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

}  // namespace

bool make_tensor_map(CUtensorMap* m, bool f32, int rank, const void* base, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box, TmaSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) gs[i] = strides_bytes[i];
  }
  const CUtensorMapSwizzle sw = swizzle == kTma128B         ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle == kTma128BAtom32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B
                                                            : CU_TENSOR_MAP_SWIZZLE_NONE;
  const CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        rank, const_cast<void*>(base), gd, gs, bx, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

int persistent_grid(int units, int stride_mult, int nsm) {
  const int rounds = (units + nsm - 1) / nsm;
  int grid = (units + rounds - 1) / rounds;
  if (stride_mult > 1 && stride_mult <= nsm) {
    const int g2 = (grid + stride_mult - 1) / stride_mult * stride_mult;
    if (g2 <= nsm) grid = g2;
  }
  return grid < units ? grid : units;
}

}  // namespace bha
