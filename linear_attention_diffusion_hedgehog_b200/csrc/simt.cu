// Generic CUDA-core kernels: the feature map, the block-hybrid decode step, the block
// commit and the softmax teacher for any supported dims (d <= 256, F <= 512, b <= 128) and
// both activation dtypes, with fp32 arithmetic throughout.  They are the path for dims the
// tensor-core kernels do not cover and for fp32 activations (where tf32 tensor-core
// rounding would not meet a 1e-5 relative tolerance).
//
// Source: "Retrofitting Linear Attention into Diffusion Language Models", §3.1 (feature
// map, within-block softmax, states, commit, cross-block read, gated merge) and §2.2
// (softmax attention, for the teacher).
#include "common.cuh"
#include "kernels.h"

namespace bha {

namespace {

constexpr int kMaxD = 256;          // head_dim limit of the generic kernels
constexpr int kMaxFh = 256;         // F/2 limit
constexpr int kMaxB = 128;          // block-length limit
constexpr int kCols = kMaxFh / 32;  // per-lane columns of u = xW
constexpr int kDCols = kMaxD / 32;  // per-lane columns of a d-vector

// phi(x) = [softmax(xW), softmax(-xW)] for one row, computed by one warp.
// xs: the row in shared memory (d floats).  Wg: [d][Fh] in global memory.  Writes the F
// entries to out (shared memory).  Lane l owns columns f = l + 32c of u = xW.
template <typename T>
__device__ void warp_phi(const float* xs, const T* __restrict__ Wg, int d, int Fh, float* out) {
  const int lane = threadIdx.x & 31;
  float u[kCols];
#pragma unroll
  for (int c = 0; c < kCols; ++c) u[c] = 0.f;
  for (int k = 0; k < d; ++k) {
    const float xk = xs[k];
    const T* wrow = Wg + (size_t)k * Fh;
#pragma unroll
    for (int c = 0; c < kCols; ++c) {
      const int f = lane + 32 * c;
      if (f < Fh) u[c] = fmaf(xk, to_f32(wrow[f]), u[c]);
    }
  }
  float mx = -INFINITY, mn = INFINITY;
#pragma unroll
  for (int c = 0; c < kCols; ++c) {
    if (lane + 32 * c < Fh) {
      mx = fmaxf(mx, u[c]);
      mn = fminf(mn, u[c]);
    }
  }
  mx = warp_max(mx);
  mn = warp_min(mn);
  float ep[kCols], en[kCols], sp = 0.f, sn = 0.f;
#pragma unroll
  for (int c = 0; c < kCols; ++c) {
    ep[c] = en[c] = 0.f;
    if (lane + 32 * c < Fh) {
      ep[c] = expf(u[c] - mx);  // softmax(u): shifted by max u
      en[c] = expf(mn - u[c]);  // softmax(-u): shifted by max(-u) = -min u
      sp += ep[c];
      sn += en[c];
    }
  }
  sp = warp_sum(sp);
  sn = warp_sum(sn);
#pragma unroll
  for (int c = 0; c < kCols; ++c) {
    const int f = lane + 32 * c;
    if (f < Fh) {
      out[f] = ep[c] / sp;
      out[Fh + f] = en[c] / sn;
    }
  }
}

template <typename T>
__device__ __forceinline__ void load_row(float* dst, const T* __restrict__ src, int n) {
  for (int i = threadIdx.x & 31; i < n; i += 32) dst[i] = to_f32(src[i]);
}

// ----------------------------------------------------------------- feature map
template <typename T, typename TO>
__global__ void __launch_bounds__(128) featuremap_simt(const T* __restrict__ x, int T_rows,
                                                       int H, int Hw, int d, int Fh,
                                                       const T* __restrict__ W,
                                                       TO* __restrict__ phi) {
  __shared__ float xs[4][kMaxD];
  __shared__ float ps[4][2 * kMaxFh];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const T* Wg = W + (size_t)((h * Hw) / H) * d * Fh;
  const int F = 2 * Fh;
  for (int t = blockIdx.x * 4 + warp; t < T_rows; t += gridDim.x * 4) {
    load_row(xs[warp], x + ((size_t)t * H + h) * d, d);
    __syncwarp();
    warp_phi(xs[warp], Wg, d, Fh, ps[warp]);
    __syncwarp();
    TO* o = phi + ((size_t)t * H + h) * F;
    for (int f = lane; f < F; f += 32) o[f] = from_f32<TO>(ps[warp][f]);
    __syncwarp();
  }
}

// ----------------------------------------------------------------- hybrid decode step
// One CTA per (request, query head); each warp handles queries i = warp, warp + 4, ...
template <typename T>
__global__ void __launch_bounds__(128) hybrid_simt(HybridArgs a) {
  __shared__ float qs[4][kMaxD];
  __shared__ float ss[4][kMaxB];
  __shared__ float ps[4][2 * kMaxFh];
  const int r = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  RowRange rr;
  int slot;
  const bool report = (h == 0 && threadIdx.x == 0);
  if (!request_rows(a.cu_blk, r, a.T, a.Bmax, a.dev_err, report, &rr)) return;
  if (rr.n == 0) return;
  if (!request_slot(a.state_slot, r, a.num_slots, a.dev_err, report, &slot)) return;

  const int d = a.d, Fh = a.F / 2, F = a.F, G = a.Hq / a.Hkv, g = h / G;
  const T* Qp = static_cast<const T*>(a.Q);
  const T* Kp = static_cast<const T*>(a.K);
  const T* Vp = static_cast<const T*>(a.V);
  const T* Wg = static_cast<const T*>(a.W) + (size_t)g * d * Fh;
  const float* Sg = a.S + ((size_t)slot * a.Hkv + g) * F * d;
  const float* Zg = a.Z + ((size_t)slot * a.Hkv + g) * F;
  const float w = a.alpha ? 1.f / (1.f + expf(-a.alpha[h])) : 1.f;
  const float scale = rsqrtf((float)d);

  for (int i = warp; i < rr.n; i += 4) {
    const int t = rr.lo + i;
    load_row(qs[warp], Qp + ((size_t)t * a.Hq + h) * d, d);
    __syncwarp();
    // scores s_j = q.k_j / sqrt(d) over every key of the block (no mask)
    for (int j = 0; j < rr.n; ++j) {
      const T* kr = Kp + ((size_t)(rr.lo + j) * a.Hkv + g) * d;
      float acc = 0.f;
      for (int k = lane; k < d; k += 32) acc = fmaf(qs[warp][k], to_f32(kr[k]), acc);
      acc = warp_sum(acc);
      if (lane == 0) ss[warp][j] = acc * scale;
    }
    __syncwarp();
    float m = -INFINITY;
    for (int j = lane; j < rr.n; j += 32) m = fmaxf(m, ss[warp][j]);
    m = warp_max(m);
    float den_sm = 0.f;
    for (int j = lane; j < rr.n; j += 32) {
      const float p = expf(ss[warp][j] - m);
      ss[warp][j] = p;
      den_sm += p;
    }
    den_sm = warp_sum(den_sm);
    __syncwarp();
    // sm_num (scaled by e^{-m}) over the lane's d columns
    float num_sm[kDCols];
#pragma unroll
    for (int c = 0; c < kDCols; ++c) num_sm[c] = 0.f;
    for (int j = 0; j < rr.n; ++j) {
      const float p = ss[warp][j];
      const T* vr = Vp + ((size_t)(rr.lo + j) * a.Hkv + g) * d;
#pragma unroll
      for (int c = 0; c < kDCols; ++c) {
        const int k = lane + 32 * c;
        if (k < d) num_sm[c] = fmaf(p, to_f32(vr[k]), num_sm[c]);
      }
    }
    // phi(q), then lin_num = phi^T S and lin_den = phi^T Z
    warp_phi(qs[warp], Wg, d, Fh, ps[warp]);
    __syncwarp();
    float den_lin = 0.f;
    for (int f = lane; f < F; f += 32) den_lin = fmaf(ps[warp][f], Zg[f], den_lin);
    den_lin = warp_sum(den_lin);
    float num_lin[kDCols];
#pragma unroll
    for (int c = 0; c < kDCols; ++c) num_lin[c] = 0.f;
    for (int f = 0; f < F; ++f) {
      const float p = ps[warp][f];
      const float* srow = Sg + (size_t)f * d;
#pragma unroll
      for (int c = 0; c < kDCols; ++c) {
        const int k = lane + 32 * c;
        if (k < d) num_lin[c] = fmaf(p, srow[k], num_lin[c]);
      }
    }
    // shared normaliser.  The softmax sums carry e^{-m}; both branches are brought to the
    // common scale e^{-M}, M = max(m, log den_lin), so that neither factor overflows (a
    // branch that underflows is negligible beside the other); states that are all zero add
    // nothing (den_lin = 0: the softmax branch alone, unscaled)
    float fsm = 1.f, flin = 0.f;
    if (den_lin > 0.f) {
      const float M = fmaxf(m, logf(den_lin));
      fsm = expf(m - M);
      flin = expf(-M);
    }
    const float den = w * den_sm * fsm + den_lin * flin;
    T* orow = static_cast<T*>(a.O) + ((size_t)t * a.Hq + h) * d;
#pragma unroll
    for (int c = 0; c < kDCols; ++c) {
      const int k = lane + 32 * c;
      if (k < d) {
        const float num = w * num_sm[c] * fsm + num_lin[c] * flin;
        orow[k] = from_f32<T>(den != 0.f ? num / den : 0.f);
      }
    }
    __syncwarp();
  }
}

// ----------------------------------------------------------------- block commit
// One CTA per (request, KV head): phi of 32 block tokens at a time into shared memory, then
// every (f, c) entry of S gets sum_t phi_t[f] v_t[c] and every Z[f] gets sum_t phi_t[f].
constexpr int kCommitChunk = 32;

template <typename T>
__global__ void __launch_bounds__(256) commit_simt(CommitArgs a) {
  extern __shared__ float smem[];
  const int r = blockIdx.x, g = blockIdx.y;
  const int warp = threadIdx.x >> 5;
  const int d = a.d, Fh = a.F / 2, F = a.F;
  float* phis = smem;                               // [32][F]
  float* vs = phis + kCommitChunk * F;              // [32][d]
  float* xs = vs + kCommitChunk * d;                // [8][d]
  RowRange rr;
  int slot;
  const bool report = (g == 0 && threadIdx.x == 0);
  if (!request_rows(a.cu_blk, r, a.T, a.Bmax, a.dev_err, report, &rr)) return;
  if (rr.n == 0) return;
  if (!request_slot(a.state_slot, r, a.num_slots, a.dev_err, report, &slot)) return;
  const T* Kp = static_cast<const T*>(a.K);
  const T* Vp = static_cast<const T*>(a.V);
  const T* Wg = static_cast<const T*>(a.W) + (size_t)g * d * Fh;
  float* Sg = a.S + ((size_t)slot * a.Hkv + g) * F * d;
  float* Zg = a.Z + ((size_t)slot * a.Hkv + g) * F;

  for (int t0 = 0; t0 < rr.n; t0 += kCommitChunk) {
    const int nt = min(kCommitChunk, rr.n - t0);
    for (int tt = warp; tt < nt; tt += 8) {
      const size_t row = (size_t)(rr.lo + t0 + tt) * a.Hkv + g;
      load_row(xs + warp * d, Kp + row * d, d);
      load_row(vs + tt * d, Vp + row * d, d);
      __syncwarp();
      warp_phi(xs + warp * d, Wg, d, Fh, phis + tt * F);
      __syncwarp();
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < F * d; idx += blockDim.x) {
      const int f = idx / d, c = idx - f * d;
      float acc = 0.f;
      for (int tt = 0; tt < nt; ++tt) acc = fmaf(phis[tt * F + f], vs[tt * d + c], acc);
      Sg[idx] += acc;
    }
    for (int f = threadIdx.x; f < F; f += blockDim.x) {
      float acc = 0.f;
      for (int tt = 0; tt < nt; ++tt) acc += phis[tt * F + f];
      Zg[f] += acc;
    }
    __syncthreads();
  }
}

// ----------------------------------------------------------------- softmax teacher
// One warp per (request, query head, query row); online softmax over the request's cache,
// 32 keys per step with one key per lane.
template <typename T>
__global__ void __launch_bounds__(128) full_prefix_simt(FullPrefixArgs a) {
  __shared__ float qs[4][kMaxD];
  const int r = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  RowRange rr;
  const bool report = (h == 0 && threadIdx.x == 0);
  if (!request_rows(a.cu_blk, r, a.T, a.Bmax, a.dev_err, report, &rr)) return;
  if (rr.n == 0) return;
  int L = a.kv_len[r];
  if (L < 0 || L > a.kv_capacity) {
    if (report) set_error(a.dev_err, BHA_ERR_INVALID);
    return;
  }
  const int d = a.d, G = a.Hq / a.Hkv, g = h / G;
  const T* Qp = static_cast<const T*>(a.Q);
  const T* Kc = static_cast<const T*>(a.Kc) + ((size_t)r * a.Hkv + g) * a.kv_capacity * d;
  const T* Vc = static_cast<const T*>(a.Vc) + ((size_t)r * a.Hkv + g) * a.kv_capacity * d;
  const float scale = rsqrtf((float)d);
  for (int i = blockIdx.z * 4 + warp; i < rr.n; i += gridDim.z * 4) {
    const int t = rr.lo + i;
    load_row(qs[warp], Qp + ((size_t)t * a.Hq + h) * d, d);
    __syncwarp();
    float m = -INFINITY, l = 0.f, acc[kDCols];
#pragma unroll
    for (int c = 0; c < kDCols; ++c) acc[c] = 0.f;
    for (int j0 = 0; j0 < L; j0 += 32) {
      const int j = j0 + lane;
      float s = -INFINITY;
      if (j < L) {
        const T* kr = Kc + (size_t)j * d;
        float dot = 0.f;
        for (int k = 0; k < d; ++k) dot = fmaf(qs[warp][k], to_f32(kr[k]), dot);
        s = dot * scale;
      }
      const float mc = warp_max(s);
      const float mn = fmaxf(m, mc);
      const float corr = expf(m - mn);  // m = -inf on the first chunk gives 0
      const float p = (j < L) ? expf(s - mn) : 0.f;
      l = l * corr + warp_sum(p);
#pragma unroll
      for (int c = 0; c < kDCols; ++c) acc[c] *= corr;
      const int nj = min(32, L - j0);
      for (int jj = 0; jj < nj; ++jj) {
        const float pj = __shfl_sync(0xffffffffu, p, jj);
        const T* vr = Vc + (size_t)(j0 + jj) * d;
#pragma unroll
        for (int c = 0; c < kDCols; ++c) {
          const int k = lane + 32 * c;
          if (k < d) acc[c] = fmaf(pj, to_f32(vr[k]), acc[c]);
        }
      }
      m = mn;
    }
    T* orow = static_cast<T*>(a.O) + ((size_t)t * a.Hq + h) * d;
#pragma unroll
    for (int c = 0; c < kDCols; ++c) {
      const int k = lane + 32 * c;
      if (k < d) orow[k] = from_f32<T>(l > 0.f ? acc[c] / l : 0.f);
    }
    __syncwarp();
  }
}

}  // namespace

// ----------------------------------------------------------------- launchers
bool simt_supports(int d, int F, int Bmax) {
  return d >= 1 && d <= kMaxD && F >= 2 && F <= 2 * kMaxFh && (F % 2) == 0 && Bmax >= 1 &&
         Bmax <= kMaxB;
}

cudaError_t launch_featuremap_simt(const void* x, int T_rows, int H, int Hw, int d, int F,
                                   const void* W, void* phi, bool act_bf16, bool out_bf16,
                                   cudaStream_t st) {
  if (T_rows == 0 || H == 0) return cudaSuccess;
  const int gx = (T_rows + 3) / 4 < 4096 ? (T_rows + 3) / 4 : 4096;
  dim3 grid(gx, H);
  const int Fh = F / 2;
  if (act_bf16) {
    auto xp = static_cast<const __nv_bfloat16*>(x);
    auto wp = static_cast<const __nv_bfloat16*>(W);
    if (out_bf16)
      featuremap_simt<<<grid, 128, 0, st>>>(xp, T_rows, H, Hw, d, Fh, wp,
                                            static_cast<__nv_bfloat16*>(phi));
    else
      featuremap_simt<<<grid, 128, 0, st>>>(xp, T_rows, H, Hw, d, Fh, wp,
                                            static_cast<float*>(phi));
  } else {
    auto xp = static_cast<const float*>(x);
    auto wp = static_cast<const float*>(W);
    if (out_bf16)
      featuremap_simt<<<grid, 128, 0, st>>>(xp, T_rows, H, Hw, d, Fh, wp,
                                            static_cast<__nv_bfloat16*>(phi));
    else
      featuremap_simt<<<grid, 128, 0, st>>>(xp, T_rows, H, Hw, d, Fh, wp,
                                            static_cast<float*>(phi));
  }
  return cudaGetLastError();
}

cudaError_t launch_hybrid_simt(const HybridArgs& a, bool act_bf16, cudaStream_t st) {
  if (a.R == 0) return cudaSuccess;
  dim3 grid(a.R, a.Hq);
  if (act_bf16)
    hybrid_simt<__nv_bfloat16><<<grid, 128, 0, st>>>(a);
  else
    hybrid_simt<float><<<grid, 128, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_commit_simt(const CommitArgs& a, bool act_bf16, cudaStream_t st) {
  if (a.R == 0) return cudaSuccess;
  dim3 grid(a.R, a.Hkv);
  const size_t smem = sizeof(float) * (kCommitChunk * a.F + kCommitChunk * a.d + 8 * a.d);
  cudaError_t e;
  if (act_bf16) {
    e = cudaFuncSetAttribute(commit_simt<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    commit_simt<__nv_bfloat16><<<grid, 256, smem, st>>>(a);
  } else {
    e = cudaFuncSetAttribute(commit_simt<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    commit_simt<float><<<grid, 256, smem, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_full_prefix_simt(const FullPrefixArgs& a, bool act_bf16, cudaStream_t st) {
  if (a.R == 0) return cudaSuccess;
  const int zsplit = (a.Bmax + 3) / 4;
  dim3 grid(a.R, a.Hq, zsplit);
  if (act_bf16)
    full_prefix_simt<__nv_bfloat16><<<grid, 128, 0, st>>>(a);
  else
    full_prefix_simt<float><<<grid, 128, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace bha
