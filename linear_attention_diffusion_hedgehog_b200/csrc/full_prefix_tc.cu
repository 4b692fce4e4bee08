// Tensor-core softmax teacher for sm_100a: exact attention of every active-block query over
// its request's whole KV cache (committed prefix followed by the active block), unmasked.
// bf16 activations, d = 128, four query heads per KV head, blocks of up to 32 tokens.
//
// Source: "Retrofitting Linear Attention into Diffusion Language Models", §2.2 (softmax
// attention, exp(q.k/sqrt d)-weighted average of the visible values) and Appendix A (the
// softmax kernel whose cost grows linearly with the prefix, kept here as the comparison
// point for the block-hybrid layer).
//
// Work unit: (request r, KV head g, KV split s).  The 4 query heads x 32 block rows of (r, g)
// form one 128-row MMA tile (as in the block-hybrid kernel); the unit sweeps its share of the
// cache in 128-key tiles:
//   S_i   = Q K_i^T              bf16 MMA into one of two TMEM score buffers (the next
//                                tile's scores are computed while this tile's softmax runs)
//   P_i   = 2^{S_i log2e/sqrt d - m_ref}   online softmax, one thread per row, P in bf16
//                                written to TMEM (two keys per column)
//   O    += P_i V_i              bf16 MMA with P from TMEM, accumulating in a TMEM O
// The reference max m_ref is raised only when a tile's row max exceeds it by more than
// kTau (log2 units); only then is the row's O (and l) rescaled in place, between two P V
// products, so P <= 2^kTau.  With one split the unit writes O / l; with several, it writes
// the unnormalised O, m_ref and l to the workspace and a combine kernel merges the splits.
// Keys at or past kv_len are masked by index and their V rows are cleared in shared memory,
// so whatever the cache holds there (even non-finite bytes) has no effect.
//
// Roles (192 threads): warp 0 TMA producer (Q per unit, K/V tiles through a 3-stage ring:
// P lives in TMEM, so shared memory holds only Q and the ring), warp 1 TMEM owner and MMA
// issuer, warps 2-5 softmax, rescaling and epilogue.  Every wait is bounded; on expiry the CTA
// records BHA_ERR_TIMEOUT, drains, frees TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_util.cuh"

namespace bha {
namespace {

constexpr int kD = 128;
constexpr int kG = 4;
constexpr int kBlk = 32;
constexpr int kM = kG * kBlk;  // 128 query rows
constexpr int kKT = 128;       // keys per tile
constexpr int kStages = 3;
constexpr int kThreads = 192;

constexpr uint32_t kQBytes = kM * kD * 2;    // 32 KiB: [d half][128 rows][128 B]
constexpr uint32_t kTileBytes = kKT * kD * 2;  // 32 KiB: [d half][128 keys][128 B]

constexpr uint32_t kColS = 0;    // two score buffers, 128 columns each
constexpr uint32_t kColO = 256;  // the output accumulator O (128 columns), P V accumulates here
constexpr uint32_t kColP = 384;  // P in bf16, two keys per column (64 columns), the A operand of P V
constexpr uint32_t kTmemCols = 512;
// Lazy rescaling: P is formed against a reference max m_ref that is raised only when a tile's
// row max exceeds it by more than kTau (log2 units), so P <= 2^kTau and O, l are rescaled in
// place only then.
constexpr float kTau = 8.f;

constexpr uint32_t kIdQK = tc::instr_desc(1, 0, 0, kM, kKT);
constexpr uint32_t kIdPV = tc::instr_desc(1, 0, 1, kM, kD);

struct __align__(1024) Smem {
  uint8_t q[kQBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  uint64_t q_full, q_empty, kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], s_free[2], p_full, pv_done, drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory budget");

struct Unit {
  int r, g, s, lo, n, L, t0, nt;  // nt: number of 128-key tiles this split covers
};

__device__ __forceinline__ bool decode_unit(const TcFullParams& p, int u, bool report, Unit* x) {
  x->s = u % p.nsplit;
  const int pair = u / p.nsplit;
  x->g = pair % p.Hkv;
  x->r = pair / p.Hkv;
  RowRange rr;
  if (!request_rows(p.cu_blk, x->r, p.T, p.Bmax, p.dev_err, report, &rr)) return false;
  if (rr.n == 0) return false;
  const int L = p.kv_len[x->r];
  if (L < 0 || L > p.cap) {
    if (report) set_error(p.dev_err, BHA_ERR_INVALID);
    return false;
  }
  x->lo = rr.lo;
  x->n = rr.n;
  x->L = L;
  const int tiles = (L + kKT - 1) / kKT;
  x->t0 = x->s * p.tiles_per_split;
  x->nt = max(0, min(tiles, x->t0 + p.tiles_per_split) - x->t0);
  return true;
}

__global__ void __launch_bounds__(kThreads, 1) full_prefix_tc_kernel(const __grid_constant__ TcFullParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;
  const long long lim = p.wait_limit;
  const int units = p.R * p.Hkv * p.nsplit;

  if (threadIdx.x == 0) {
    tc::mbar_init(&sm.q_full, 1);
    tc::mbar_init(&sm.q_empty, 1);
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&sm.kv_full[i], 1);
      tc::mbar_init(&sm.kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&sm.s_full[i], 1);
      tc::mbar_init(&sm.s_free[i], 4);
    }
    tc::mbar_init(&sm.p_full, 4);
    tc::mbar_init(&sm.pv_done, 1);
    tc::mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tensormap(&p.tm_q);
    tc::prefetch_tensormap(&p.tm_k);
    tc::prefetch_tensormap(&p.tm_v);
  }
  if (warp == 1) {
    tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int qk = 0, gt = 0;
      int armed_q = -1, armed_kv[kStages] = {-1, -1};
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        Unit x;
        if (!decode_unit(p, u, true, &x) || x.nt == 0) continue;
        if (qk >= 1 && !tc::mbar_wait(&sm.q_empty, (qk - 1) & 1, abort_flag, lim)) { ok = false; break; }
        tc::mbar_arrive_expect_tx(&sm.q_full, kQBytes);
        tc::tma_load_3d(sm.q, &p.tm_q, &sm.q_full, 0, kG * x.g, x.lo);
        tc::tma_load_3d(sm.q + kQBytes / 2, &p.tm_q, &sm.q_full, 64, kG * x.g, x.lo);
        armed_q = qk & 1;
        ++qk;
        const int row0 = (x.r * p.Hkv + x.g) * p.cap;
        for (int i = 0; i < x.nt; ++i, ++gt) {
          const int st = gt % kStages, j = gt / kStages;
          if (j >= 1 && !tc::mbar_wait(&sm.kv_empty[st], (j - 1) & 1, abort_flag, lim)) { ok = false; break; }
          tc::mbar_arrive_expect_tx(&sm.kv_full[st], 2 * kTileBytes);
          const int key0 = row0 + (x.t0 + i) * kKT;
          tc::tma_load_2d(sm.k[st], &p.tm_k, &sm.kv_full[st], 0, key0);
          tc::tma_load_2d(sm.k[st] + kTileBytes / 2, &p.tm_k, &sm.kv_full[st], 64, key0);
          tc::tma_load_2d(sm.v[st], &p.tm_v, &sm.kv_full[st], 0, key0);
          tc::tma_load_2d(sm.v[st] + kTileBytes / 2, &p.tm_v, &sm.kv_full[st], 64, key0);
          armed_kv[st] = j & 1;
        }
      }
      volatile int never = 0;
      if (armed_q >= 0) tc::mbar_wait(&sm.q_full, armed_q, &never, lim);
      for (int st = 0; st < kStages; ++st)
        if (armed_kv[st] >= 0) tc::mbar_wait(&sm.kv_full[st], armed_kv[st], &never, lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int qk = 0, gt = 0;
      bool ok = true, issued = false;
      // O (+)= P_tile V_tile: the first tile of a unit overwrites O, the others accumulate
      // (the softmax warps rescale O in place, between two of these, when m_ref rises)
      auto issue_pv = [&](int tile, bool first) -> bool {
        const int st = tile % kStages;
        if (!tc::mbar_wait(&sm.p_full, tile & 1, abort_flag, lim)) return false;
        tc::tc_fence_after();
        const uint32_t va = tc::smem_u32(sm.v[st]);
#pragma unroll
        for (int kk = 0; kk < kKT / 16; ++kk) {
          const uint64_t b = tc::smem_desc(va + kk * 2048, kTileBytes / 2, 1024, tc::kSwizzle128B);
          tc::mma_bf16_ts(tbase + kColO, tbase + kColP + kk * 8, b, kIdPV, (first && kk == 0) ? 0u : 1u);
        }
        tc::mma_commit(&sm.pv_done);
        tc::mma_commit(&sm.kv_empty[st]);
        return true;
      };
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        Unit x;
        if (!decode_unit(p, u, false, &x) || x.nt == 0) continue;
        if (!tc::mbar_wait(&sm.q_full, qk & 1, abort_flag, lim)) { ok = false; break; }
        ++qk;
        const uint32_t qa = tc::smem_u32(sm.q);
        for (int i = 0; i < x.nt; ++i, ++gt) {
          const int st = gt % kStages, sb = gt & 1;
          if (!tc::mbar_wait(&sm.kv_full[st], (gt / kStages) & 1, abort_flag, lim)) { ok = false; break; }
          if (gt >= 2 && !tc::mbar_wait(&sm.s_free[sb], ((gt >> 1) - 1) & 1, abort_flag, lim)) { ok = false; break; }
          tc::tc_fence_after();
          const uint32_t ka = tc::smem_u32(sm.k[st]);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t a = tc::smem_desc(qa + (kk >> 2) * (kQBytes / 2) + (kk & 3) * 32, 16, 1024, tc::kSwizzle128B);
            const uint64_t b = tc::smem_desc(ka + (kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32, 16, 1024, tc::kSwizzle128B);
            tc::mma_bf16_ss(tbase + kColS + sb * 128, a, b, kIdQK, kk > 0);
          }
          tc::mma_commit(&sm.s_full[sb]);
          if (i == x.nt - 1) tc::mma_commit(&sm.q_empty);
          issued = true;
          if (i >= 1 && !issue_pv(gt - 1, i == 1)) { ok = false; break; }
        }
        if (!ok) break;
        if (!issue_pv(gt - 1, x.nt == 1)) { ok = false; break; }
      }
      if (issued) {
        volatile int never = 0;
        tc::mma_commit(&sm.drain);
        tc::mbar_wait(&sm.drain, 0, &never, lim);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / accumulation / epilogue
    const int wq = warp & 3;
    const int row = wq * 32 + lane;          // 4 t + head-in-group
    const int t = row >> 2, hl = row & 3;
    const int tid = threadIdx.x - 64;        // 0..127
    const uint32_t tl = tbase + ((uint32_t)(wq * 32) << 16);
    const float scale_log2 = 1.4426950408889634f * 0.08838834764831845f;  // log2(e)/sqrt(128)
    int gt = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      Unit x;
      if (!decode_unit(p, u, false, &x)) continue;
      // m_ref: the reference max P is formed against (log2 units); l: sum of P against it
      float m = -INFINITY, l = 0.f;
      for (int i = 0; i < x.nt; ++i, ++gt) {
        const int sb = gt & 1, st = gt % kStages;
        if (!tc::mbar_wait(&sm.s_full[sb], (gt >> 1) & 1, abort_flag, lim)) { ok = false; break; }
        tc::tc_fence_after();
        const int key0 = (x.t0 + i) * kKT;
        const int valid_keys = min(kKT, x.L - key0);
        const uint32_t scol = tl + kColS + sb * 128;
        // the row's 128 scores of this tile, scaled to log2 units; keys at or past kv_len -inf
        float sv[kKT];
#pragma unroll
        for (int c = 0; c < kKT / 32; ++c) tc::tmem_ld32(scol + c * 32, *reinterpret_cast<float(*)[32]>(sv + c * 32));
        tc::tmem_wait_ld();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sm.s_free[sb]);  // the score buffer may be refilled
        float tmax = -INFINITY;
#pragma unroll
        for (int j = 0; j < kKT; ++j) {
          sv[j] = j < valid_keys ? sv[j] * scale_log2 : -INFINITY;
          tmax = fmaxf(tmax, sv[j]);
        }
        // the P buffer (and O) are free once the previous tile's P V has completed
        if (gt >= 1 && !tc::mbar_wait(&sm.pv_done, (gt - 1) & 1, abort_flag, lim)) { ok = false; break; }
        tc::tc_fence_after();
        if (i == 0) {
          m = tmax;  // every tile of a split holds at least one key below kv_len
        } else if (tmax > m + kTau) {
          // raise m_ref: O and l are rescaled in place before this tile's P V accumulates
          const float alpha = tc::ex2(m - tmax);
#pragma unroll 1
          for (int c = 0; c < kD / 32; ++c) {
            float ov[32];
            tc::tmem_ld32(tl + kColO + c * 32, ov);
            tc::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) ov[j] *= alpha;
            tc::tmem_st32(tl + kColO + c * 32, ov);
          }
          tc::tmem_wait_st();
          l *= alpha;
          m = tmax;
        }
        // P = 2^{s - m_ref} in bf16, two keys per TMEM column (the A operand of P V)
        float psum = 0.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[32];
#pragma unroll
          for (int j = 0; j < 64; j += 2) {
            const float a0 = tc::ex2(sv[c * 64 + j] - m);   // 2^-inf = 0 for masked keys
            const float a1 = tc::ex2(sv[c * 64 + j + 1] - m);
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(a0, a1);
            psum += __low2float(b2) + __high2float(b2);
            pk[j >> 1] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          tc::tmem_st16u(tl + kColP + c * 32, *reinterpret_cast<const uint32_t(*)[16]>(pk));
          tc::tmem_st16u(tl + kColP + c * 32 + 16, *reinterpret_cast<const uint32_t(*)[16]>(pk + 16));
        }
        tc::tmem_wait_st();
        l += psum;
        if (valid_keys < kKT) {
          // V rows past kv_len are cleared (the cache may hold anything there)
          const int per_half = (kKT - valid_keys) * 8;
          for (int q = tid; q < 2 * per_half; q += 128) {
            const int hh = q / per_half, rem = q % per_half;
            *reinterpret_cast<uint4*>(sm.v[st] + hh * (kTileBytes / 2) + (valid_keys + rem / 8) * 128 + (rem % 8) * 16) =
                make_uint4(0, 0, 0, 0);
          }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sm.p_full);
      }
      if (!ok) break;
      // O of this unit is complete once its last P V has
      if (x.nt > 0) {
        if (!tc::mbar_wait(&sm.pv_done, (gt - 1) & 1, abort_flag, lim)) { ok = false; break; }
        tc::tc_fence_after();
      }
      float o[kD];
#pragma unroll
      for (int c = 0; c < kD / 32; ++c) {
        if (x.nt > 0) {
          tc::tmem_ld32(tl + kColO + c * 32, *reinterpret_cast<float(*)[32]>(o + c * 32));
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) o[c * 32 + j] = 0.f;
        }
      }
      tc::tmem_wait_ld();
      // epilogue
      if (t < x.n) {
        const size_t orow = (size_t)(x.lo + t) * p.Hq + kG * x.g + hl;
        if (p.nsplit == 1) {
          const float inv = l > 0.f ? 1.f / l : 0.f;
          __nv_bfloat16* op = p.O + orow * kD;
          // output rows are not read back here: no L1 allocation, whole 32-byte sectors when
          // O is 32-byte aligned
          if (p.o32) {
#pragma unroll
            for (int c = 0; c < kD; c += 16) {
              uint32_t w[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) w[j] = pack_bf16(o[c + 2 * j] * inv, o[c + 2 * j + 1] * inv);
              tc::st_global_32B(op + c, w);
            }
          } else {
#pragma unroll
            for (int c = 0; c < kD; c += 8)
              tc::st_global_16B(op + c, pack_bf16(o[c] * inv, o[c + 1] * inv), pack_bf16(o[c + 2] * inv, o[c + 3] * inv),
                                pack_bf16(o[c + 4] * inv, o[c + 5] * inv), pack_bf16(o[c + 6] * inv, o[c + 7] * inv));
          }
        } else {
          const size_t prow = (size_t)x.s * p.T * p.Hq + orow;
          float* op = p.opart + prow * kD;
#pragma unroll
          for (int c = 0; c < kD; c += 4)
            tc::st_global_16B(op + c, __float_as_uint(o[c]), __float_as_uint(o[c + 1]), __float_as_uint(o[c + 2]),
                              __float_as_uint(o[c + 3]));
          p.mpart[prow] = m;
          p.lpart[prow] = l;
        }
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tbase, kTmemCols);
  if (threadIdx.x == 0 && sm.abort_flag) set_error(p.dev_err, BHA_ERR_TIMEOUT);
}

// Merges the splits of one (request, query head): O = sum_s 2^{m_s - m*} O_s / sum_s 2^{m_s - m*} l_s.
__global__ void __launch_bounds__(128) combine_splits_kernel(const TcFullParams p) {
  const int r = blockIdx.x, h = blockIdx.y, d = threadIdx.x;
  RowRange rr;
  if (!request_rows(p.cu_blk, r, p.T, p.Bmax, p.dev_err, false, &rr)) return;
  const int L = p.kv_len[r];
  if (L < 0 || L > p.cap) return;
  for (int i = 0; i < rr.n; ++i) {
    const size_t orow = (size_t)(rr.lo + i) * p.Hq + h;
    float mx = -INFINITY;
    for (int s = 0; s < p.nsplit; ++s) mx = fmaxf(mx, p.mpart[(size_t)s * p.T * p.Hq + orow]);
    float num = 0.f, den = 0.f;
    if (mx != -INFINITY) {
      for (int s = 0; s < p.nsplit; ++s) {
        const size_t prow = (size_t)s * p.T * p.Hq + orow;
        const float ms = p.mpart[prow];
        if (ms == -INFINITY) continue;
        const float w = tc::ex2(ms - mx);
        num = fmaf(w, p.opart[prow * kD + d], num);
        den = fmaf(w, p.lpart[prow], den);
      }
    }
    p.O[orow * kD + d] = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
  }
}

}  // namespace

bool full_prefix_tc_supports(const FullPrefixArgs& a, bool act_bf16) {
  return act_bf16 && a.d == kD && a.Hq == kG * a.Hkv && a.Bmax <= kBlk &&
         (long long)a.R * a.Hkv * (a.kv_capacity + kKT) < (1ll << 31);
}

// Number of KV splits per (request, KV head): enough units to cover the SMs several times,
// each split at least 4 tiles long.  Depends only on the call's dims and cache capacity.
// Number of key-range splits per (request, KV head).  Cost model in units of one 128-key
// K/V tile (64 KiB): a unit of work costs its tiles plus its 32 KiB Q tile and 32 KiB output
// (1 tile), and with splits also its fp32 partial output written and read back by the
// combine step (about 2 more tiles); the grid runs ceil(units / SMs) rounds.  The split count
// with the least (rounds x cost per unit) wins, keeping at least 4 tiles per split.  The SM
// count is fixed at 148 so that the workspace size does not depend on the device.
int full_prefix_splits(int R, int Hkv, int64_t cap) {
  const long long pairs = (long long)R * Hkv;
  const long long tiles = (cap + kKT - 1) / kKT;
  if (pairs <= 0 || tiles <= 0) return 1;
  const long long nsm = 148;
  long long most = (tiles + 3) / 4;
  if (most > 64) most = 64;
  if (most < 1) most = 1;
  long long best = 1;
  double best_cost = 0.0;
  for (long long s = 1; s <= most; ++s) {
    const long long rounds = (pairs * s + nsm - 1) / nsm;
    const double per_unit = (double)((tiles + s - 1) / s) + (s == 1 ? 1.0 : 3.1);
    const double cost = (double)rounds * per_unit;
    if (s == 1 || cost < best_cost) {
      best = s;
      best_cost = cost;
    }
  }
  return (int)best;
}

size_t full_prefix_tc_workspace(const FullPrefixArgs& a) {
  const int ns = full_prefix_splits(a.R, a.Hkv, a.kv_capacity);
  if (ns <= 1) return 0;
  return (size_t)ns * a.T * a.Hq * (kD + 2) * sizeof(float);
}

cudaError_t launch_full_prefix_tc(const FullPrefixArgs& a, void* workspace, cudaStream_t st) {
  TcFullParams p;
  {
    const uint64_t dims[3] = {kD, (uint64_t)a.Hq, (uint64_t)a.T};
    const uint64_t strides[2] = {kD * 2, (uint64_t)a.Hq * kD * 2};
    const uint32_t box[3] = {64, kG, kBlk};
    if (!make_tensor_map(&p.tm_q, false, 3, a.Q, dims, strides, box, kTma128B)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {kD, (uint64_t)a.R * a.Hkv * a.kv_capacity};
    const uint64_t strides[1] = {kD * 2};
    const uint32_t box[2] = {64, kKT};
    if (!make_tensor_map(&p.tm_k, false, 2, a.Kc, dims, strides, box, kTma128B)) return cudaErrorInvalidValue;
    if (!make_tensor_map(&p.tm_v, false, 2, a.Vc, dims, strides, box, kTma128B)) return cudaErrorInvalidValue;
  }
  p.cu_blk = a.cu_blk;
  p.kv_len = a.kv_len;
  p.O = static_cast<__nv_bfloat16*>(a.O);
  p.o32 = (reinterpret_cast<uintptr_t>(a.O) & 31) == 0;
  p.dev_err = a.dev_err;
  p.R = a.R;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.T = a.T;
  p.Bmax = a.Bmax;
  p.cap = (int)a.kv_capacity;
  p.nsplit = full_prefix_splits(a.R, a.Hkv, a.kv_capacity);
  const int tiles_cap = (int)((a.kv_capacity + kKT - 1) / kKT);
  p.tiles_per_split = (tiles_cap + p.nsplit - 1) / p.nsplit;
  if (p.tiles_per_split < 1) p.tiles_per_split = 1;
  p.wait_limit = 2000000000ll;
  if (p.nsplit > 1) {
    float* ws = static_cast<float*>(workspace);
    const size_t rows = (size_t)p.nsplit * a.T * a.Hq;
    p.opart = ws;
    p.mpart = ws + rows * kD;
    p.lpart = p.mpart + rows;
  } else {
    p.opart = p.mpart = p.lpart = nullptr;
  }
  const int units = a.R * a.Hkv * p.nsplit;
  int nsm = device_sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  // fewest CTAs that finish in the same number of rounds
  const int rounds = (units + nsm - 1) / nsm;
  int grid = (units + rounds - 1) / rounds;
  if (grid > nsm) grid = nsm;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(full_prefix_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  full_prefix_tc_kernel<<<grid, kThreads, smem, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.nsplit == 1) return e;
  combine_splits_kernel<<<dim3(a.R, a.Hq), 128, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace bha
