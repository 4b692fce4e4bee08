// Tensor-core decode step fused with the block commit, for the last denoising step of a block
// (sm_100a; bf16 activations, d = 128, F = 256, G = 1, 2 or 4 query heads per KV head, blocks
// of up to 32 tokens).
//
// Source: "Retrofitting Linear Attention into Diffusion Language Models", §3.1 and §3.3: the
// output of the step reads the states of the committed blocks,
//   out = (w sm_num + phi(q)^T S) / (w sm_den + phi(q)^T Z),
// and the finished block is then folded in, S += sum_t phi(k_t) v_t^T, Z += sum_t phi(k_t);
// in §3.3 a single kernel launch does both, the state update included.
//
// Each (request, KV head) unit runs the decode step exactly as the decode-only kernel does
// (the same roles, rings, feature map and shared-normaliser merge; the states are read once,
// through the S ring), then its commit:
//   u_k  = K W_g                  bf16 MMA, M 128 (the 32 block rows from the unit's own K
//                                  buffer, which the next unit's K waits for; the other
//                                  rows are ignored), N 128, into the feature-map columns
//                                  the unit has finished with
//   phi  = [softmax(u_k), softmax(-u_k)] per block row: the feature-map warp of TMEM lane
//          quarter 0 stages u_k's 32 rows in the second half of the ring stage the unit's last
//          state group has released (fp32), then all eight feature-map and epilogue
//          warps (idle between the unit's output and its dS^T) form phi, eight threads per row
//          agreeing on its max, min and sums by shuffles, rounded to bf16 into the stage's
//          first half (the producer holds the stage back until dS^T and dZ have read it);
//          rows past the block are zero
//   dZ   = column sums of the bf16 phi (one column per thread of the eight warps), added to
//          Z with reducing atomics
//   dS^T = V^T phi                 bf16 MMA, M 128 (d), N 256 (F), K 32, into the accumulator
//                                  columns once the epilogue has read the output
//   S   += dS                      the epilogue warps add dS^T into S with reducing atomics
//                                  straight from TMEM (lane = d: each warp instruction is one
//                                  128-byte row piece); the lines were read by this unit's
//                                  state stream moments before, so L2 serves the
//                                  read-modify-write and S crosses HBM once each way.
// dS^T is issued as soon as phi is in shared memory and the output has been read, and the
// next unit's u and s right after it, so the drain starts early and the next unit's feature
// map runs while dS^T is drained.
//
// Every wait is bounded; on expiry the CTA raises BHA_ERR_TIMEOUT in dev_err, drains its
// own copies and MMAs, frees its TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_util.cuh"

namespace bha {
namespace {

constexpr int kD = 128;
constexpr int kF = 256;
constexpr int kFh = 128;
constexpr int kG = 4;            // query heads per KV head that fill the 128-row tile
constexpr int kBlk = 32;
constexpr int kM = kG * kBlk;  // 128 tile rows
constexpr int kChunk = 32;         // F rows of S per chunk = one group of 32 e values
constexpr int kGroups = kFh / kChunk;  // groups of 32 e values per half
constexpr int kStages = 4;         // S ring: each stage holds group g of both halves
constexpr int kThreads = 320;

constexpr uint32_t kQBytes = kM * kD * 2;      // 32 KiB
constexpr uint32_t kKBytes = kBlk * kD * 2;    // 8 KiB
constexpr uint32_t kZBytes = kF * 4;           // 1 KiB
constexpr uint32_t kWBytes = kD * kFh * 2;     // 32 KiB
constexpr uint32_t kSBytes = kChunk * kD * 4;  // 16 KiB fp32: [d quarter][32 rows][128 B]
constexpr uint32_t kPBytes = kM * 64;          // 8 KiB (64-byte rows, 64-byte swizzle)

// TMEM columns
constexpr uint32_t kColU = 0;      // u = Q W_g, then e+ in place
constexpr uint32_t kColEm = 128;   // e-
constexpr uint32_t kColS = 224;    // block scores (32 columns, top of the e- block)
constexpr uint32_t kColAm = 256;   // A- accumulator
constexpr uint32_t kColAp = 384;   // A+ accumulator (also receives P V)
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kIdQW = tc::instr_desc(1, 0, 1, kM, kFh);   // bf16, B MN-major
constexpr uint32_t kIdQK = tc::instr_desc(1, 0, 0, kM, kBlk);  // bf16, B K-major
constexpr uint32_t kIdPV = tc::instr_desc(1, 0, 1, kM, kD);    // bf16, B MN-major
constexpr uint32_t kIdES = tc::instr_desc(2, 0, 1, kM, kD);    // tf32, A from TMEM, B MN-major
constexpr uint32_t kIdVP = tc::instr_desc(1, 1, 1, kD, kF);    // bf16, A MN-major (V^T), B MN-major
constexpr uint32_t kPhiBytes = kBlk * kF * 2;  // 16 KiB: [F quarter][32 rows][128 B]
constexpr int kCommitStage = kStages - 1;       // ring stage lent to the commit

struct __align__(1024) Smem {
  uint8_t q[kQBytes];           // [d half][128 rows][128 B], 128-byte swizzle
  uint8_t w[kWBytes];           // [f half][128 rows of d][128 B]
  uint8_t s[kStages][2][kSBytes];  // group g of S+ and S-: fp32 [d quarter][32 rows][128 B],
                                   // 32-byte-atom swizzle
  uint8_t k[kKBytes];           // [d half][32 rows][128 B]
  uint8_t v[kKBytes];
  uint8_t p[kPBytes];           // P: [128 rows][64 B], 64-byte swizzle
  float z[2][kF];
  float fin[2][2][kM];          // per unit (double-buffered): epilogue factors c+/den, c-/den
  uint64_t q_full, k_full, qk_empty, v_full, v_empty, v_ready, z_full[2], z_empty[2];
  uint64_t s_full[kStages], s_empty[kStages];
  uint64_t e_ready[kGroups], p_ready;
  uint64_t w_full, u_full, s_ready, acc_full, acc_empty, drain, fin_full[2], fin_empty[2];
  uint64_t uk_done, u_staged, phi_ready, ds_full, ds_empty, commit_done;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory budget of one CTA per SM");
static_assert(kStages <= kGroups, "V is loaded ahead of the S pair that reuses the first stage");

struct Unit {
  int r, g, lo, n, slot;
};

// Decodes unit u and validates it; every role calls this with the same arguments and so
// skips the same units.
// Order in which the S pairs are loaded and contracted: the order the feature-map warps
// produce the groups.
__device__ __forceinline__ int group_at(int i) { return i; }

__device__ __forceinline__ bool decode_unit(const TcHybridParams& p, int u, bool report, Unit* x) {
  x->g = u % p.Hkv;
  x->r = u / p.Hkv;
  RowRange rr;
  if (!request_rows(p.cu_blk, x->r, p.T, p.Bmax, p.dev_err, report, &rr)) return false;
  if (rr.n == 0) return false;
  x->lo = rr.lo;
  x->n = rr.n;
  return request_slot(p.state_slot, x->r, p.num_slots, p.dev_err, report, &x->slot);
}

// Next valid unit of this CTA at or after *u; advances *u past it.
__device__ __forceinline__ bool next_unit(const TcHybridParams& p, int units, int* u, bool report,
                                          Unit* x) {
  for (; *u < units; *u += gridDim.x)
    if (decode_unit(p, *u, report, x)) {
      *u += gridDim.x;
      return true;
    }
  return false;
}

// phi of the block's rows from u_k staged in shared memory (U: [32 rows][128] fp32, float4
// slot j of row t at slot j ^ (t % 8)), by the eight feature-map and epilogue warps: thread
// gt (0..255) owns row t = gt / 8 and the float4 slots s8 + 8 i (i = 0..3, s8 = gt % 8), i.e.
// u columns 4 s8 + 32 i + m, so the eight lanes of a row read eight different bank groups and
// agree on its max, min and sums by shuffles.  phi = [e+ / sum e+, e- / sum e-] rounded to
// bf16 into phib as the B operand of dS^T: F quarter a = f / 64, row t, 16-byte chunk
// (f % 64) / 8 stored at chunk ^ (t % 8); rows past the block (t >= n) are written as zeros.
__device__ __forceinline__ void block_phi(const float* U, uint8_t* phib, int gt, int n) {
  const float log2e = 1.4426950408889634f;
  const int t = gt >> 3, s8 = gt & 7;
  float u[16];
  const float4* src = reinterpret_cast<const float4*>(U + t * kFh);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 v = src[(s8 + 8 * i) ^ (t & 7)];
    u[4 * i] = v.x;
    u[4 * i + 1] = v.y;
    u[4 * i + 2] = v.z;
    u[4 * i + 3] = v.w;
  }
  float mx = u[0], mn = u[0];
#pragma unroll
  for (int i = 1; i < 16; ++i) {
    mx = fmaxf(mx, u[i]);
    mn = fminf(mn, u[i]);
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  const float bx = mx * log2e, bn = mn * log2e;
  float ep[16], em[16], sp = 0.f, sm_ = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float a = u[i] * log2e;
    ep[i] = tc::ex2(a - bx);
    em[i] = tc::ex2(bn - a);
    sp += ep[i];
    sm_ += em[i];
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    sp += __shfl_xor_sync(0xffffffffu, sp, o);
    sm_ += __shfl_xor_sync(0xffffffffu, sm_, o);
  }
  const bool live = t < n;
  const float ip = 1.f / sp, im = 1.f / sm_;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float* e = h ? em : ep;
    const float sc = h ? im : ip;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // features h F/2 + 4 s8 + 32 i + (0..3): F quarter 2 h + i / 2, chunk s8 / 2 + 4 (i % 2),
      // bytes 8 (s8 % 2) .. + 7 of the chunk
      const int ch = (s8 >> 1) + 4 * (i & 1);
      uint8_t* dst = phib + (2 * h + (i >> 1)) * (kPhiBytes / 4) + t * 128 + ((ch ^ (t & 7)) << 4) + (s8 & 1) * 8;
      uint2 v = make_uint2(0, 0);
      if (live) v = make_uint2(pack_bf16(e[4 * i] * sc, e[4 * i + 1] * sc), pack_bf16(e[4 * i + 2] * sc, e[4 * i + 3] * sc));
      *reinterpret_cast<uint2*>(dst) = v;
    }
  }
}

// dZ[f]: the column sum of the bf16 phi over the block's n rows.
__device__ __forceinline__ float block_dz(const uint8_t* phib, int f, int n) {
  const int quarter = f >> 6, ch = (f & 63) >> 3, w8 = f & 7;
  const uint8_t* base = phib + quarter * (kPhiBytes / 4) + w8 * 2;
  float acc = 0.f;
  for (int tt = 0; tt < n; ++tt)
    acc += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + tt * 128 + ((ch ^ (tt & 7)) << 4)));
  return acc;
}

__global__ void __launch_bounds__(kThreads, 1) hybrid_commit_tc_kernel(const __grid_constant__ TcHybridCommitParams pc) {
  const TcHybridParams& p = pc.h;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;
  const long long lim = p.wait_limit;
  const int units = p.R * p.Hkv;

  if (threadIdx.x == 0) {
    tc::mbar_init(&sm.q_full, 1);
    tc::mbar_init(&sm.k_full, 1);
    tc::mbar_init(&sm.qk_empty, 1);
    tc::mbar_init(&sm.v_full, 1);
    tc::mbar_init(&sm.v_empty, 1);
    tc::mbar_init(&sm.v_ready, 4);  // the four feature-map warps clear V rows past a short block
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&sm.z_full[i], 1);
      tc::mbar_init(&sm.z_empty[i], 4);
      tc::mbar_init(&sm.fin_full[i], 4);   // the four feature-map warps
      tc::mbar_init(&sm.fin_empty[i], 4);  // the four epilogue warps
    }
    for (int j = 0; j < kGroups; ++j) tc::mbar_init(&sm.e_ready[j], 4);  // the 4 feature-map warps
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&sm.s_full[i], 1);
      tc::mbar_init(&sm.s_empty[i], 1);
    }
    tc::mbar_init(&sm.p_ready, 4);
    tc::mbar_init(&sm.w_full, 1);
    tc::mbar_init(&sm.u_full, 1);
    tc::mbar_init(&sm.s_ready, 1);
    tc::mbar_init(&sm.acc_full, 1);
    tc::mbar_init(&sm.acc_empty, 4);  // the four epilogue warps
    tc::mbar_init(&sm.drain, 1);
    tc::mbar_init(&sm.uk_done, 1);
    tc::mbar_init(&sm.u_staged, 1);     // the feature-map warp of lane quarter 0 (the block rows)
    tc::mbar_init(&sm.phi_ready, 8);    // the feature-map and epilogue warps, 4 block rows each
    tc::mbar_init(&sm.ds_full, 1);
    tc::mbar_init(&sm.ds_empty, 4);     // the four epilogue warps
    tc::mbar_init(&sm.commit_done, 8);  // the feature-map and epilogue warps, done reading phi
    sm.abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tensormap(&p.tm_q);
    tc::prefetch_tensormap(&p.tm_k);
    tc::prefetch_tensormap(&p.tm_v);
    tc::prefetch_tensormap(&p.tm_w);
    tc::prefetch_tensormap(&p.tm_s);
  }
  if (warp == 1) {
    tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = sm.tmem_base;
  // phi and dZ of unit k's block by the eight feature-map and epilogue warps (gt = 0..255):
  // waits for the staged u_k, writes phi into the lent stage, and once every warp's rows are
  // there sums this thread's column f = gt into Z.
  auto commit_phi = [&](const Unit& y, int k, int gt) -> bool {
    if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.u_staged, k & 1, abort_flag, lim))) return false;
    uint8_t* phib = sm.s[kCommitStage][0];
    block_phi(reinterpret_cast<const float*>(sm.s[kCommitStage][1]), phib, gt, y.n);
    tc::fence_proxy_async_smem();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) tc::mbar_arrive(&sm.phi_ready);
    if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.phi_ready, k & 1, abort_flag, lim))) return false;
    atomicAdd(pc.Zw + ((size_t)y.slot * p.Hkv + y.g) * kF + gt, block_dz(phib, gt, y.n));
    __syncwarp();
    if ((threadIdx.x & 31) == 0) tc::mbar_arrive(&sm.commit_done);  // done reading the lent stage
    return true;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int g_res = -1, q = 0;
      uint32_t w_loads = 0;
      int armed_q = -1, armed_k = -1, armed_v = -1, armed_w = -1, armed_z[2] = {-1, -1};
      int armed_s[kStages];
#pragma unroll
      for (int i = 0; i < kStages; ++i) armed_s[i] = -1;
      bool ok = true;
      int ucur = blockIdx.x;
      Unit x{};
      for (int k = 0; ok && next_unit(p, units, &ucur, true, &x); ++k) {
        if (x.g != g_res) {
          // W is read by each unit's u and by its commit's u_k: the previous unit's must be done
          if (k >= 1 && !tc::mbar_wait(&sm.uk_done, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
          tc::mbar_arrive_expect_tx(&sm.w_full, kWBytes);
          tc::tma_load_2d(sm.w, &p.tm_w, &sm.w_full, 0, x.g * kD);
          tc::tma_load_2d(sm.w + kWBytes / 2, &p.tm_w, &sm.w_full, 64, x.g * kD);
          armed_w = w_loads & 1;
          ++w_loads;
          g_res = x.g;
        }
        if (k >= 1 && !tc::mbar_wait(&sm.qk_empty, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
        // Q: two d halves of 32 G rows, each at the start of its 16 KiB half of the tile
        tc::mbar_arrive_expect_tx(&sm.q_full, (kQBytes / kG) * p.G);
        tc::tma_load_3d(sm.q, &p.tm_q, &sm.q_full, 0, p.G * x.g, x.lo);
        tc::tma_load_3d(sm.q + kQBytes / 2, &p.tm_q, &sm.q_full, 64, p.G * x.g, x.lo);
        armed_q = k & 1;
        // K stays until the previous unit's commit has read its own K (u_k): the first unit's
        // goes out now, the others just ahead of the last S pair (below)
        if (k == 0) {
          tc::mbar_arrive_expect_tx(&sm.k_full, kKBytes);
          tc::tma_load_3d(sm.k, &p.tm_k, &sm.k_full, 0, x.g, x.lo);
          tc::tma_load_3d(sm.k + kKBytes / 2, &p.tm_k, &sm.k_full, 64, x.g, x.lo);
          armed_k = 0;
        }
        const int zb = k & 1, zj = k >> 1;
        if (zj >= 1 && !tc::mbar_wait(&sm.z_empty[zb], (zj - 1) & 1, abort_flag, lim)) { ok = false; break; }
        tc::mbar_arrive_expect_tx(&sm.z_full[zb], kZBytes);
        tc::bulk_load(sm.z[zb], p.Z + ((size_t)x.slot * p.Hkv + x.g) * kF, kZBytes, &sm.z_full[zb]);
        armed_z[zb] = zj & 1;
        const int srow0 = (x.slot * p.Hkv + x.g) * kF;
        for (int i = 0; i < kGroups; ++i, ++q) {
          const int grp = group_at(i);
          if (i == kStages - 1) {
            // this unit's K once the previous unit's commit has read its own (u_k), then V of
            // this unit (once the previous commit's dS^T has read V), then the last S pair goes
            // into the stage the previous commit borrowed, once that commit is done
            if (k >= 1) {
              if (!tc::mbar_wait(&sm.uk_done, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
              tc::mbar_arrive_expect_tx(&sm.k_full, kKBytes);
              tc::tma_load_3d(sm.k, &p.tm_k, &sm.k_full, 0, x.g, x.lo);
              tc::tma_load_3d(sm.k + kKBytes / 2, &p.tm_k, &sm.k_full, 64, x.g, x.lo);
              armed_k = k & 1;
            }
            if (k >= 1 && !tc::mbar_wait(&sm.v_empty, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
            tc::mbar_arrive_expect_tx(&sm.v_full, kKBytes);
            tc::tma_load_3d(sm.v, &p.tm_v, &sm.v_full, 0, x.g, x.lo);
            tc::tma_load_3d(sm.v + kKBytes / 2, &p.tm_v, &sm.v_full, 64, x.g, x.lo);
            armed_v = k & 1;
            if (k >= 1 && !tc::mbar_wait(&sm.commit_done, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
          }
          const int st = q % kStages, j = q / kStages;
          if (j >= 1 && !tc::mbar_wait(&sm.s_empty[st], (j - 1) & 1, abort_flag, lim)) { ok = false; break; }
          tc::mbar_arrive_expect_tx(&sm.s_full[st], 2 * kSBytes);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int dq = 0; dq < 4; ++dq)
              tc::tma_load_2d(sm.s[st][hf] + dq * (kSBytes / 4), &p.tm_s, &sm.s_full[st], dq * 32,
                              srow0 + hf * kFh + grp * kChunk);
          armed_s[st] = j & 1;
        }
      }
      // Drain: every copy this thread started has landed before the CTA can exit.
      volatile int never = 0;
      if (armed_q >= 0) tc::mbar_wait(&sm.q_full, armed_q, &never, lim);
      if (armed_k >= 0) tc::mbar_wait(&sm.k_full, armed_k, &never, lim);
      if (armed_v >= 0) tc::mbar_wait(&sm.v_full, armed_v, &never, lim);
      for (int b = 0; b < 2; ++b)
        if (armed_z[b] >= 0) tc::mbar_wait(&sm.z_full[b], armed_z[b], &never, lim);
      for (int c = 0; c < kStages; ++c)
        if (armed_s[c] >= 0) tc::mbar_wait(&sm.s_full[c], armed_s[c], &never, lim);
      if (armed_w >= 0) tc::mbar_wait(&sm.w_full, armed_w, &never, lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Per unit k: A+/- += e S group by group, A+ += P V, then the commit: u_k = K W_g over the
    // unit's finished feature-map columns, the next unit's u and s once phi is in shared
    // memory, and dS^T = V^T phi over the accumulator once the epilogue has read it.  MMAs of
    // one thread execute in issue order, so each overwrites TMEM only after the MMAs issued
    // before it have read it.
    if (lane == 0) {
      int g_res = -1, q = 0;
      uint32_t w_seen = 0;
      bool ok = true, issued = false;
      int ucur = blockIdx.x;
      Unit x{}, xn{};
      const uint32_t wa = tc::smem_u32(sm.w);
      const uint32_t qa = tc::smem_u32(sm.q);
      const uint32_t ka = tc::smem_u32(sm.k);
      const uint32_t phia = tc::smem_u32(sm.s[kCommitStage][0]);    // phi of the block
      // s = Q K^T, then u = Q W_g of unit j
      auto issue_uqk = [&](const Unit& y, int j) -> bool {
        if (y.g != g_res) {
          if (!tc::mbar_wait(&sm.w_full, w_seen & 1, abort_flag, lim)) return false;
          ++w_seen;
          g_res = y.g;
        }
        if (!tc::mbar_wait(&sm.q_full, j & 1, abort_flag, lim)) return false;
        if (!tc::mbar_wait(&sm.k_full, j & 1, abort_flag, lim)) return false;
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t a = tc::smem_desc(qa + (kk >> 2) * (kQBytes / 2) + (kk & 3) * 32, 16, 1024, tc::kSwizzle128B);
          const uint64_t b = tc::smem_desc(ka + (kk >> 2) * (kKBytes / 2) + (kk & 3) * 32, 16, 1024, tc::kSwizzle128B);
          tc::mma_bf16_ss(tbase + kColS, a, b, kIdQK, kk > 0);
        }
        tc::mma_commit(&sm.s_ready);  // the feature map starts on the scores
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t a = tc::smem_desc(qa + (kk >> 2) * (kQBytes / 2) + (kk & 3) * 32, 16, 1024, tc::kSwizzle128B);
          const uint64_t b = tc::smem_desc(wa + kk * 2048, kWBytes / 2, 1024, tc::kSwizzle128B);
          tc::mma_bf16_ss(tbase + kColU, a, b, kIdQW, kk > 0);
        }
        tc::mma_commit(&sm.u_full);
        tc::mma_commit(&sm.qk_empty);
        issued = true;
        return true;
      };
      bool have = next_unit(p, units, &ucur, false, &x);
      if (have) ok = issue_uqk(x, 0);
      for (int k = 0; ok && have; ++k) {
        // the accumulators are free once the previous unit's dS^T has been drained
        if (k >= 1 && !tc::mbar_wait(&sm.ds_empty, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
        // A+ += e+ S+ and A- += e- S-, group by group as the feature-map warps release them
        for (int i = 0; i < kGroups; ++i, ++q) {
          const int grp = group_at(i);
          if (!tc::mbar_wait(&sm.e_ready[grp], k & 1, abort_flag, lim)) { ok = false; break; }
          const int st = q % kStages;
          if (!tc::mbar_wait(&sm.s_full[st], (q / kStages) & 1, abort_flag, lim)) { ok = false; break; }
          tc::tc_fence_after();
          // MN-major tf32 B: 128-byte swizzle with 32-byte atoms, 4-row K groups (SBO 512 B),
          // d quarters 4 KiB apart (LBO); K steps of 8 rows are 1 KiB apart, i.e. 64 in the
          // descriptor's 16-byte address units
          const uint64_t bp = tc::smem_desc(tc::smem_u32(sm.s[st][0]), kSBytes / 4, 512, tc::kSwizzle128BBase32B);
          const uint64_t bm = bp + (kSBytes >> 4);
          const uint32_t ep = tbase + kColU + grp * 32, em = tbase + kColEm + grp * 32;
#pragma unroll
          for (int kk = 0; kk < kChunk / 8; ++kk)
            tc::mma_tf32_ts(tbase + kColAp, ep + kk * 8, bp + (uint64_t)(kk * 64), kIdES, (i > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < kChunk / 8; ++kk)
            tc::mma_tf32_ts(tbase + kColAm, em + kk * 8, bm + (uint64_t)(kk * 64), kIdES, (i > 0 || kk > 0) ? 1u : 0u);
          tc::mma_commit(&sm.s_empty[st]);
        }
        if (!ok) break;
        // A+ += P V
        if (!tc::mbar_wait(&sm.p_ready, k & 1, abort_flag, lim)) { ok = false; break; }
        if (!tc::mbar_wait(&sm.v_ready, k & 1, abort_flag, lim)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t pa = tc::smem_u32(sm.p);
        const uint32_t va = tc::smem_u32(sm.v);
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk) {
          const uint64_t a = tc::smem_desc(pa + kk * 32, 16, 512, tc::kSwizzle64B);
          const uint64_t b = tc::smem_desc(va + kk * 2048, kKBytes / 2, 1024, tc::kSwizzle128B);
          tc::mma_bf16_ss(tbase + kColAp, a, b, kIdPV, 1);
        }
        tc::mma_commit(&sm.acc_full);
        // commit: u_k = K W_g (the block's 32 rows lead the 128-row tile) into u's columns
        // u_k reads K from its own buffer, still holding this unit's K: an M = 128 tile whose
        // rows 32 .. 127 run on into the V and P buffers (in bounds, and not written until
        // this unit's dS^T and the next unit's P); those rows of u_k are never read
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t a = tc::smem_desc(ka + (kk >> 2) * (kKBytes / 2) + (kk & 3) * 32, 16, 1024, tc::kSwizzle128B);
          const uint64_t b = tc::smem_desc(wa + kk * 2048, kWBytes / 2, 1024, tc::kSwizzle128B);
          tc::mma_bf16_ss(tbase + kColU, a, b, kIdQW, kk > 0);
        }
        tc::mma_commit(&sm.uk_done);
        // dS^T = V^T phi over the accumulator columns, once phi is in shared memory and the
        // epilogue has read the output (first, so that its drain, which the next unit's
        // contraction waits for, starts as early as possible)
        if (!tc::mbar_wait(&sm.phi_ready, k & 1, abort_flag, lim)) { ok = false; break; }
        if (!tc::mbar_wait(&sm.acc_empty, k & 1, abort_flag, lim)) { ok = false; break; }
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk) {
          // A = V^T (M = d, K = tokens), MN-major: d halves 4 KiB apart, 8-token groups 1 KiB;
          // B = phi (K = tokens, N = F), MN-major: F quarters 4 KiB apart
          const uint64_t a = tc::smem_desc(va + kk * 2048, kKBytes / 2, 1024, tc::kSwizzle128B);
          const uint64_t b = tc::smem_desc(phia + kk * 2048, kPhiBytes / 4, 1024, tc::kSwizzle128B);
          tc::mma_bf16_ss(tbase + kColAm, a, b, kIdVP, kk > 0);
        }
        tc::mma_commit(&sm.ds_full);
        tc::mma_commit(&sm.v_empty);
        // then the next unit's u and s (u_k, in u's columns, was staged before phi was ready)
        const bool have_next = next_unit(p, units, &ucur, false, &xn);
        if (have_next && !issue_uqk(xn, k + 1)) { ok = false; break; }
        x = xn;
        have = have_next;
      }
      if (issued) {
        volatile int never = 0;
        tc::mma_commit(&sm.drain);
        tc::mbar_wait(&sm.drain, 0, &never, lim);
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ feature map
    // One warp per TMEM lane quarter, one thread per tile row (its own TMEM lane).  A failed
    // bounded wait ends the loop for the whole warp (the vote keeps its lanes together).
    const int wq = warp & 3;           // TMEM lane quarter this warp may access
    const int row = wq * 32 + lane;    // tile row = G t + head-in-group
    const int hl = row % p.G;
    const uint32_t tl = tbase + ((uint32_t)(wq * 32) << 16);
    const float scale_log2 = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(128)
    const float log2e = 1.4426950408889634f;
    int ucur = blockIdx.x;
    Unit x{};
    for (int k = 0; next_unit(p, units, &ucur, false, &x); ++k) {
      // the block scores first (u is still being computed behind them)
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.s_ready, k & 1, abort_flag, lim))) break;
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.z_full[k & 1], (k >> 1) & 1, abort_flag, lim))) break;
      tc::tc_fence_after();

      // block softmax over the x.n keys of this request (bidirectional, no mask): only the
      // row max m of s_j = q.k_j log2(e) / sqrt d here; P itself is formed once its scale is
      // known (below, from the scores still in TMEM)
      float m2;
      {
        float sv[32];
        tc::tmem_ld32(tl + kColS, sv);
        tc::tmem_wait_ld();
        float mraw = -INFINITY;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < x.n) mraw = fmaxf(mraw, sv[j]);
        m2 = mraw * scale_log2;
      }
      const float wgt = p.alpha && row < kBlk * p.G ? 1.f / (1.f + expf(-p.alpha[p.G * x.g + hl])) : 1.f;
      // Scale of the linear branch (log2 units).  Both branches meet in A+ with P stored as
      // w 2^{s_j} sum e+, so e+ and e- are shifted down by tl = max(0, m - 100): then every
      // stored P is below 2^{107} and no e exceeds 1, and when m > 100 the linear branch,
      // which tl makes smaller still, is in any case below 2^{-90} of the softmax branch (if
      // the shift flushes every e+ and e- to 0, P is formed as if sum e+ were 2^{-tl}).
      // States that are all zero (no committed block) add nothing: e+ = e- = 0 and P is
      // shifted by m instead, so a block whose scores are all very negative stays exact.
      float zmax;
      {
        const float* zk0 = sm.z[k & 1];
        const float4 a = *reinterpret_cast<const float4*>(zk0 + lane * 8);
        const float4 b = *reinterpret_cast<const float4*>(zk0 + lane * 8 + 4);
        zmax = warp_max(fmaxf(fmaxf(fmaxf(a.x, a.y), fmaxf(a.z, a.w)), fmaxf(fmaxf(b.x, b.y), fmaxf(b.z, b.w))));
      }
      const bool lin = zmax > 0.f;
      const float tl2 = lin ? fmaxf(0.f, m2 - 100.f) : INFINITY;

      // max and min of u over the row's 128 features
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.u_full, k & 1, abort_flag, lim))) break;
      tc::tc_fence_after();
      float mx = -INFINITY, mn = INFINITY;
#pragma unroll 1
      for (int c = 0; c < kGroups; c += 2) {
        float u0[32], u1[32];
        tc::tmem_ld32(tl + kColU + c * 32, u0);
        tc::tmem_ld32(tl + kColU + c * 32 + 32, u1);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          mx = fmaxf(mx, fmaxf(u0[i], u1[i]));
          mn = fminf(mn, fminf(u0[i], u1[i]));
        }
      }

      // e+_f = 2^{(u_f - max u) log2e - tl} over u in place, e-_f = 2^{(min u - u_f) log2e - tl},
      // group by group, each released to the MMA as soon as the four warps have written it
      // (e- group 3 overwrites the scores, which this thread has read)
      const float bpl = mx * log2e + tl2, bml = mn * log2e - tl2;
      const float* zk = sm.z[k & 1];
      float esp = 0.f, esm = 0.f, zsp = 0.f, zsm = 0.f, psum = 0.f;
      bool vgood = true;
#pragma unroll 1
      for (int c = 0; c < kGroups; ++c) {
        float uu[32];
        tc::tmem_ld32(tl + kColU + c * 32, uu);
        tc::tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float ep[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a = uu[16 * h + i] * log2e;
            const float e1 = tc::ex2(a - bpl);
            const float e2 = tc::ex2(bml - a);
            esp += e1;
            esm += e2;
            zsp = fmaf(e1, zk[c * 32 + 16 * h + i], zsp);
            zsm = fmaf(e2, zk[kFh + c * 32 + 16 * h + i], zsm);
            ep[i] = e1;
            uu[16 * h + i] = e2;
          }
          tc::tmem_st16(tl + kColU + c * 32 + 16 * h, ep);
        }
        if (c == kGroups - 1) {
          // sum e+ is complete, so P (bf16, w 2^{s_j} sum e+, or w 2^{s_j - m} for empty
          // states) is formed now, from the scores that e- group 3 is about to overwrite.  P's
          // buffer is free once V has landed (V is reloaded only after the previous P V has
          // completed).
          vgood = __all_sync(0xffffffffu, tc::mbar_wait(&sm.v_full, k & 1, abort_flag, lim));
          const float lsp = lin ? (esp > 0.f ? tc::lg2(esp) : -tl2) : -m2;
          float sv[32];
          tc::tmem_ld32(tl + kColS, sv);
          tc::tmem_wait_ld();
          uint32_t packed[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float a0 = j < x.n ? wgt * tc::ex2(fmaf(sv[j], scale_log2, lsp)) : 0.f;
            const float a1 = j + 1 < x.n ? wgt * tc::ex2(fmaf(sv[j + 1], scale_log2, lsp)) : 0.f;
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(a0, a1);
            psum += __low2float(b2) + __high2float(b2);
            packed[j >> 1] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          // 64-byte rows, 16-byte chunk c stored at chunk c ^ ((row / 2) % 4) (64-byte swizzle)
          uint8_t* prow = sm.p + row * 64;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            *reinterpret_cast<uint4*>(prow + ((q4 ^ ((row >> 1) & 3)) << 4)) =
                make_uint4(packed[4 * q4], packed[4 * q4 + 1], packed[4 * q4 + 2], packed[4 * q4 + 3]);
        }
        tc::tmem_st32(tl + kColEm + c * 32, uu);
        tc::tmem_wait_st();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sm.e_ready[c]);
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sm.z_empty[k & 1]);
      if (!vgood) break;

      // V of this unit: rows past a short block belong to another request; clear them
      if (x.n < kBlk) {
        const int per_half = (kBlk - x.n) * 8;
        for (int i = wq * 32 + lane; i < 2 * per_half; i += 128) {
          const int hh = i / per_half, rem = i % per_half;
          *reinterpret_cast<uint4*>(sm.v + hh * (kKBytes / 2) + (x.n + rem / 8) * 128 + (rem % 8) * 16) =
              make_uint4(0, 0, 0, 0);
        }
      }
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(&sm.v_ready);
        tc::mbar_arrive(&sm.p_ready);
      }

      // epilogue factors: out = f+ A+ + f- A- with, after multiplying numerator and
      // denominator by sum e+,  den = sum_j P_j + e+.Z+ + (sum e+ / sum e-) e-.Z-,  f+ = 1/den,
      // f- = (sum e+ / sum e-) / den (every term bounded), using the same rounded P that the
      // P V product uses; handed to the epilogue warps through a double buffer
      const int fb = k & 1;
      if (k >= 2 && !__all_sync(0xffffffffu, tc::mbar_wait(&sm.fin_empty[fb], ((k - 2) >> 1) & 1, abort_flag, lim)))
        break;
      const float rpm = lin && esm > 0.f ? esp / esm : 0.f;
      const float den = psum + (lin ? zsp + zsm * rpm : 0.f);
      const float inv = den != 0.f ? 1.f / den : 0.f;
      sm.fin[fb][0][row] = inv;
      sm.fin[fb][1][row] = rpm * inv;
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sm.fin_full[fb]);

      // ---- the commit of this unit: u_k = K W_g, whose 32 block rows sit in TMEM lanes 0-31
      // (lane quarter 0), is staged by that quarter's warp in the lent stage's second half as
      // U [32 rows][128] fp32; then the eight feature-map and epilogue warps form phi and dZ
      if (wq == 0) {
        if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.uk_done, k & 1, abort_flag, lim))) break;
        tc::tc_fence_after();
        float* U = reinterpret_cast<float*>(sm.s[kCommitStage][1]);
#pragma unroll 1
        for (int c = 0; c < kGroups; ++c) {
          float uu[32];
          tc::tmem_ld32(tl + kColU + c * 32, uu);
          tc::tmem_wait_ld();
          // float4 slot j of row `lane` at slot j ^ (lane % 8): the eight lanes of each
          // quarter-warp store into eight different bank groups
          float4* dst = reinterpret_cast<float4*>(U + lane * kFh);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[(c * 8 + i) ^ (lane & 7)] = make_float4(uu[4 * i], uu[4 * i + 1], uu[4 * i + 2], uu[4 * i + 3]);
        }
        // u_k has been read from TMEM (the next unit's u may overwrite it once phi is ready)
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sm.u_staged);
      }
      if (!commit_phi(x, k, wq * 32 + lane)) break;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // One warp per TMEM lane quarter: out = f+ A+ + f- A- for its 32 rows, written straight
    // from registers (each thread its row's 64-byte chunks) while the feature-map warps
    // already work on the next unit.
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int tok = row / p.G, hl = row % p.G;  // rows past 32 G have tok >= 32: never stored
    const uint32_t tl = tbase + ((uint32_t)(wq * 32) << 16);
    int ucur = blockIdx.x;
    Unit x{};
    for (int k = 0; next_unit(p, units, &ucur, false, &x); ++k) {
      const int fb = k & 1;
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.acc_full, k & 1, abort_flag, lim))) break;
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.fin_full[fb], (k >> 1) & 1, abort_flag, lim))) break;
      tc::tc_fence_after();
      const float fp = sm.fin[fb][0][row], fm = sm.fin[fb][1][row];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sm.fin_empty[fb]);
      __nv_bfloat16* orow = p.O + ((size_t)(x.lo + tok) * p.Hq + p.G * x.g + hl) * kD;
      const bool live = tok < x.n, o32 = p.o32 != 0;
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        float a32[32], b32[32];
        tc::tmem_ld32(tl + kColAp + c * 32, a32);
        tc::tmem_ld32(tl + kColAm + c * 32, b32);
        tc::tmem_wait_ld();
        if (c == kD / 32 - 1) {
          // every read of the accumulators is done: the next unit's MMAs may overwrite them
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&sm.acc_empty);
        }
        if (live && o32) {
          // 32-byte stores, each one whole L2 sector of the row (16-byte pieces would leave
          // every sector half-written by one instruction and cost the L2 a merge), not
          // allocated in L1
#pragma unroll
          for (int q8 = 0; q8 < 2; ++q8) {
            uint32_t w[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
              w[j] = pack_bf16(fmaf(fp, a32[16 * q8 + 2 * j], fm * b32[16 * q8 + 2 * j]),
                               fmaf(fp, a32[16 * q8 + 2 * j + 1], fm * b32[16 * q8 + 2 * j + 1]));
            tc::st_global_32B(orow + c * 32 + q8 * 16, w);
          }
        } else if (live) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            float o[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) o[j] = fmaf(fp, a32[8 * q4 + j], fm * b32[8 * q4 + j]);
            tc::st_global_16B(orow + c * 32 + q4 * 8, pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]),
                              pack_bf16(o[4], o[5]), pack_bf16(o[6], o[7]));
          }
        }
      }

      // ---- phi and dZ of this unit's block, with the feature-map warps
      if (!commit_phi(x, k, (warp - 2) * 32 + lane)) break;
      // ---- the commit of this unit: S[f][d] += dS^T[d][f] by reducing atomic adds straight
      // from the accumulator (lane = d, so each warp instruction adds one 128-byte row piece)
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.ds_full, k & 1, abort_flag, lim))) break;
      tc::tc_fence_after();
      {
        float* Srow = pc.Sw + ((size_t)(x.slot * p.Hkv + x.g) * kF) * kD + wq * 32 + lane;
#pragma unroll 1
        for (int c = 0; c < kF / 32; ++c) {
          float dv[32];
          tc::tmem_ld32(tl + kColAm + c * 32, dv);
          tc::tmem_wait_ld();
          if (c == kF / 32 - 1) {
            // dS^T has been read: the next unit's MMAs may overwrite the accumulator columns
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.ds_empty);
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) atomicAdd(Srow + (size_t)(c * 32 + i) * kD, dv[i]);
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

}  // namespace

// ----------------------------------------------------------------- host side
cudaError_t launch_hybrid_commit_tc(const HybridArgs& a, float* S, float* Z, cudaStream_t st) {
  TcHybridCommitParams pc;
  TcHybridParams& p = pc.h;
  const uint64_t T = (uint64_t)a.T;
  {
    const uint64_t dims[3] = {kD, (uint64_t)a.Hq, T};
    const uint64_t strides[2] = {kD * 2, (uint64_t)a.Hq * kD * 2};
    const uint32_t box[3] = {64, (uint32_t)(a.Hq / a.Hkv), kBlk};
    if (!make_tensor_map(&p.tm_q, false, 3, a.Q, dims, strides, box, kTma128B)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {kD, (uint64_t)a.Hkv, T};
    const uint64_t strides[2] = {kD * 2, (uint64_t)a.Hkv * kD * 2};
    const uint32_t box[3] = {64, 1, kBlk};
    if (!make_tensor_map(&p.tm_k, false, 3, a.K, dims, strides, box, kTma128B)) return cudaErrorInvalidValue;
    if (!make_tensor_map(&p.tm_v, false, 3, a.V, dims, strides, box, kTma128B)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {kFh, (uint64_t)a.Hkv * kD};
    const uint64_t strides[1] = {kFh * 2};
    const uint32_t box[2] = {64, kD};
    if (!make_tensor_map(&p.tm_w, false, 2, a.W, dims, strides, box, kTma128B)) return cudaErrorInvalidValue;
  }
  {
    // 32 x 32 fp32 boxes, 128-byte swizzle with 32-byte atoms (tf32 MN-major operand layout)
    const uint64_t dims[2] = {kD, (uint64_t)a.num_slots * a.Hkv * kF};
    const uint64_t strides[1] = {kD * 4};
    const uint32_t box[2] = {32, kChunk};
    if (!make_tensor_map(&p.tm_s, true, 2, a.S, dims, strides, box, kTma128BAtom32)) return cudaErrorInvalidValue;
  }
  pc.Sw = S;
  pc.Zw = Z;
  p.cu_blk = a.cu_blk;
  p.state_slot = a.state_slot;
  p.Z = a.Z;
  p.alpha = a.alpha;
  p.O = static_cast<__nv_bfloat16*>(a.O);
  p.o32 = (reinterpret_cast<uintptr_t>(a.O) & 31) == 0;
  p.dev_err = a.dev_err;
  p.R = a.R;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.T = a.T;
  p.Bmax = a.Bmax;
  p.num_slots = a.num_slots;
  p.wait_limit = 2000000000ll;  // about one second of SM cycles

  const int units = a.R * a.Hkv;
  int nsm = device_sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  // Fewest CTAs that still finish in the least number of rounds, a multiple of Hkv when that
  // costs no round (each CTA then stays on one KV head).
  const int grid = persistent_grid(units, a.Hkv, nsm);
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(hybrid_commit_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  hybrid_commit_tc_kernel<<<grid, kThreads, smem, st>>>(pc);
  return cudaGetLastError();
}

}  // namespace bha
