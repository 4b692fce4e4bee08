// Tensor-core block-hybrid decode step for sm_100a (bf16 activations, d = 128, F = 256,
// G = 1, 2 or 4 query heads per KV head, blocks of up to 32 tokens).
//
// Source: "Retrofitting Linear Attention into Diffusion Language Models", §3.1: per query q
//   sm_num = sum_j exp(q.k_j/sqrt d) v_j,  sm_den = sum_j exp(q.k_j/sqrt d)   (active block)
//   lin_num = phi(q)^T S,  lin_den = phi(q)^T Z,  phi(q) = [softmax(qW), softmax(-qW)]
//   out = (w sm_num + lin_num) / (w sm_den + lin_den),  w = sigmoid(alpha_h)
//
// Work unit: one (request r, KV head g).  Its G query heads x 32 block rows fill 32 G rows of
// one 128-row MMA tile (row = G t + head-in-group, the order Q has in memory; for G < 4 the
// other rows hold whatever follows in shared memory and are never stored; with G = 1 this
// is the per-query-head layout, W and the states per query head), and they share
// K_g, V_g, W_g, S_g and Z_g, so S_g (128 KiB fp32, the dominant traffic) is read once per
// unit.  A persistent grid walks the units; unit u is (r = u / Hkv, g = u % Hkv), so a CTA
// whose grid stride is a multiple of Hkv keeps one W_g resident.
//
// The state is contracted while the feature map is still being computed.  With u = qW,
//   e+_f = 2^{(u_f - max u) log2 e},  e-_f = 2^{(min u - u_f) log2 e}   (unnormalised, <= 1)
//   A+ = sum_{f<F/2} e+_f S_f,  A- = sum_{f>=F/2} e-_f S_f
//   lin_num = e^{-m} (A+ / sum e+  +  A- / sum e-)
// so each group of 32 e values goes to the tensor cores as soon as it exists (fp32 in TMEM,
// contracted in tf32 against the fp32 S tile exactly as TMA delivered it), and the
// normalisation by sum e+/-, known only at the end, moves to the epilogue.  A+ and A-
// accumulate in two TMEM accumulators; P V joins A+ with P stored as w 2^{s_j} sum e+
// (s_j the scaled score in log2 units), which the epilogue's factor 1 / sum e+ undoes:
//   out = (A+ + r A-) / den,  r = sum e+ / sum e-,  den = sum_j P_j + e+.Z+ + r e-.Z-.
// For large scores both e+ and e- are shifted down by tl = max(0, max_j s_j - 100) (a common
// factor of the linear branch), so P stays below 2^107; for states that are all zero the
// linear branch is dropped and P is shifted by max_j s_j instead.
// TMEM columns: u [0,128), overwritten in place by e+; e- [128,256) (the block scores sit in
// its top 32 columns until e- overwrites them); A- [256,384); A+ [384,512).
//
// Roles (320 threads):
//   warp 0      TMA producer: Q/K and Z of unit k, then S of unit k as four stages of two
//               32-row fp32 chunks (rows 32g.. of S+ and of S-; 128-byte swizzle with 32-byte
//               atoms, the layout a tf32 MN-major operand needs) through a 4-stage ring that
//               holds one whole unit, with V issued ahead of the last stage.
//   warp 1      TMEM owner and MMA issuer (one thread), per unit k: A+ += e+ S+ and
//               A- += e- S- group by group (tf32, e from TMEM), then s = Q K^T and u = Q W_g of
//               unit k+1 (bf16, each announced on its own barrier, so that the feature map
//               takes the row max of the scores while u is computed), then A+ += P V of unit k
//               (bf16).  MMAs of one thread execute in issue order, so unit k+1's s and u
//               overwrite the top of e- and e+ only after unit k's e S has read them, and unit
//               k+1's feature map can start while unit k's P V is still waiting for its P.
//   warps 2-5   feature map, one warp per TMEM lane quarter and one thread per tile row (its
//               own TMEM lane): block-softmax max, e+ / e- group by group (each group released
//               to the MMA as soon as the four warps have written it), P from the block scores
//               (saved to registers before e- group 3 overwrites them) once the last group
//               has gone to the MMA, and the epilogue factors for the row.
//   warps 6-9   epilogue, one warp per lane quarter: out = f+ A+ + f- A- once the unit's MMAs
//               are done, each thread storing its row straight from registers as whole
//               32-byte sectors, not allocated in L1 (16-byte pieces when O is only 16-byte
//               aligned), while the feature-map warps already work on the next unit.
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
  uint64_t qk_full, qk_empty, v_full, v_empty, v_ready, z_full[2], z_empty[2];
  uint64_t s_full[kStages], s_empty[kStages];
  uint64_t e_ready[kGroups], p_ready;
  uint64_t w_full, u_full, s_ready, acc_full, acc_empty, drain, fin_full[2], fin_empty[2];
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

__global__ void __launch_bounds__(kThreads, 1) hybrid_tc_kernel(const __grid_constant__ TcHybridParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;
  const long long lim = p.wait_limit;
  const int units = p.R * p.Hkv;

  if (threadIdx.x == 0) {
    tc::mbar_init(&sm.qk_full, 1);
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int g_res = -1, q = 0;
      uint32_t w_loads = 0;
      int armed_qk = -1, armed_v = -1, armed_w = -1, armed_z[2] = {-1, -1};
      int armed_s[kStages];
#pragma unroll
      for (int i = 0; i < kStages; ++i) armed_s[i] = -1;
      bool ok = true;
      int ucur = blockIdx.x;
      Unit x{};
      for (int k = 0; ok && next_unit(p, units, &ucur, true, &x); ++k) {
        if (x.g != g_res) {
          // W is read only by each unit's first MMA: the previous unit's must be done
          if (k >= 1 && !tc::mbar_wait(&sm.u_full, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
          tc::mbar_arrive_expect_tx(&sm.w_full, kWBytes);
          tc::tma_load_2d(sm.w, &p.tm_w, &sm.w_full, 0, x.g * kD);
          tc::tma_load_2d(sm.w + kWBytes / 2, &p.tm_w, &sm.w_full, 64, x.g * kD);
          armed_w = w_loads & 1;
          ++w_loads;
          g_res = x.g;
        }
        if (k >= 1 && !tc::mbar_wait(&sm.qk_empty, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
        // Q: two d halves of 32 G rows, each at the start of its 16 KiB half of the tile
        tc::mbar_arrive_expect_tx(&sm.qk_full, (kQBytes / kG) * p.G + kKBytes);
        tc::tma_load_3d(sm.q, &p.tm_q, &sm.qk_full, 0, p.G * x.g, x.lo);
        tc::tma_load_3d(sm.q + kQBytes / 2, &p.tm_q, &sm.qk_full, 64, p.G * x.g, x.lo);
        tc::tma_load_3d(sm.k, &p.tm_k, &sm.qk_full, 0, x.g, x.lo);
        tc::tma_load_3d(sm.k + kKBytes / 2, &p.tm_k, &sm.qk_full, 64, x.g, x.lo);
        armed_qk = k & 1;
        const int zb = k & 1, zj = k >> 1;
        if (zj >= 1 && !tc::mbar_wait(&sm.z_empty[zb], (zj - 1) & 1, abort_flag, lim)) { ok = false; break; }
        tc::mbar_arrive_expect_tx(&sm.z_full[zb], kZBytes);
        tc::bulk_load(sm.z[zb], p.Z + ((size_t)x.slot * p.Hkv + x.g) * kF, kZBytes, &sm.z_full[zb]);
        armed_z[zb] = zj & 1;
        const int srow0 = (x.slot * p.Hkv + x.g) * kF;
        for (int i = 0; i < kGroups; ++i, ++q) {
          const int grp = group_at(i);
          if (i == kStages - 1) {
            // V (read by the unit's P V) goes ahead of the last S pair, which waits for the
            // previous unit's last pair to be consumed, so that it lands before it is needed
            if (k >= 1 && !tc::mbar_wait(&sm.v_empty, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
            tc::mbar_arrive_expect_tx(&sm.v_full, kKBytes);
            tc::tma_load_3d(sm.v, &p.tm_v, &sm.v_full, 0, x.g, x.lo);
            tc::tma_load_3d(sm.v + kKBytes / 2, &p.tm_v, &sm.v_full, 64, x.g, x.lo);
            armed_v = k & 1;
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
      if (armed_qk >= 0) tc::mbar_wait(&sm.qk_full, armed_qk, &never, lim);
      if (armed_v >= 0) tc::mbar_wait(&sm.v_full, armed_v, &never, lim);
      for (int b = 0; b < 2; ++b)
        if (armed_z[b] >= 0) tc::mbar_wait(&sm.z_full[b], armed_z[b], &never, lim);
      for (int c = 0; c < kStages; ++c)
        if (armed_s[c] >= 0) tc::mbar_wait(&sm.s_full[c], armed_s[c], &never, lim);
      if (armed_w >= 0) tc::mbar_wait(&sm.w_full, armed_w, &never, lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Per unit k: A+/- += e S group by group, then the next unit's s and u, then A+ += P V.
    // Issuing s(k+1) and u(k+1) ahead of P V(k) lets the feature map of unit k+1 start as soon
    // as the tensor pipe has finished e S(k), not after P V(k), which waits for unit k's P.
    // MMAs of one thread execute in issue order, so s(k+1) and u(k+1) overwrite the top of e-
    // and e+ only after e S(k) has read them.
    if (lane == 0) {
      int g_res = -1, q = 0;
      uint32_t w_seen = 0;
      bool ok = true, issued = false;
      int ucur = blockIdx.x;
      Unit x{}, xn{};
      const uint32_t wa = tc::smem_u32(sm.w);
      const uint32_t qa = tc::smem_u32(sm.q);
      const uint32_t ka = tc::smem_u32(sm.k);
      // s = Q K^T, then u = Q W_g of unit j
      auto issue_uqk = [&](const Unit& y, int j) -> bool {
        if (y.g != g_res) {
          if (!tc::mbar_wait(&sm.w_full, w_seen & 1, abort_flag, lim)) return false;
          ++w_seen;
          g_res = y.g;
        }
        if (!tc::mbar_wait(&sm.qk_full, j & 1, abort_flag, lim)) return false;
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
        // the accumulators are free once the previous epilogue has read them
        if (k >= 1 && !tc::mbar_wait(&sm.acc_empty, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
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
        // the next unit's u and s
        const bool have_next = next_unit(p, units, &ucur, false, &xn);
        if (have_next && !issue_uqk(xn, k + 1)) { ok = false; break; }
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
        tc::mma_commit(&sm.v_empty);
        tc::mma_commit(&sm.acc_full);
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
      float sv[32];
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
        // the block scores leave TMEM before e- group 3 overwrites them
        if (c == kGroups - 1) {
          tc::tmem_ld32(tl + kColS, sv);
          tc::tmem_wait_ld();
        }
        tc::tmem_st32(tl + kColEm + c * 32, uu);
        tc::tmem_wait_st();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sm.e_ready[c]);
      }
      {
        // sum e+ is complete, so P (bf16, w 2^{s_j} sum e+, or w 2^{s_j - m} for empty
        // states) is formed now, from the scores saved above, after the last group has gone
        // to the MMA.  P's buffer is free once V has landed (V is reloaded only after the
        // previous P V has completed).
        vgood = __all_sync(0xffffffffu, tc::mbar_wait(&sm.v_full, k & 1, abort_flag, lim));
        const float lsp = lin ? (esp > 0.f ? tc::lg2(esp) : -tl2) : -m2;
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
bool hybrid_tc_supports(const HybridArgs& a, bool act_bf16) {
  const int G = a.Hkv > 0 && a.Hq % a.Hkv == 0 ? a.Hq / a.Hkv : 0;
  return act_bf16 && a.d == kD && a.F == kF && (G == 1 || G == 2 || G == kG) && a.Bmax <= kBlk &&
         (long long)a.num_slots * a.Hkv * kF < (1ll << 31);
}

cudaError_t launch_hybrid_tc(const HybridArgs& a, cudaStream_t st) {
  TcHybridParams p;
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
  // Fewest CTAs that still finish in the least number of rounds (every CTA then takes the
  // same number of units and a larger share of the memory bandwidth), a multiple of Hkv when
  // that costs no round, so that each CTA stays on one KV head.
  const int grid = persistent_grid(units, a.Hkv, nsm);
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(hybrid_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  hybrid_tc_kernel<<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace bha
