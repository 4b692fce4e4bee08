// Tensor-core block-hybrid decode step for sm_100a (bf16 activations, d = 128, F = 256,
// four query heads per KV head, blocks of up to 32 tokens).
//
// Source: "Retrofitting Linear Attention into Diffusion Language Models", §3.1: per query q
//   sm_num = sum_j exp(q.k_j/sqrt d) v_j,  sm_den = sum_j exp(q.k_j/sqrt d)   (active block)
//   lin_num = phi(q)^T S,  lin_den = phi(q)^T Z,  phi(q) = [softmax(qW), softmax(-qW)]
//   out = (w sm_num + lin_num) / (w sm_den + lin_den),  w = sigmoid(alpha_h)
//
// Work unit: one (request r, KV head g).  Its 4 query heads x 32 block rows are exactly
// one 128-row MMA tile (row = 4 t + head-in-group, the order Q has in memory), and they
// share K_g, V_g, W_g, S_g and Z_g, so S_g (128 KiB fp32, the dominant traffic) is read
// once per unit.  A persistent grid walks the units; unit u is (r = u / Hkv, g = u % Hkv),
// so a CTA whose grid stride is a multiple of Hkv keeps one W_g resident.
//
// Roles (320 threads):
//   warp 0     TMA producer.  Q/K (single buffer, refilled once the unit's score MMA has
//              read them), V/Z (refilled after the unit's P.V MMA), W_g when g changes, and
//              S_g as eight 32-row fp32 chunks, one ring stage each, so a whole unit's state
//              streams in while the previous unit is still being contracted.
//   warp 1     TMEM owner and MMA issuer (one thread):
//                u   = Q W_g          bf16 x bf16 -> fp32   TMEM cols [256, 384)
//                s   = Q K_g^T        bf16 x bf16 -> fp32   TMEM cols [384, 416)
//                acc = P V_g          bf16 x bf16 -> fp32   TMEM cols [384, 512) (after s is read)
//                acc += phi' S_g      tf32, A = phi' from TMEM cols [0, 256), B = the fp32 S
//                                     tile exactly as TMA delivered it
//   warps 2-9  two threads per tile row (warps 2-5: softmax(u) half, warps 6-9: softmax(-u)
//              half): block softmax (row max m over the block's keys, P = w e^{s/sqrt d - m}
//              in bf16), that thread's half of phi' = e^{-m} [softmax(u), softmax(-u)] into
//              TMEM, its half of the linear denominator e^{-m} phi.Z on CUDA cores, then the
//              epilogue out = acc / (w sum_j P + e^{-m} phi.Z) for 64 of the 128 columns.
// The shift m cancels between numerator and denominator; folding e^{-m} into phi and w
// into P lets both branches share one TMEM accumulator.
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
constexpr int kG = 4;
constexpr int kBlk = 32;
constexpr int kM = kG * kBlk;  // 128 tile rows
constexpr int kStages = 8;  // a whole unit of S in flight
constexpr int kChunk = 32;  // F rows of S per stage
constexpr int kChunks = kF / kChunk;
constexpr int kThreads = 320;  // producer, MMA issuer, 8 softmax / epilogue warps

constexpr uint32_t kQBytes = kM * kD * 2;      // 32 KiB
constexpr uint32_t kKBytes = kBlk * kD * 2;    // 8 KiB
constexpr uint32_t kZBytes = kF * 4;           // 1 KiB
constexpr uint32_t kWBytes = kD * kFh * 2;     // 32 KiB
constexpr uint32_t kSBytes = kChunk * kD * 4;  // 16 KiB
constexpr uint32_t kPBytes = kM * 64;          // 8 KiB (64-byte rows, 64-byte swizzle)

// TMEM columns
constexpr uint32_t kColPhi = 0;    // phi' (256 columns): A operand of the state read
constexpr uint32_t kColS = 224;    // block scores (32 columns), read before phi' overwrites them
constexpr uint32_t kColU = 256;    // u = Q W_g (128 columns)
constexpr uint32_t kColAcc = 384;  // output accumulator (128 columns)
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kIdQW = tc::instr_desc(1, 0, 1, kM, kFh);
constexpr uint32_t kIdQK = tc::instr_desc(1, 0, 0, kM, kBlk);
constexpr uint32_t kIdPV = tc::instr_desc(1, 0, 1, kM, kD);
constexpr uint32_t kIdPS = tc::instr_desc(2, 0, 1, kM, kD);

struct __align__(1024) Smem {
  uint8_t q[kQBytes];         // [d half][128 rows][128 B], 128-byte swizzle
  uint8_t w[kWBytes];         // [f half][128 rows of d][128 B]
  uint8_t s[kStages][kSBytes];// [d quarter][32 rows of f][128 B], 128-byte swizzle, 32-byte atoms
  uint8_t k[kKBytes];         // [d half][32 rows][128 B]
  uint8_t v[kKBytes];
  uint8_t p[kPBytes];         // [128 rows][64 B], 64-byte swizzle
  float z[kF];
  float red[2][kM];           // per-row linear-denominator halves
  uint64_t qk_full, qk_empty, vz_full, vz_empty, s_full[kStages], s_empty[kStages];
  uint64_t w_full, u_full, phi_ready, acc_full, acc_empty, drain;
  uint32_t tmem_base;
  int abort_flag;
};

static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory budget of one CTA per SM");

struct Unit {
  int r, g, lo, n, slot;
};

// Decodes unit u and validates it; every role calls this with the same arguments and so
// skips the same units.
__device__ __forceinline__ bool decode_unit(const TcHybridParams& p, int u, bool report,
                                            Unit* x) {
  x->g = u % p.Hkv;
  x->r = u / p.Hkv;
  RowRange rr;
  if (!request_rows(p.cu_blk, x->r, p.T, p.Bmax, p.dev_err, report, &rr)) return false;
  if (rr.n == 0) return false;
  x->lo = rr.lo;
  x->n = rr.n;
  return request_slot(p.state_slot, x->r, p.num_slots, p.dev_err, report, &x->slot);
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
    tc::mbar_init(&sm.vz_full, 1);
    tc::mbar_init(&sm.vz_empty, 1);
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&sm.s_full[i], 1);
      tc::mbar_init(&sm.s_empty[i], 1);
    }
    tc::mbar_init(&sm.w_full, 1);
    tc::mbar_init(&sm.u_full, 1);
    tc::mbar_init(&sm.phi_ready, 8);
    tc::mbar_init(&sm.acc_full, 1);
    tc::mbar_init(&sm.acc_empty, 8);
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
    // Each buffer is refilled as soon as its last reader is done: Q/K after the unit's
    // score MMA, V/Z after its P.V MMA, S stage c after the state-read MMAs of chunk c.
    // With one stage per S chunk, unit k+1's whole state streams in while unit k's MMAs run.
    if (lane == 0) {
      int k = 0, g_res = -1;
      uint32_t w_loads = 0;
      int armed_qk = -1, armed_vz = -1, armed_w = -1;
      int armed_s[kStages];
#pragma unroll
      for (int i = 0; i < kStages; ++i) armed_s[i] = -1;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        Unit x;
        if (!decode_unit(p, u, true, &x)) continue;
        if (x.g != g_res) {
          // W is read only by the first MMA of each unit: wait for the previous unit's
          if (k >= 1 && !tc::mbar_wait(&sm.u_full, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
          tc::mbar_arrive_expect_tx(&sm.w_full, kWBytes);
          tc::tma_load_2d(sm.w, &p.tm_w, &sm.w_full, 0, x.g * kD);
          tc::tma_load_2d(sm.w + kWBytes / 2, &p.tm_w, &sm.w_full, 64, x.g * kD);
          armed_w = w_loads & 1;
          ++w_loads;
          g_res = x.g;
        }
        if (k >= 1 && !tc::mbar_wait(&sm.qk_empty, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
        tc::mbar_arrive_expect_tx(&sm.qk_full, kQBytes + kKBytes);
        tc::tma_load_3d(sm.q, &p.tm_q, &sm.qk_full, 0, kG * x.g, x.lo);
        tc::tma_load_3d(sm.q + kQBytes / 2, &p.tm_q, &sm.qk_full, 64, kG * x.g, x.lo);
        tc::tma_load_3d(sm.k, &p.tm_k, &sm.qk_full, 0, x.g, x.lo);
        tc::tma_load_3d(sm.k + kKBytes / 2, &p.tm_k, &sm.qk_full, 64, x.g, x.lo);
        armed_qk = k & 1;
        if (k >= 1 && !tc::mbar_wait(&sm.vz_empty, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
        tc::mbar_arrive_expect_tx(&sm.vz_full, kKBytes + kZBytes);
        tc::tma_load_3d(sm.v, &p.tm_v, &sm.vz_full, 0, x.g, x.lo);
        tc::tma_load_3d(sm.v + kKBytes / 2, &p.tm_v, &sm.vz_full, 64, x.g, x.lo);
        tc::bulk_load(sm.z, p.Z + ((size_t)x.slot * p.Hkv + x.g) * kF, kZBytes, &sm.vz_full);
        armed_vz = k & 1;
        const int srow0 = (x.slot * p.Hkv + x.g) * kF;
        for (int c = 0; c < kChunks; ++c) {
          if (k >= 1 && !tc::mbar_wait(&sm.s_empty[c], (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
          tc::mbar_arrive_expect_tx(&sm.s_full[c], kSBytes);
#pragma unroll
          for (int dq = 0; dq < 4; ++dq)
            tc::tma_load_2d(sm.s[c] + dq * (kSBytes / 4), &p.tm_s, &sm.s_full[c], dq * 32,
                            srow0 + c * kChunk);
          armed_s[c] = k & 1;
        }
        ++k;
      }
      // Drain: every copy this thread started has landed before the CTA can exit.
      volatile int never = 0;
      if (armed_qk >= 0) tc::mbar_wait(&sm.qk_full, armed_qk, &never, lim);
      if (armed_vz >= 0) tc::mbar_wait(&sm.vz_full, armed_vz, &never, lim);
      for (int c = 0; c < kStages; ++c)
        if (armed_s[c] >= 0) tc::mbar_wait(&sm.s_full[c], armed_s[c], &never, lim);
      if (armed_w >= 0) tc::mbar_wait(&sm.w_full, armed_w, &never, lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int k = 0, g_res = -1;
      uint32_t w_seen = 0;
      bool ok = true;
      bool issued = false;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        Unit x;
        if (!decode_unit(p, u, false, &x)) continue;
        if (x.g != g_res) {
          if (!tc::mbar_wait(&sm.w_full, w_seen & 1, abort_flag, lim)) { ok = false; break; }
          ++w_seen;
          g_res = x.g;
        }
        if (!tc::mbar_wait(&sm.qk_full, k & 1, abort_flag, lim)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t qa = tc::smem_u32(sm.q);
        const uint32_t wa = tc::smem_u32(sm.w);
        const uint32_t ka = tc::smem_u32(sm.k);
        // u = Q W_g: the previous unit's u was consumed before its phi was published
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t a = tc::smem_desc(qa + (kk >> 2) * (kQBytes / 2) + (kk & 3) * 32, 16, 1024, tc::kSwizzle128B);
          const uint64_t b = tc::smem_desc(wa + kk * 2048, kWBytes / 2, 1024, tc::kSwizzle128B);
          tc::mma_bf16_ss(tbase + kColU, a, b, kIdQW, kk > 0);
        }
        // s = Q K^T lands in the top phi' columns: the previous unit's state-read MMAs must be done
        if (k >= 1 && !tc::mbar_wait(&sm.acc_full, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t a = tc::smem_desc(qa + (kk >> 2) * (kQBytes / 2) + (kk & 3) * 32, 16, 1024, tc::kSwizzle128B);
          const uint64_t b = tc::smem_desc(ka + (kk >> 2) * (kKBytes / 2) + (kk & 3) * 32, 16, 1024, tc::kSwizzle128B);
          tc::mma_bf16_ss(tbase + kColS, a, b, kIdQK, kk > 0);
        }
        tc::mma_commit(&sm.u_full);
        tc::mma_commit(&sm.qk_empty);
        issued = true;
        if (!tc::mbar_wait(&sm.phi_ready, k & 1, abort_flag, lim)) { ok = false; break; }
        if (!tc::mbar_wait(&sm.vz_full, k & 1, abort_flag, lim)) { ok = false; break; }
        // P V overwrites the accumulator: the previous epilogue must have read it
        if (k >= 1 && !tc::mbar_wait(&sm.acc_empty, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t pa = tc::smem_u32(sm.p);
        const uint32_t va = tc::smem_u32(sm.v);
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk) {
          const uint64_t a = tc::smem_desc(pa + kk * 32, 16, 512, tc::kSwizzle64B);
          const uint64_t b = tc::smem_desc(va + kk * 2048, kKBytes / 2, 1024, tc::kSwizzle128B);
          tc::mma_bf16_ss(tbase + kColAcc, a, b, kIdPV, kk > 0);
        }
        tc::mma_commit(&sm.vz_empty);
        for (int c = 0; c < kChunks; ++c) {
          const int st = c;
          if (!tc::mbar_wait(&sm.s_full[st], k & 1, abort_flag, lim)) { ok = false; break; }
          tc::tc_fence_after();
          const uint32_t sa = tc::smem_u32(sm.s[st]);
#pragma unroll
          for (int kk = 0; kk < kChunk / 8; ++kk) {
            // MN-major tf32 operands use the 128-byte swizzle with 32-byte atoms: rows of 128 B,
            // 4-row K groups (SBO 512 B), d quarters 4 KiB apart (LBO).
            const uint64_t b = tc::smem_desc(sa + kk * 1024, kSBytes / 4, 512, tc::kSwizzle128BBase32B);
            tc::mma_tf32_ts(tbase + kColAcc, tbase + kColPhi + c * kChunk + kk * 8, b, kIdPS, 1);
          }
          tc::mma_commit(&sm.s_empty[st]);
        }
        if (!ok) break;
        tc::mma_commit(&sm.acc_full);
        ++k;
      }
      if (issued) {
        // all MMAs of this thread complete before TMEM is released
        volatile int never = 0;
        tc::mma_commit(&sm.drain);
        tc::mbar_wait(&sm.drain, 0, &never, lim);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / feature map / epilogue
    // Two threads per tile row: warps 2-5 take the softmax(u) half of phi and output columns
    // [0, 64), warps 6-9 the softmax(-u) half and output columns [64, 128).
    const int sw = warp - 2;                    // 0..7
    const int half = sw >> 2;                   // 0: softmax(u), 1: softmax(-u)
    const float sgn = half ? -1.f : 1.f;
    const int wq = warp & 3;                    // TMEM lane quarter this warp may access
    const int row = wq * 32 + lane;             // tile row = 4 t + head-in-group
    const int t = row >> 2, hl = row & 3;
    const uint32_t tl = tbase + ((uint32_t)(wq * 32) << 16);
    const float scale_log2 = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(128)
    const float log2e = 1.4426950408889634f;
    const int tid = sw * 32 + lane;             // 0..255
    int k = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      Unit x;
      if (!decode_unit(p, u, false, &x)) continue;
      const int h = kG * x.g + hl;
      if (!tc::mbar_wait(&sm.u_full, k & 1, abort_flag, lim)) break;
      if (!tc::mbar_wait(&sm.vz_full, k & 1, abort_flag, lim)) break;
      tc::tc_fence_after();

      // block softmax over the x.n keys of this request (bidirectional, no mask)
      float sv[32];
      tc::tmem_ld32(tl + kColS, sv);
      tc::tmem_wait_ld();
      float mraw = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < x.n) mraw = fmaxf(mraw, sv[j]);
      // m in log2 units of the scaled score, floored so e^{-m} stays finite
      const float m2 = fmaxf(mraw * scale_log2, -40.f * log2e);
      const float wgt = p.alpha ? 1.f / (1.f + expf(-p.alpha[h])) : 1.f;
      float den_sm = 0.f;
      if (half == 0) {
        // P = w e^{s/sqrt d - m} in bf16; the denominator sums the rounded values P V uses
        uint32_t packed[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          float a0 = 0.f, a1 = 0.f;
          if (j < x.n) a0 = wgt * tc::ex2(fmaf(sv[j], scale_log2, -m2));
          if (j + 1 < x.n) a1 = wgt * tc::ex2(fmaf(sv[j + 1], scale_log2, -m2));
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(a0, a1);
          den_sm += __low2float(b2) + __high2float(b2);
          packed[j >> 1] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        // P row: 64 bytes, 16-byte chunk c stored at chunk c ^ ((row / 2) % 4) (64-byte swizzle)
        uint8_t* prow = sm.p + row * 64;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 v4 = make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
          *reinterpret_cast<uint4*>(prow + ((c ^ ((row >> 1) & 3)) << 4)) = v4;
        }
      }
      if (x.n < kBlk) {
        // rows of V past the block belong to another request (or are zero fill): clear them
        const int per_half = (kBlk - x.n) * 8;  // 16-byte chunks per d half
        for (int i = tid; i < 2 * per_half; i += 256) {
          const int hh = i / per_half, rem = i % per_half;
          const int jr = x.n + rem / 8, ch = rem % 8;
          *reinterpret_cast<uint4*>(sm.v + hh * (kKBytes / 2) + jr * 128 + ch * 16) =
              make_uint4(0, 0, 0, 0);
        }
      }
      tc::fence_proxy_async_smem();
      // every thread has read its scores before the softmax(-u) half overwrites their columns
      tc::tc_fence_before();
      tc::named_barrier_sync(1, 256);
      tc::tc_fence_after();

      // this thread's half of the feature map: e = 2^{(sgn u - max sgn u) log2 e}
      float ext = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < kFh / 32; ++c) {
        float uv[32];
        tc::tmem_ld32(tl + kColU + c * 32, uv);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) ext = fmaxf(ext, sgn * uv[i]);
      }
      const float ext2 = ext * log2e;
      const float slog2e = sgn * log2e;
      float esum = 0.f, zsum = 0.f;
      const float* zb = sm.z + half * kFh;
#pragma unroll 1
      for (int c = 0; c < kFh / 32; ++c) {
        float uv[32];
        tc::tmem_ld32(tl + kColU + c * 32, uv);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float e = tc::ex2(fmaf(uv[i], slog2e, -ext2));
          uv[i] = e;
          esum += e;
          zsum = fmaf(e, zb[c * 32 + i], zsum);
        }
        tc::tmem_st32(tl + kColPhi + half * kFh + c * 32, uv);
      }
      tc::tmem_wait_st();
      const float em = tc::ex2(-m2);
      const float a = em / esum;
#pragma unroll 1
      for (int c = 0; c < kFh / 32; ++c) {
        float ev[32];
        tc::tmem_ld32(tl + kColPhi + half * kFh + c * 32, ev);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) ev[i] *= a;
        tc::tmem_st32(tl + kColPhi + half * kFh + c * 32, ev);
      }
      tc::tmem_wait_st();
      // shared denominator w sum_j P + e^{-m} (zsum_+/esum_+ + zsum_-/esum_-)
      sm.red[half][row] = half == 0 ? den_sm + em * (zsum / esum) : em * (zsum / esum);
      tc::named_barrier_sync(1, 256);
      const float den = sm.red[0][row] + sm.red[1][row];
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sm.phi_ready);

      // epilogue: this thread's 64 output columns
      if (!tc::mbar_wait(&sm.acc_full, k & 1, abort_flag, lim)) break;
      tc::tc_fence_after();
      const float inv = den != 0.f ? 1.f / den : 0.f;
      float ov[64];
      {
        float a32[32], b32[32];
        tc::tmem_ld32(tl + kColAcc + half * 64, a32);
        tc::tmem_ld32(tl + kColAcc + half * 64 + 32, b32);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          ov[i] = a32[i] * inv;
          ov[32 + i] = b32[i] * inv;
        }
      }
      // Coalesced store through this warp's 1 KiB of the (now idle) P buffer: 8 rows at a time
      // are staged (16-byte chunk c of staged row r at chunk c ^ r), then each store
      // instruction writes 4 rows x 128 contiguous bytes.
      uint8_t* stg = sm.p + sw * 1024;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if ((lane >> 3) == j) {
          const int rr = lane & 7;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 o4 = make_uint4(pack_bf16(ov[8 * c], ov[8 * c + 1]), pack_bf16(ov[8 * c + 2], ov[8 * c + 3]),
                                        pack_bf16(ov[8 * c + 4], ov[8 * c + 5]), pack_bf16(ov[8 * c + 6], ov[8 * c + 7]));
            *reinterpret_cast<uint4*>(stg + rr * 128 + ((c ^ rr) << 4)) = o4;
          }
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int rr = 4 * i + (lane >> 3), c = lane & 7;
          const uint4 o4 = *reinterpret_cast<const uint4*>(stg + rr * 128 + ((c ^ rr) << 4));
          const int grow = wq * 32 + 8 * j + rr;       // tile row
          const int gt = grow >> 2, ghl = grow & 3;
          if (gt < x.n)
            *reinterpret_cast<uint4*>(p.O + ((size_t)(x.lo + gt) * p.Hq + kG * x.g + ghl) * kD + half * 64 + c * 8) = o4;
        }
        __syncwarp();
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sm.acc_empty);
      ++k;
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
                     const uint64_t* strides_bytes, const uint32_t* box, bool swizzle_atom32) {
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
  const CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        rank, const_cast<void*>(base), gd, gs, bx, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle_atom32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

bool hybrid_tc_supports(const HybridArgs& a, bool act_bf16) {
  return act_bf16 && a.d == kD && a.F == kF && a.Hq == kG * a.Hkv && a.Bmax <= kBlk &&
         (long long)a.num_slots * a.Hkv * kF < (1ll << 31);
}

cudaError_t launch_hybrid_tc(const HybridArgs& a, cudaStream_t st) {
  TcHybridParams p;
  const uint64_t T = (uint64_t)a.T;
  {
    const uint64_t dims[3] = {kD, (uint64_t)a.Hq, T};
    const uint64_t strides[2] = {kD * 2, (uint64_t)a.Hq * kD * 2};
    const uint32_t box[3] = {64, kG, kBlk};
    if (!make_tensor_map(&p.tm_q, false, 3, a.Q, dims, strides, box, false)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {kD, (uint64_t)a.Hkv, T};
    const uint64_t strides[2] = {kD * 2, (uint64_t)a.Hkv * kD * 2};
    const uint32_t box[3] = {64, 1, kBlk};
    if (!make_tensor_map(&p.tm_k, false, 3, a.K, dims, strides, box, false)) return cudaErrorInvalidValue;
    if (!make_tensor_map(&p.tm_v, false, 3, a.V, dims, strides, box, false)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {kFh, (uint64_t)a.Hkv * kD};
    const uint64_t strides[1] = {kFh * 2};
    const uint32_t box[2] = {64, kD};
    if (!make_tensor_map(&p.tm_w, false, 2, a.W, dims, strides, box, false)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {kD, (uint64_t)a.num_slots * a.Hkv * kF};
    const uint64_t strides[1] = {kD * 4};
    const uint32_t box[2] = {32, kChunk};
    if (!make_tensor_map(&p.tm_s, true, 2, a.S, dims, strides, box, true)) return cudaErrorInvalidValue;
  }
  p.cu_blk = a.cu_blk;
  p.state_slot = a.state_slot;
  p.Z = a.Z;
  p.alpha = a.alpha;
  p.O = static_cast<__nv_bfloat16*>(a.O);
  p.dev_err = a.dev_err;
  p.R = a.R;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.T = a.T;
  p.Bmax = a.Bmax;
  p.num_slots = a.num_slots;
  p.wait_limit = 2000000000ll;  // about one second of SM cycles

  const int units = a.R * a.Hkv;
  int nsm = device_sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  int grid = nsm;
  if (a.Hkv <= nsm) grid = (nsm / a.Hkv) * a.Hkv;  // keeps each CTA on one KV head
  if (grid > units) grid = units;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(hybrid_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  hybrid_tc_kernel<<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace bha
