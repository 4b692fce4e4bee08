// Tensor-core block commit for sm_100a (bf16 activations, d = 128, F = 256, blocks of up
// to 128 tokens).
//
// Source: "Retrofitting Linear Attention into Diffusion Language Models", §3.1, the commit
// of a finished block:  S_n = S_{n-1} + sum_{t in B_n} phi(k_t) v_t^T,  Z_n = Z_{n-1} +
// sum_{t in B_n} phi(k_t),  phi(k) = [softmax(kW), softmax(-kW)].
//
// Work unit: 128 / kBt requests that share KV head g, kBt = 32, 64 or 128 the smallest that
// holds the call's largest block (their key rows form one 128-row MMA tile for u = K W_g).
// Per unit:
//   u     = K W_g                 bf16 MMA, M 128 (requests x kBt tokens), N 128, K 128
//   phi   = [softmax(u), softmax(-u)] per row on CUDA cores (two threads per row), rounded
//           to bf16 into shared memory as the B operand of the next MMA; rows past a
//           request's block are zero, so they add nothing
//   dZ    = column sums of the bf16 phi over each request's tokens (CUDA cores)
//   dS^T  = V_r^T phi_r           bf16 MMA per request, M 128 (d), N 256 (F), K kBt (tokens)
//                                 into one of two TMEM buffers
//   S += dS, Z += dZ               TMA bulk reduce-add: each of 8 warps copies 16 columns of
//                                 dS^T at a time from TMEM (its lane quarter = 32 values of d)
//                                 into a 2 KiB shared tile [16 rows of F][32 d] and hands it
//                                 to the tensor memory accelerator, which adds it into S in
//                                 L2; Z by reducing atomic adds.  No thread waits on a load of
//                                 S, and the other dS buffer's MMA overlaps the update.
// Computing dS transposed (lanes = d) is what lets each warp write whole 128-byte rows of its
// shared tile, one per instruction, without bank conflicts.  When each CTA has one unit, its
// states are prefetched into L2 as soon as K, V and W have landed, so the reduce-adds find
// them there.
//
// Roles (320 threads): warp 0 TMA producer (K, V, W), warp 1 TMEM owner and MMA issuer,
// warps 2-9 feature map, dZ and the state update.  Every wait is bounded; on expiry the CTA
// records BHA_ERR_TIMEOUT, drains its copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "tc_util.cuh"

namespace bha {
namespace {

constexpr int kD = 128;
constexpr int kF = 256;
constexpr int kFh = 128;
constexpr int kM = 128;          // key rows per unit: kM / kBt requests of up to kBt tokens
constexpr int kThreads = 320;

constexpr uint32_t kKBytes = kM * kD * 2;        // 32 KiB: [d half][128 rows][128 B]
constexpr uint32_t kWBytes = kD * kFh * 2;       // 32 KiB: [f half][128 rows of d][128 B]
constexpr int kRedRows = 16;                      // F rows per reduce-add tile

constexpr uint32_t kColU = 0;     // u (128 columns), inside dS buffer 0
constexpr uint32_t kColD0 = 0;    // dS^T buffers: 256 columns each
constexpr uint32_t kColD1 = 256;
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kIdKW = tc::instr_desc(1, 0, 1, kM, kFh);   // A K-major, B MN-major
constexpr uint32_t kIdVP = tc::instr_desc(1, 1, 1, kD, kF);    // A MN-major (V^T), B MN-major

// Block rows per request kBt = 32, 64 or 128 (the smallest that holds the call's largest
// block); a unit is kM / kBt requests.  Per request, V is [d half][kBt rows][128 B] and phi
// [F quarter][kBt rows][128 B], so the buffers of a unit have the same size for every kBt.
template <int kBt>
struct Shape {
  static constexpr int kReq = kM / kBt;
  static constexpr uint32_t kVReqBytes = kBt * kD * 2;
  static constexpr uint32_t kPhiReqBytes = kBt * kF * 2;
};

template <int kBt>
struct __align__(1024) Smem {
  uint8_t k[kKBytes];
  uint8_t w[kWBytes];
  uint8_t v[Shape<kBt>::kReq][Shape<kBt>::kVReqBytes];
  uint8_t phi[Shape<kBt>::kReq][Shape<kBt>::kPhiReqBytes];
  float dz[Shape<kBt>::kReq][kF];
  float red[8][2][kRedRows * 32];  // per update warp, double-buffered: [16 rows of F][32 d]
  uint64_t k_full, k_empty, v_full, v_empty, w_full, u_full, phi_ready;
  uint64_t d_full[2], d_empty[2], drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Smem<32>) + 1024 <= 232448 && sizeof(Smem<128>) + 1024 <= 232448,
              "shared memory budget");

struct Req {
  int lo, n, slot;  // n = 0: absent (no request, empty block or invalid)
};

// The kReq requests of unit (j0, g); every role decodes them identically.
template <int kReq>
__device__ __forceinline__ void decode_unit(const TcCommitParams& p, int j0, bool report,
                                            Req (&rq)[kReq]) {
#pragma unroll
  for (int j = 0; j < kReq; ++j) {
    rq[j].n = 0;
    rq[j].lo = 0;
    rq[j].slot = 0;
    const int r = j0 + j;
    if (r >= p.R) continue;
    RowRange rr;
    if (!request_rows(p.cu_blk, r, p.T, p.Bmax, p.dev_err, report, &rr)) continue;
    int slot;
    if (!request_slot(p.state_slot, r, p.num_slots, p.dev_err, report, &slot)) continue;
    rq[j].lo = rr.lo;
    rq[j].n = rr.n;
    rq[j].slot = slot;
  }
}

// One thread's half of phi for one key row: e = 2^{(s u - max_f s u) log2 e} over the 128
// values s u of its half (s = +1 or -1, u read from TMEM a 32-column chunk at a time),
// phi = e / sum e rounded to bf16 and written as 16 row chunks of 16 bytes, chunk c of F
// quarter q at quarter q, chunk position c ^ (t % 8) (the 128-byte swizzle the MMA reads).
// Rows past the block (live false) are written as zeros, selected rather than multiplied, so
// stale shared memory cannot inject a NaN.
//
// Two forms with the same result up to rounding: phi_row_fp32 keeps the 128 e values in fp32
// registers; phi_row_fp16 reads u twice and keeps e as fp16 pairs (11 significant bits,
// eight times finer than the bf16 phi they become; e <= 1 and the values fp16 flushes are
// below 2^-24 of the sum), which leaves about 64 more registers for the rest of the thread.
__device__ __forceinline__ void phi_row_store(uint8_t* row_base, uint32_t quarter_bytes, int t, bool live,
                                              int c, uint4 v) {
  const int quarter = c >> 3, ch = c & 7;
  *reinterpret_cast<uint4*>(row_base + quarter * quarter_bytes + ((ch ^ (t & 7)) << 4)) =
      live ? v : make_uint4(0, 0, 0, 0);
}

__device__ __forceinline__ void phi_row_fp32(uint32_t tu, float sgn, uint8_t* row_base,
                                             uint32_t quarter_bytes, int t, bool live) {
  const float log2e = 1.4426950408889634f;
  float e[kFh];
  float ext = -INFINITY;
#pragma unroll
  for (int c = 0; c < kFh / 32; ++c) {
    float uv[32];
    tc::tmem_ld32(tu + c * 32, uv);
    tc::tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      e[c * 32 + i] = sgn * uv[i];
      ext = fmaxf(ext, e[c * 32 + i]);
    }
  }
  float esum = 0.f;
#pragma unroll
  for (int i = 0; i < kFh; ++i) {
    e[i] = tc::ex2((e[i] - ext) * log2e);
    esum += e[i];
  }
  const float inv = 1.f / esum;
#pragma unroll
  for (int c = 0; c < kFh / 8; ++c)
    phi_row_store(row_base, quarter_bytes, t, live, c,
                  make_uint4(pack_bf16(e[8 * c] * inv, e[8 * c + 1] * inv),
                             pack_bf16(e[8 * c + 2] * inv, e[8 * c + 3] * inv),
                             pack_bf16(e[8 * c + 4] * inv, e[8 * c + 5] * inv),
                             pack_bf16(e[8 * c + 6] * inv, e[8 * c + 7] * inv)));
}

__device__ __forceinline__ void phi_row_fp16(uint32_t tu, float sgn, uint8_t* row_base,
                                             uint32_t quarter_bytes, int t, bool live) {
  const float log2e = 1.4426950408889634f;
  float ext = -INFINITY;
#pragma unroll 1
  for (int c = 0; c < kFh / 32; ++c) {
    float uv[32];
    tc::tmem_ld32(tu + c * 32, uv);
    tc::tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) ext = fmaxf(ext, sgn * uv[i]);
  }
  float esum = 0.f;
  __half2 eh[kFh / 2];
#pragma unroll
  for (int c = 0; c < kFh / 32; ++c) {
    float uv[32];
    tc::tmem_ld32(tu + c * 32, uv);
    tc::tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float e0 = tc::ex2((sgn * uv[i] - ext) * log2e);
      const float e1 = tc::ex2((sgn * uv[i + 1] - ext) * log2e);
      esum += e0 + e1;
      eh[(c * 32 + i) / 2] = __floats2half2_rn(e0, e1);
    }
  }
  const float inv = 1.f / esum;
#pragma unroll
  for (int c = 0; c < kFh / 8; ++c) {
    const float2 p0 = __half22float2(eh[4 * c]), p1 = __half22float2(eh[4 * c + 1]);
    const float2 p2 = __half22float2(eh[4 * c + 2]), p3 = __half22float2(eh[4 * c + 3]);
    phi_row_store(row_base, quarter_bytes, t, live, c,
                  make_uint4(pack_bf16(p0.x * inv, p0.y * inv), pack_bf16(p1.x * inv, p1.y * inv),
                             pack_bf16(p2.x * inv, p2.y * inv), pack_bf16(p3.x * inv, p3.y * inv)));
  }
}

// dZ[f] of one request: the sum over its n tokens of the bf16 phi column f (base: the
// request's phi at f's quarter and f's 2-byte position in its chunk ch); kAcc independent
// partial sums keep that many loads in flight.
template <int kAcc>
__device__ __forceinline__ float phi_column_sum(const uint8_t* base, int n, int ch) {
  auto at = [&](int tt) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + tt * 128 + ((ch ^ (tt & 7)) << 4)));
  };
  float a[kAcc];
#pragma unroll
  for (int i = 0; i < kAcc; ++i) a[i] = 0.f;
  int tt = 0;
  for (; tt + kAcc <= n; tt += kAcc)
#pragma unroll
    for (int i = 0; i < kAcc; ++i) a[i] += at(tt + i);
  for (; tt < n; ++tt) a[0] += at(tt);
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < kAcc; ++i) sum += a[i];
  return sum;
}

// The four-sum form as a call of its own, so that its registers are allocated apart from the
// feature map's (inlined, it pushes the 64- and 128-row instantiations into spills).
__device__ __noinline__ float phi_column_sum4(const uint8_t* base, int n, int ch) {
  return phi_column_sum<4>(base, n, ch);
}

template <int kBt>
__global__ void __launch_bounds__(kThreads, 1) commit_tc_kernel(const __grid_constant__ TcCommitParams p) {
  constexpr int kReq = Shape<kBt>::kReq;
  constexpr uint32_t kVReqBytes = Shape<kBt>::kVReqBytes;
  constexpr uint32_t kPhiReqBytes = Shape<kBt>::kPhiReqBytes;
  extern __shared__ uint8_t smem_raw[];
  Smem<kBt>& sm = *reinterpret_cast<Smem<kBt>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;
  const long long lim = p.wait_limit;
  const int groups = (p.R + kReq - 1) / kReq;
  const int units = groups * p.Hkv;

  if (threadIdx.x == 0) {
    tc::mbar_init(&sm.k_full, 1);
    tc::mbar_init(&sm.k_empty, 1);
    tc::mbar_init(&sm.v_full, 1);
    tc::mbar_init(&sm.v_empty, 1);
    tc::mbar_init(&sm.w_full, 1);
    tc::mbar_init(&sm.u_full, 1);
    tc::mbar_init(&sm.phi_ready, 8);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&sm.d_full[i], 1);
      tc::mbar_init(&sm.d_empty[i], 8);
    }
    tc::mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
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
      int k = 0, g_res = -1;
      uint32_t w_loads = 0;
      int armed_k = -1, armed_v = -1, armed_w = -1;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const int g = u % p.Hkv, j0 = (u / p.Hkv) * kReq;
        Req rq[kReq];
        decode_unit(p, j0, true, rq);
        int nreq = 0;
#pragma unroll
        for (int j = 0; j < kReq; ++j) nreq += rq[j].n > 0;
        if (nreq == 0) continue;
        if (g != g_res) {
          if (k >= 1 && !tc::mbar_wait(&sm.u_full, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
          tc::mbar_arrive_expect_tx(&sm.w_full, kWBytes);
          tc::tma_load_2d(sm.w, &p.tm_w, &sm.w_full, 0, g * kD);
          tc::tma_load_2d(sm.w + kWBytes / 2, &p.tm_w, &sm.w_full, 64, g * kD);
          armed_w = w_loads & 1;
          ++w_loads;
          g_res = g;
        }
        if (k >= 1 && !tc::mbar_wait(&sm.k_empty, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
        tc::mbar_arrive_expect_tx(&sm.k_full, nreq * 2 * (kBt * 64 * 2));
#pragma unroll
        for (int j = 0; j < kReq; ++j) {
          if (rq[j].n == 0) continue;
          tc::tma_load_3d(sm.k + j * kBt * 128, &p.tm_k, &sm.k_full, 0, g, rq[j].lo);
          tc::tma_load_3d(sm.k + kKBytes / 2 + j * kBt * 128, &p.tm_k, &sm.k_full, 64, g, rq[j].lo);
        }
        armed_k = k & 1;
        if (k >= 1 && !tc::mbar_wait(&sm.v_empty, (k - 1) & 1, abort_flag, lim)) { ok = false; break; }
        tc::mbar_arrive_expect_tx(&sm.v_full, nreq * kVReqBytes);
#pragma unroll
        for (int j = 0; j < kReq; ++j) {
          if (rq[j].n == 0) continue;
          tc::tma_load_3d(sm.v[j], &p.tm_v, &sm.v_full, 0, g, rq[j].lo);
          tc::tma_load_3d(sm.v[j] + kVReqBytes / 2, &p.tm_v, &sm.v_full, 64, g, rq[j].lo);
        }
        armed_v = k & 1;
        // When every CTA has a single unit (the serving commit: 128 requests x 4 KV heads in
        // 128 units), the unit's states are asked into L2 once its K, V and W have landed:
        // their HBM reads then overlap the feature map instead of starting with the first
        // reduce-add, and do not delay the loads the feature map needs first (30.9 us
        // against 34.5 us without the prefetch and 32.2 us issuing it with K and V).  With
        // more units per CTA one unit's state traffic already overlaps the next unit's
        // compute, and the extra requests only contend.
        if (units <= (int)gridDim.x) {
          if (!tc::mbar_wait(&sm.k_full, k & 1, abort_flag, lim) || !tc::mbar_wait(&sm.v_full, k & 1, abort_flag, lim) ||
              !tc::mbar_wait(&sm.w_full, (w_loads - 1) & 1, abort_flag, lim)) { ok = false; break; }
#pragma unroll 1
          for (int j = 0; j < kReq; ++j) {
            if (rq[j].n == 0) continue;
            // one (slot, head) state: 128 KiB, asked for in four 32 KiB pieces
            constexpr uint32_t kPiece = kF * kD * 4 / 4;
            const char* sb = reinterpret_cast<const char*>(p.S + ((size_t)rq[j].slot * p.Hkv + g) * kF * kD);
#pragma unroll 1
            for (int c = 0; c < 4; ++c) tc::bulk_prefetch_l2(sb + c * kPiece, kPiece);
          }
        }
        ++k;
      }
      volatile int never = 0;
      if (armed_k >= 0) tc::mbar_wait(&sm.k_full, armed_k, &never, lim);
      if (armed_v >= 0) tc::mbar_wait(&sm.v_full, armed_v, &never, lim);
      if (armed_w >= 0) tc::mbar_wait(&sm.w_full, armed_w, &never, lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int k = 0, g_res = -1, rc = 0;
      uint32_t w_seen = 0;
      int uses[2] = {0, 0};  // completed-or-issued uses of each dS buffer
      bool ok = true, issued = false;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const int g = u % p.Hkv, j0 = (u / p.Hkv) * kReq;
        Req rq[kReq];
        decode_unit(p, j0, false, rq);
        int nreq = 0;
#pragma unroll
        for (int j = 0; j < kReq; ++j) nreq += rq[j].n > 0;
        if (nreq == 0) continue;
        if (g != g_res) {
          if (!tc::mbar_wait(&sm.w_full, w_seen & 1, abort_flag, lim)) { ok = false; break; }
          ++w_seen;
          g_res = g;
        }
        if (!tc::mbar_wait(&sm.k_full, k & 1, abort_flag, lim)) { ok = false; break; }
        // u lands in dS buffer 0: its last state update must have read it
        if (uses[0] >= 1 && !tc::mbar_wait(&sm.d_empty[0], (uses[0] - 1) & 1, abort_flag, lim)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t ka = tc::smem_u32(sm.k), wa = tc::smem_u32(sm.w);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t a = tc::smem_desc(ka + (kk >> 2) * (kKBytes / 2) + (kk & 3) * 32, 16, 1024, tc::kSwizzle128B);
          const uint64_t b = tc::smem_desc(wa + kk * 2048, kWBytes / 2, 1024, tc::kSwizzle128B);
          tc::mma_bf16_ss(tbase + kColU, a, b, kIdKW, kk > 0);
        }
        tc::mma_commit(&sm.u_full);
        tc::mma_commit(&sm.k_empty);
        issued = true;
        if (!tc::mbar_wait(&sm.phi_ready, k & 1, abort_flag, lim)) { ok = false; break; }
        if (!tc::mbar_wait(&sm.v_full, k & 1, abort_flag, lim)) { ok = false; break; }
        for (int j = 0; j < kReq && ok; ++j) {
          if (rq[j].n == 0) continue;
          const int b = rc & 1;
          if (uses[b] >= 1 && !tc::mbar_wait(&sm.d_empty[b], (uses[b] - 1) & 1, abort_flag, lim)) { ok = false; break; }
          tc::tc_fence_after();
          const uint32_t va = tc::smem_u32(sm.v[j]), pa = tc::smem_u32(sm.phi[j]);
#pragma unroll
          for (int kk = 0; kk < kBt / 16; ++kk) {
            // A = V^T (M = d, K = tokens), MN-major: d halves 4 KiB apart, 8-token groups 1 KiB
            const uint64_t a = tc::smem_desc(va + kk * 2048, kVReqBytes / 2, 1024, tc::kSwizzle128B);
            // B = phi (K = tokens, N = F), MN-major: F quarters 4 KiB apart
            const uint64_t bd = tc::smem_desc(pa + kk * 2048, kPhiReqBytes / 4, 1024, tc::kSwizzle128B);
            tc::mma_bf16_ss(tbase + (b ? kColD1 : kColD0), a, bd, kIdVP, kk > 0);
          }
          tc::mma_commit(&sm.d_full[b]);
          ++uses[b];
          ++rc;
        }
        if (!ok) break;
        tc::mma_commit(&sm.v_empty);
        ++k;
      }
      if (issued) {
        volatile int never = 0;
        tc::mma_commit(&sm.drain);
        tc::mbar_wait(&sm.drain, 0, &never, lim);
      }
    }
  } else {
    // ------------------------------------------------------------ feature map, dZ, state update
    const int sw = warp - 2;          // 0..7
    const int half = sw >> 2;         // feature-map half / F half of the state update
    const float sgn = half ? -1.f : 1.f;
    const int wq = warp & 3;          // TMEM lane quarter
    const int row = wq * 32 + lane;   // key row = kBt j + t during the feature map; d afterwards
    const int tid = sw * 32 + lane;   // 0..255
    const uint32_t tl = tbase + ((uint32_t)(wq * 32) << 16);
    int k = 0, rc = 0, nred = 0;
    // A failed wait does not leave the loop at once: these 256 threads meet at a named barrier
    // each unit, so all of them reach it and leave together, decided by the reducing barrier.
    // Work done after a failed wait goes no further than shared memory (S and Z are not
    // written).
    bool good = true;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      const int g = u % p.Hkv, j0 = (u / p.Hkv) * kReq;
      Req rq[kReq];
      decode_unit(p, j0, false, rq);
      int nreq = 0;
#pragma unroll
      for (int j = 0; j < kReq; ++j) nreq += rq[j].n > 0;
      if (nreq == 0) continue;
      good = tc::mbar_wait(&sm.u_full, k & 1, abort_flag, lim) && good;
      good = tc::mbar_wait(&sm.v_full, k & 1, abort_flag, lim) && good;
      tc::tc_fence_after();
      // ---- this thread's half of phi for key row `row`, rounded to bf16.  With 32-row request
      // slots the fp32 form fits the register budget; the 64- and 128-row instantiations
      // spill with it (about 200 bytes) and take the fp16 form.
      {
        const int jr = row / kBt, t = row % kBt;
        const bool live = t < rq[jr].n;
        uint8_t* row_base = sm.phi[jr] + (2 * half) * (kPhiReqBytes / 4) + t * 128;
        if constexpr (kBt == 32)
          phi_row_fp32(tl + kColU, sgn, row_base, kPhiReqBytes / 4, t, live);
        else
          phi_row_fp16(tl + kColU, sgn, row_base, kPhiReqBytes / 4, t, live);
      }
      // rows of V past a request's block (or of an absent request) are cleared, so that
      // nothing from another request can leak in through 0 x (non-finite) products
#pragma unroll
      for (int j = 0; j < kReq; ++j) {
        const int n = rq[j].n;
        if (n >= kBt || n == 0) continue;
        const int per_half = (kBt - n) * 8;
        for (int i = tid; i < 2 * per_half; i += 256) {
          const int hh = i / per_half, rem = i % per_half;
          *reinterpret_cast<uint4*>(sm.v[j] + hh * (kVReqBytes / 2) + (n + rem / 8) * 128 + (rem % 8) * 16) =
              make_uint4(0, 0, 0, 0);
        }
      }
      // phi and the cleared V rows go to the tensor cores (async proxy); once all 256 threads
      // have written theirs, the dS^T products may start
      tc::fence_proxy_async_smem();
      // ---- dZ[j][f] = sum over the block's tokens of the bf16 phi (thread tid owns f = tid).
      // With four requests per tile it is summed before phi is handed to the dS^T products,
      // one running sum; with one or two it is summed while the first product runs, four
      // partial sums at a time in a call of its own.  Measured at 32- and 128-token blocks:
      // 30.9-31.2 us and 39.7 us this way; 31.8 us with the four-sum call before the hand-off
      // at 32 tokens, 52.1 us with the one-sum form before the hand-off at 128.
      const int zf = tid, zq = zf >> 6, zch = (zf & 63) >> 3, zw = zf & 7;
      auto column_sums = [&](auto acc_tag) {
        constexpr int kAcc = decltype(acc_tag)::value;
#pragma unroll 1
        for (int j = 0; j < kReq; ++j) {
          const uint8_t* base = sm.phi[j] + zq * (kPhiReqBytes / 4) + zw * 2;
          sm.dz[j][zf] = kAcc == 1 ? phi_column_sum<1>(base, rq[j].n, zch) : phi_column_sum4(base, rq[j].n, zch);
        }
      };
      if constexpr (kBt == 32) {
        tc::tc_fence_before();
        if (tc::named_barrier_any(1, 256, !good)) break;
        tc::tc_fence_after();
        column_sums(std::integral_constant<int, 1>{});
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sm.phi_ready);
      } else {
        // phi and the cleared V rows go to the tensor cores (async proxy) once all 256 threads
        // have written theirs
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        if (tc::named_barrier_any(1, 256, !good)) break;
        tc::tc_fence_after();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sm.phi_ready);
        column_sums(std::integral_constant<int, 4>{});
      }

      // ---- state update per request: S[f][d] += dS^T[d][f] by tiled reduce-add, Z[f] += dZ[f]
      for (int j = 0; j < kReq; ++j) {
        if (rq[j].n == 0) continue;
        const int b = rc & 1;
        // (a failed wait skips this unit's remaining updates; the next barrier ends the loop)
        good = __all_sync(0xffffffffu, tc::mbar_wait(&sm.d_full[b], (rc >> 1) & 1, abort_flag, lim));
        if (!good) break;
        tc::tc_fence_after();
        const int srow0 = (rq[j].slot * p.Hkv + g) * kF + half * kFh;
        const uint32_t col0 = (b ? kColD1 : kColD0) + half * kFh;
#pragma unroll 1
        for (int fc = 0; fc < kFh / kRedRows; ++fc, ++nred) {
          float dv[kRedRows];
          tc::tmem_ld16(tl + col0 + fc * kRedRows, dv);
          // the tile's previous reduce (two tiles back) has read it
          if (lane == 0 && nred >= 2) tc::bulk_wait_read<1>();
          __syncwarp();
          tc::tmem_wait_ld();
          float* tile = sm.red[sw][nred & 1];
#pragma unroll
          for (int i = 0; i < kRedRows; ++i) tile[i * 32 + lane] = dv[i];
          tc::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tc::tma_reduce_add_2d(&p.tm_s, tile, wq * 32, srow0 + fc * kRedRows);
            tc::bulk_commit();
          }
        }
        // every column of this dS buffer has been read: the next request's MMA may reuse it
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sm.d_empty[b]);
        atomicAdd(p.Z + ((size_t)rq[j].slot * p.Hkv + g) * kF + tid, sm.dz[j][tid]);
        ++rc;
      }
      ++k;
    }
    // every reduce this warp started has completed (its shared tile read, its adds performed)
    if (lane == 0) tc::bulk_wait_all();
  }

  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tbase, kTmemCols);
  if (threadIdx.x == 0 && sm.abort_flag) set_error(p.dev_err, BHA_ERR_TIMEOUT);
}

}  // namespace

bool commit_tc_supports(const CommitArgs& a, bool act_bf16) {
  return act_bf16 && a.d == kD && a.F == kF && a.Bmax <= kM &&
         (long long)a.num_slots * a.Hkv * kF * kD < (1ll << 40);
}

namespace {

template <int kBt>
cudaError_t launch_commit_tc_bt(const CommitArgs& a, cudaStream_t st) {
  constexpr int kReq = Shape<kBt>::kReq;
  TcCommitParams p;
  const uint64_t T = (uint64_t)a.T;
  {
    const uint64_t dims[3] = {kD, (uint64_t)a.Hkv, T};
    const uint64_t strides[2] = {kD * 2, (uint64_t)a.Hkv * kD * 2};
    const uint32_t box[3] = {64, 1, kBt};
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
    // reduce-add target: S as rows of d fp32 values, 16 x 32 boxes (one warp's tile)
    const uint64_t dims[2] = {kD, (uint64_t)a.num_slots * a.Hkv * kF};
    const uint64_t strides[1] = {kD * 4};
    const uint32_t box[2] = {32, kRedRows};
    if (!make_tensor_map(&p.tm_s, true, 2, a.S, dims, strides, box, kTmaNone)) return cudaErrorInvalidValue;
  }
  p.cu_blk = a.cu_blk;
  p.state_slot = a.state_slot;
  p.S = a.S;
  p.Z = a.Z;
  p.dev_err = a.dev_err;
  p.R = a.R;
  p.Hkv = a.Hkv;
  p.T = a.T;
  p.Bmax = a.Bmax;
  p.num_slots = a.num_slots;
  p.wait_limit = 2000000000ll;
  const int units = ((a.R + kReq - 1) / kReq) * a.Hkv;
  int nsm = device_sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  int grid = nsm;
  if (a.Hkv <= nsm) grid = (nsm / a.Hkv) * a.Hkv;
  if (grid > units) grid = units;
  const size_t smem = sizeof(Smem<kBt>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(commit_tc_kernel<kBt>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  commit_tc_kernel<kBt><<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

// Requests of up to 32, 64 or 128 tokens per unit tile: 4, 2 or 1 request per unit.
cudaError_t launch_commit_tc(const CommitArgs& a, cudaStream_t st) {
  if (a.Bmax <= 32) return launch_commit_tc_bt<32>(a, st);
  if (a.Bmax <= 64) return launch_commit_tc_bt<64>(a, st);
  return launch_commit_tc_bt<128>(a, st);
}

}  // namespace bha
