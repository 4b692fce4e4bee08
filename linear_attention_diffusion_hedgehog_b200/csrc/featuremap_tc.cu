// Tensor-core Hedgehog feature map for sm_100a (bf16 x, d = 128, F = 256, fp32 or bf16 phi).
//
// Source: "Retrofitting Linear Attention into Diffusion Language Models", §3.1:
//   phi(x) = [softmax(x W), softmax(-x W)],  each half normalised over its F/2 = 128 entries.
//
// Tile: 128 rows that share one weight matrix W_g: row r = t * G + j is head g G + j of token
// t0 + t (G = x_heads / Hkv heads per weight matrix), exactly the order x has in memory, so a
// tile is one 3-D TMA box.  Tiles are numbered (token tile, g) with g fastest; a persistent
// grid whose stride is a multiple of Hkv keeps one W_g resident per CTA.
//
// With u = x W_g (tcgen05, bf16, fp32 accumulator in TMEM):
//   e+_f = 2^{(u_f - max u) log2 e},  e-_f = 2^{(min u - u_f) log2 e},
//   phi = [e+ / sum e+, e- / sum e-].
// Roles (320 threads):
//   warp 0      TMA producer: W_g when it changes, x tiles through a 2-stage ring.
//   warp 1      TMEM owner and MMA issuer: u of tile k into TMEM buffer k % 2 (two buffers of
//               256 columns: u, then e- in place, and e+ beside it), so the next tile's MMA
//               overlaps this tile's epilogue.
//   warps 2-9   two groups of four, taking alternate tiles (warps 2-5 the even ones, 6-9 the
//               odd ones, matching the TMEM buffers), so one group's exponentials overlap the
//               other group's read-out and stores.  In a group, warp wq owns TMEM lane quarter
//               wq and each thread one whole row: max and min of its 128 u values; e+ written
//               beside u with its sum and read back normalised, 128 bytes of the row at a
//               time, each thread storing them as whole 32-byte sectors not allocated in L1
//               (when phi is only 16-byte aligned: 32 rows x 128 bytes at a time through a
//               double-buffered staging slot and one asynchronous bulk tensor store); then e-
//               over u in place, likewise.  Storing phi+ before e- is computed halves the time
//               from a tile's u to its first store.
//
// Every wait is bounded.  On expiry the CTA stops early, the call's output is undefined and
// BHA_ERR_TIMEOUT goes to dev_err when the caller passed one; nothing traps and TMEM is freed.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_util.cuh"

namespace bha {
namespace {

constexpr int kD = 128;
constexpr int kFh = 128;
constexpr int kM = 128;
constexpr int kThreads = 320;

constexpr uint32_t kXBytes = kM * kD * 2;      // 32 KiB: [d half][128 rows][128 B]
constexpr uint32_t kWBytes = kD * kFh * 2;     // 32 KiB: [f half][128 rows of d][128 B]
constexpr uint32_t kStgBytes = 32 * 128;       // 4 KiB: 32 rows x 128 bytes

constexpr uint32_t kTmemCols = 512;            // two buffers of [u / e- (128) | e+ (128)]
constexpr uint32_t kIdXW = tc::instr_desc(1, 0, 1, kM, kFh);  // bf16, B MN-major

struct __align__(1024) Smem {
  uint8_t x[2][kXBytes];
  uint8_t w[kWBytes];
  uint8_t stg[8][2][kStgBytes];  // per epilogue warp, two staging slots (128-byte swizzle)
  uint64_t x_full[2], x_empty[2], u_full[2], tm_empty[2], w_full, drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory budget of one CTA per SM");

// Waits until at most one of this thread's committed bulk stores is still reading shared
// memory (the staging slot about to be rewritten belongs to the older one).
__device__ __forceinline__ void bulk_wait_read_one() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

__global__ void __launch_bounds__(kThreads, 1) featuremap_tc_kernel(const __grid_constant__ TcFeatParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;
  const long long lim = p.wait_limit;
  const int tok_per_tile = kM / p.G;
  const int tiles = p.Hw * ((p.T + tok_per_tile - 1) / tok_per_tile);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&sm.x_full[i], 1);
      tc::mbar_init(&sm.x_empty[i], 1);
      tc::mbar_init(&sm.u_full[i], 1);
      tc::mbar_init(&sm.tm_empty[i], 4);  // the four warps of the tile's group
    }
    tc::mbar_init(&sm.w_full, 1);
    tc::mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tensormap(&p.tm_x);
    tc::prefetch_tensormap(&p.tm_w);
    tc::prefetch_tensormap(&p.tm_o);
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
      int g_res = -1, k = 0, armed_x[2] = {-1, -1}, armed_w = -1;
      uint32_t w_loads = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++k) {
        const int g = t % p.Hw, t0 = (t / p.Hw) * tok_per_tile;
        if (g != g_res) {
          // W is read only by the MMAs: the previous tile's must be done
          if (k >= 1 && !tc::mbar_wait(&sm.u_full[(k - 1) & 1], ((k - 1) >> 1) & 1, abort_flag, lim)) { ok = false; break; }
          tc::mbar_arrive_expect_tx(&sm.w_full, kWBytes);
          tc::tma_load_2d(sm.w, &p.tm_w, &sm.w_full, 0, g * kD);
          tc::tma_load_2d(sm.w + kWBytes / 2, &p.tm_w, &sm.w_full, 64, g * kD);
          armed_w = w_loads & 1;
          ++w_loads;
          g_res = g;
        }
        const int b = k & 1;
        if (k >= 2 && !tc::mbar_wait(&sm.x_empty[b], ((k - 2) >> 1) & 1, abort_flag, lim)) { ok = false; break; }
        tc::mbar_arrive_expect_tx(&sm.x_full[b], kXBytes);
        tc::tma_load_3d(sm.x[b], &p.tm_x, &sm.x_full[b], 0, g * p.G, t0);
        tc::tma_load_3d(sm.x[b] + kXBytes / 2, &p.tm_x, &sm.x_full[b], 64, g * p.G, t0);
        armed_x[b] = (k >> 1) & 1;
      }
      // Drain: every copy this thread started has landed before the CTA can exit.
      volatile int never = 0;
      for (int b = 0; b < 2; ++b)
        if (armed_x[b] >= 0) tc::mbar_wait(&sm.x_full[b], armed_x[b], &never, lim);
      if (armed_w >= 0) tc::mbar_wait(&sm.w_full, armed_w, &never, lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int g_res = -1, k = 0;
      uint32_t w_seen = 0;
      bool ok = true, issued = false;
      const uint32_t wa = tc::smem_u32(sm.w);
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++k) {
        const int g = t % p.Hw, b = k & 1;
        if (g != g_res) {
          if (!tc::mbar_wait(&sm.w_full, w_seen & 1, abort_flag, lim)) { ok = false; break; }
          ++w_seen;
          g_res = g;
        }
        if (!tc::mbar_wait(&sm.x_full[b], (k >> 1) & 1, abort_flag, lim)) { ok = false; break; }
        // the TMEM buffer is free once the epilogue of tile k - 2 has read it
        if (k >= 2 && !tc::mbar_wait(&sm.tm_empty[b], ((k - 2) >> 1) & 1, abort_flag, lim)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t xa = tc::smem_u32(sm.x[b]);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t a = tc::smem_desc(xa + (kk >> 2) * (kXBytes / 2) + (kk & 3) * 32, 16, 1024, tc::kSwizzle128B);
          const uint64_t bd = tc::smem_desc(wa + kk * 2048, kWBytes / 2, 1024, tc::kSwizzle128B);
          tc::mma_bf16_ss(tbase + b * 256, a, bd, kIdXW, kk > 0);
        }
        tc::mma_commit(&sm.x_empty[b]);
        tc::mma_commit(&sm.u_full[b]);
        issued = true;
      }
      if (issued) {
        volatile int never = 0;
        tc::mma_commit(&sm.drain);
        tc::mbar_wait(&sm.drain, 0, &never, lim);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    // Two groups of four warps take alternate tiles (warps 2-5 the even ones, 6-9 the odd
    // ones, matching the two TMEM buffers), so one group's exponentials (MUFU) overlap the
    // other group's read-out and stores.  In a group, warp wq owns TMEM lane quarter wq and
    // each thread one whole row.
    const int sw = warp - 2;         // 0..7
    const int grp = sw >> 2;         // tile parity this warp's group takes
    const int wq = warp & 3;         // TMEM lane quarter this warp may access
    const uint32_t tl = tbase + ((uint32_t)(wq * 32) << 16);
    const float log2e = 1.4426950408889634f;
    const int row0 = wq * 32;  // the warp's 32 rows are one store box (see the host side)
    bool good = true;
    int k = 0, nst = 0;  // nst: bulk stores this warp has committed (staging slot rotation)
    for (int t = blockIdx.x; good && t < tiles; t += gridDim.x, ++k) {
      const int b = k & 1;
      if (b != grp) continue;
      const int g = t % p.Hw, t0 = (t / p.Hw) * tok_per_tile;
      const uint32_t tb = tl + b * 256;
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.u_full[b], (k >> 1) & 1, abort_flag, lim))) { good = false; break; }
      tc::tc_fence_after();

      // max and min of the row's 128 u values
      float mx = -INFINITY, mn = INFINITY;
#pragma unroll 1
      for (int c = 0; c < kFh / 32; c += 2) {
        float u0[32], u1[32];
        tc::tmem_ld32(tb + c * 32, u0);
        tc::tmem_ld32(tb + c * 32 + 32, u1);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          mx = fmaxf(mx, fmaxf(u0[i], u1[i]));
          mn = fminf(mn, fminf(u0[i], u1[i]));
        }
      }
      // phi, 32 rows x 128 bytes per store: fp32 in chunks of 32 columns, bf16 in chunks of
      // 64; half 0 (phi+) is stored while half 1's exponentials are computed
      const int tok_w = t0 + row0 / p.G;       // first token of this warp's rows
      const int head_w = g * p.G + row0 % p.G;  // first head of this warp's rows
      const bool store = tok_w < p.T;
      // this thread's row of phi: token t0 + row / G, head g G + row % G
      const int rtok = t0 + (row0 + lane) / p.G, rhead = g * p.G + (row0 + lane) % p.G;
      const bool rlive = rtok < p.T;
      char* rowp = static_cast<char*>(p.phi) + ((size_t)rtok * p.H + rhead) * (size_t)(2 * kFh) * (p.out_bf16 ? 2 : 4);
      const int nchunks = p.out_bf16 ? 2 : 4;  // per half
      // normalised read-out of one half (e at TMEM column src), one bulk store per chunk
      auto readout = [&](const int half, const uint32_t src, const float sc, const bool last) {
        for (int c = 0; c < nchunks; ++c) {
          uint32_t packed[32];
          int f0;  // first phi column of the chunk
          if (p.out_bf16) {
            float a[32], bb[32];
            tc::tmem_ld32(tb + src + c * 64, a);
            tc::tmem_ld32(tb + src + c * 64 + 32, bb);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              packed[i] = pack_bf16(a[2 * i] * sc, a[2 * i + 1] * sc);
              packed[16 + i] = pack_bf16(bb[2 * i] * sc, bb[2 * i + 1] * sc);
            }
            f0 = half * kFh + c * 64;
          } else {
            float a[32];
            tc::tmem_ld32(tb + src + c * 32, a);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) packed[i] = __float_as_uint(a[i] * sc);
            f0 = half * kFh + c * 32;
          }
          if (last && c == nchunks - 1) {
            // every TMEM read of this tile is done: the MMA may refill the buffer
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.tm_empty[b]);
          }
          if (p.o32) {
            // the row's 128 bytes of this chunk as four whole 32-byte sectors, not in L1
            if (rlive) {
              char* dst = rowp + (size_t)f0 * (p.out_bf16 ? 2 : 4);
#pragma unroll
              for (int q8 = 0; q8 < 4; ++q8) {
                uint32_t w[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) w[j] = packed[8 * q8 + j];
                tc::st_global_32B(dst + q8 * 32, w);
              }
            }
          } else {
          // staging slot nst % 2: its previous store (two stores ago) must have read it
          uint8_t* slot = sm.stg[sw][nst & 1];
          if (lane == 0) bulk_wait_read_one();
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(slot + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
          tc::fence_proxy_async_smem();
          __syncwarp();
          if (store) {
            if (lane == 0) {
              tc::tma_store_3d(&p.tm_o, slot, f0, head_w, tok_w);
              tc::bulk_commit();
            }
            ++nst;
          }
          }
        }
      };

      // e+ (unnormalised) into columns 128.. with its sum, then phi+ stored from there
      const float bpl = mx * log2e, bml = mn * log2e;
      float esp = 0.f, esm = 0.f;
#pragma unroll 1
      for (int c = 0; c < kFh / 32; ++c) {
        float uu[32];
        tc::tmem_ld32(tb + c * 32, uu);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          uu[i] = tc::ex2(uu[i] * log2e - bpl);
          esp += uu[i];
        }
        tc::tmem_st32(tb + 128 + c * 32, uu);
      }
      tc::tmem_wait_st();
      readout(0, 128, 1.f / esp, false);
      // e- over u in place with its sum, then phi- stored from there
#pragma unroll 1
      for (int c = 0; c < kFh / 32; ++c) {
        float uu[32];
        tc::tmem_ld32(tb + c * 32, uu);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          uu[i] = tc::ex2(bml - uu[i] * log2e);
          esm += uu[i];
        }
        tc::tmem_st32(tb + c * 32, uu);
      }
      tc::tmem_wait_st();
      readout(1, 0, 1.f / esm, true);
    }
    if (lane == 0) tc::bulk_wait_all();
  }

  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tbase, kTmemCols);
  if (threadIdx.x == 0 && sm.abort_flag) set_error(p.dev_err, BHA_ERR_TIMEOUT);
}

}  // namespace

// ----------------------------------------------------------------- host side
bool featuremap_tc_supports(int T, int x_heads, int Hw, int d, int F, bool act_bf16) {
  if (!act_bf16 || d != kD || F != 2 * kFh || T <= 0 || x_heads % Hw != 0) return false;
  const int G = x_heads / Hw;
  return G >= 1 && G <= kM && (G & (G - 1)) == 0;
}

cudaError_t launch_featuremap_tc(const void* x, int T, int x_heads, int Hw, const void* W, void* phi,
                                 bool out_bf16, int32_t* dev_err, cudaStream_t st) {
  TcFeatParams p;
  const int G = x_heads / Hw;
  {
    const uint64_t dims[3] = {kD, (uint64_t)x_heads, (uint64_t)T};
    const uint64_t strides[2] = {kD * 2, (uint64_t)x_heads * kD * 2};
    const uint32_t box[3] = {64, (uint32_t)G, (uint32_t)(kM / G)};
    if (!make_tensor_map(&p.tm_x, false, 3, x, dims, strides, box, kTma128B)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {kFh, (uint64_t)Hw * kD};
    const uint64_t strides[1] = {kFh * 2};
    const uint32_t box[2] = {64, kD};
    if (!make_tensor_map(&p.tm_w, false, 2, W, dims, strides, box, kTma128B)) return cudaErrorInvalidValue;
  }
  {
    // phi [T][x_heads][256]: 128-byte rows of 32 fp32 or 64 bf16 columns, one warp's 32 rows
    const int esz = out_bf16 ? 2 : 4;
    const uint64_t dims[3] = {2 * kFh, (uint64_t)x_heads, (uint64_t)T};
    const uint64_t strides[2] = {(uint64_t)2 * kFh * esz, (uint64_t)x_heads * 2 * kFh * esz};
    const uint32_t gy = G < 32 ? G : 32;
    const uint32_t box[3] = {(uint32_t)(128 / esz), gy, 32 / gy};
    if (!make_tensor_map(&p.tm_o, !out_bf16, 3, phi, dims, strides, box, kTma128B)) return cudaErrorInvalidValue;
  }
  p.T = T;
  p.H = x_heads;
  p.Hw = Hw;
  p.G = G;
  p.out_bf16 = out_bf16 ? 1 : 0;
  p.phi = phi;
  p.o32 = (reinterpret_cast<uintptr_t>(phi) & 31) == 0;
  p.wait_limit = 2000000000ll;  // about one second of SM cycles
  p.dev_err = dev_err;

  const int tok_per_tile = kM / G;
  const int tiles = Hw * ((T + tok_per_tile - 1) / tok_per_tile);
  int nsm = device_sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  // fewest CTAs that finish in the least number of rounds, a multiple of Hw when that costs no
  // round (each CTA then keeps one W_g resident)
  const int grid = persistent_grid(tiles, Hw, nsm);
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(featuremap_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  featuremap_tc_kernel<<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace bha
