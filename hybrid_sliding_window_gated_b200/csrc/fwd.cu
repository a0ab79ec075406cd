// fwd.cu -- fused prefill forward of the gated sliding-window attention core
// for sm_100a: TMA loads, QK-RMSNorm and partial RoPE in shared memory,
// tcgen05 QK^T and PV with TMEM accumulators, single-pass softmax over the
// 256-key band, and the sigmoid-gate epilogue.
//
// Definition (ZGCM-1 pages: onedev.kr summary, "어떻게 동작하나"; jaehun.me
// review, "How Gated SWA Behaves"): for query token i and head h,
//   q' = RoPE(RMSNorm(q)), k' = RoPE(RMSNorm(k)),
//   s_j = scale q'_i . k'_j for j in [i-127, i], P = softmax(s),
//   O_i = (sum_j P_j v_j) * sigmoid(g_i)   (element-wise gate).
//
// Work decomposition.  A "chain" is one (batch row, KV head); its tokens are
// cut into 128-row tiles.  Query tile t needs key tiles t-1 and t, so each
// persistent CTA walks a contiguous range of tiles and keeps K/V of the two
// live tiles in a 2-slot ring: every K/V tile is loaded, normalised and
// rotated once per range and shared by the G = Hq/Hkv query heads of its
// group and by two query tiles.
//
// Roles (512 threads):
//   warp 0      TMA producer (one lane)
//   warp 1      TMEM allocator and tcgen05.mma issuer (one lane)
//   warps 4-7   "transform": RMSNorm + RoPE of Q and K rows, in place in the
//               128-byte-swizzled tiles, one row per thread
//   warps 8-11  softmax + epilogue for TMEM region 0 (even head slots)
//   warps 12-15 softmax + epilogue for TMEM region 1 (odd head slots)
//
// TMEM (512 columns) holds two regions of 256 columns.  For a head in region
// r: S = Q [K_{t-1} K_t]^T fills all 256 columns (fp32); the softmax writes P
// as packed bf16 over the first 128 columns; PV accumulates O (fp32) into the
// last 128 columns; the epilogue reads O.  Regions alternate between heads so
// the tensor core works on one head while the softmax runs on the other.
#include "ptx.cuh"
#include "swa_internal.h"

namespace swa {

namespace fwd {

constexpr int kThreads = 512;
constexpr int kHalfBytes = kTile * 64 * 2;  // 128 rows x 64 bf16 = 16 KiB (one TMA box)
constexpr int kTileBytes = 2 * kHalfBytes;  // a full 128 x 128 bf16 tile

struct alignas(1024) Smem {
  uint8_t k[2][kTileBytes];
  uint8_t v[2][kTileBytes];
  uint8_t q[2][kTileBytes];
  float2 cs[kMaxPairs * kTile];  // per-row (cos, sin), laid out [pair][row]
  float wq[kHeadDim];
  float wk[kHeadDim];
  uint64_t kfull[2], kready[2], kempty[2];
  uint64_t vfull[2], vempty[2];
  uint64_t qfull[2], qready[2], qempty[2];
  uint64_t sfull[2], pfull[2], ofull[2], tfree[2];
  uint64_t drain, never;
  uint32_t tmem_base;
  int abort;
};

// Wait-site ids reported through the device error word.
enum Site {
  kSiteKEmpty = 1, kSiteVEmpty, kSiteQEmpty, kSiteKFull, kSiteQFull, kSiteKReady,
  kSiteQReady, kSiteTFree, kSiteVFull, kSitePFull, kSiteSFull, kSiteOFull, kSiteForced
};

struct Tile {
  int b, kvh, t;
  bool has_prev;   // key tile t-1 exists (t > 0)
  bool need_prev;  // ... and must be loaded here (first tile of a segment)
  bool seg_last;   // last tile of this CTA's run on the chain
};

__device__ __forceinline__ Tile tile_at(const FwdArgs& a, long long u, long long u0,
                                        long long u1) {
  Tile x;
  long long chain = u / a.tiles_per_chain;
  x.t = static_cast<int>(u - chain * a.tiles_per_chain);
  x.b = static_cast<int>(chain / a.Hkv);
  x.kvh = static_cast<int>(chain - static_cast<long long>(x.b) * a.Hkv);
  x.has_prev = x.t > 0;
  x.need_prev = x.has_prev && (u == u0);
  x.seg_last = (u == u1 - 1) || (x.t == a.tiles_per_chain - 1);
  return x;
}

// Offset of element d of row `row` inside a tile stored as two 128B-swizzled
// halves (the layout TMA SWIZZLE_128B writes): 16-byte chunk c of a 128-byte
// row lands at chunk c ^ (row & 7).
__device__ __forceinline__ uint32_t sw_off(int row, int chunk16) {
  return static_cast<uint32_t>(row * 128 + ((chunk16 ^ (row & 7)) << 4));
}

__device__ __forceinline__ void unpack8(const uint4& u, float* x) {
  x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x);
  x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
  x[4] = bf16_lo(u.z); x[5] = bf16_hi(u.z);
  x[6] = bf16_lo(u.w); x[7] = bf16_hi(u.w);
}

__device__ __forceinline__ uint4 pack8(const float* x) {
  uint4 u;
  u.x = pack_bf16x2(x[0], x[1]);
  u.y = pack_bf16x2(x[2], x[3]);
  u.z = pack_bf16x2(x[4], x[5]);
  u.w = pack_bf16x2(x[6], x[7]);
  return u;
}

// Fill this thread's (cos, sin) row for tile j (position j*128 + row).
template <int kPairs>
__device__ __forceinline__ void fill_cos_sin(Smem& sm, const FwdArgs& a, int j, int row) {
  const double pos = static_cast<double>(j) * kTile + row;
#pragma unroll
  for (int p = 0; p < kPairs; ++p) {
    float c, s;
    rope_cos_sin(pos, a.inv_freq[p], &c, &s);
    sm.cs[p * kTile + row] = make_float2(c, s);
  }
}

// RMSNorm (weight w) and partial RoPE of row `row` of a tile, in place.
template <int kPairs>
__device__ __forceinline__ void transform_row(uint8_t* tile, int row, const float* w,
                                              const float2* cs, float eps) {
  uint8_t* h0 = tile;
  uint8_t* h1 = tile + kHalfBytes;
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float x[8], y[8];
    unpack8(*reinterpret_cast<const uint4*>(h0 + sw_off(row, c)), x);
    unpack8(*reinterpret_cast<const uint4*>(h1 + sw_off(row, c)), y);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(x[i], x[i], fmaf(y[i], y[i], ss));
  }
  const float rinv = rsqrtf(ss * (1.0f / kHeadDim) + eps);

  constexpr int kRopeChunks = (2 * kPairs + 7) / 8;
  if constexpr (kRopeChunks > 0) {
    float x[kRopeChunks * 8];
#pragma unroll
    for (int c = 0; c < kRopeChunks; ++c)
      unpack8(*reinterpret_cast<const uint4*>(h0 + sw_off(row, c)), x + 8 * c);
#pragma unroll
    for (int d = 0; d < kRopeChunks * 8; ++d) x[d] = x[d] * rinv * w[d];
#pragma unroll
    for (int p = 0; p < kPairs; ++p) {
      const float2 t = cs[p * kTile + row];
      const float u = x[p], v = x[p + kPairs];
      x[p] = u * t.x - v * t.y;
      x[p + kPairs] = v * t.x + u * t.y;
    }
#pragma unroll
    for (int c = 0; c < kRopeChunks; ++c)
      *reinterpret_cast<uint4*>(h0 + sw_off(row, c)) = pack8(x + 8 * c);
  }
#pragma unroll
  for (int c = kRopeChunks; c < 8; ++c) {
    float x[8];
    unpack8(*reinterpret_cast<const uint4*>(h0 + sw_off(row, c)), x);
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = x[i] * rinv * w[8 * c + i];
    *reinterpret_cast<uint4*>(h0 + sw_off(row, c)) = pack8(x);
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float x[8];
    unpack8(*reinterpret_cast<const uint4*>(h1 + sw_off(row, c)), x);
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = x[i] * rinv * w[64 + 8 * c + i];
    *reinterpret_cast<uint4*>(h1 + sw_off(row, c)) = pack8(x);
  }
}

// K-major operand descriptor for k-step kk (16 elements) of a 128 x 128 tile.
__device__ __forceinline__ uint64_t desc_kmajor(const uint8_t* tile, int kk) {
  return make_desc_sw128(smem_u32(tile) + (kk >> 2) * kHalfBytes + (kk & 3) * 32, 16, 1024);
}
// MN-major descriptor of V (keys x dims, dims contiguous) for key step kk.
__device__ __forceinline__ uint64_t desc_v(const uint8_t* tile, int kk) {
  return make_desc_sw128(smem_u32(tile) + kk * 2048, kHalfBytes, 1024);
}

constexpr uint32_t kIdescQK = make_idesc_bf16(128, 128, false, false);
constexpr uint32_t kIdescPV = make_idesc_bf16(128, 128, false, true);

template <int kPairs>
__global__ void __launch_bounds__(kThreads, 1)
    swa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                   const FwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  const long long u0 = a.total_tiles * blockIdx.x / gridDim.x;
  const long long u1 = a.total_tiles * (blockIdx.x + 1) / gridDim.x;
  const long long n_heads = (u1 - u0) * a.G;

  if (tid < kHeadDim) {
    sm.wq[tid] = a.wq[tid];
    sm.wk[tid] = a.wk[tid];
  }
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.kfull[i], 1);
      mbar_init(&sm.kready[i], 128);
      mbar_init(&sm.kempty[i], 1);
      mbar_init(&sm.vfull[i], 1);
      mbar_init(&sm.vempty[i], 1);
      mbar_init(&sm.qfull[i], 1);
      mbar_init(&sm.qready[i], 128);
      mbar_init(&sm.qempty[i], 1);
      mbar_init(&sm.sfull[i], 1);
      mbar_init(&sm.pfull[i], 128);
      mbar_init(&sm.ofull[i], 1);
      mbar_init(&sm.tfree[i], 128);
    }
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.never, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_g);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t nk[2] = {0, 0}, nv[2] = {0, 0}, nq[2] = {0, 0};
      bool ok = true;
      auto load_kv = [&](const CUtensorMap* map, uint8_t (*buf)[kTileBytes], uint64_t* full,
                         uint64_t* empty, uint32_t* cnt, int j, const Tile& x, int site) {
        const int s = j & 1;
        if (cnt[s] > 0 && !mbar_wait(&empty[s], (cnt[s] - 1) & 1, abort, a.err, site)) return false;
        mbar_arrive_expect_tx(&full[s], kTileBytes);
        tma_load_4d(buf[s], map, &full[s], 0, x.kvh, j * kTile, x.b);
        tma_load_4d(buf[s] + kHalfBytes, map, &full[s], 64, x.kvh, j * kTile, x.b);
        ++cnt[s];
        return true;
      };
      long long n = 0;  // head slots issued so far; Q slot = n & 1
      for (long long u = u0; u < u1 && ok; ++u) {
        const Tile x = tile_at(a, u, u0, u1);
        if (x.need_prev) {
          ok = ok && load_kv(&tm_k, sm.k, sm.kfull, sm.kempty, nk, x.t - 1, x, kSiteKEmpty);
          ok = ok && load_kv(&tm_v, sm.v, sm.vfull, sm.vempty, nv, x.t - 1, x, kSiteVEmpty);
        }
        ok = ok && load_kv(&tm_k, sm.k, sm.kfull, sm.kempty, nk, x.t, x, kSiteKEmpty);
        for (int h = 0; h < a.G && ok; ++h) {
          const int s = static_cast<int>(n & 1);
          if (nq[s] > 0 && !mbar_wait(&sm.qempty[s], (nq[s] - 1) & 1, abort, a.err, kSiteQEmpty)) {
            ok = false;
            break;
          }
          const int hq = x.kvh * a.G + h;
          mbar_arrive_expect_tx(&sm.qfull[s], kTileBytes);
          tma_load_4d(sm.q[s], &tm_q, &sm.qfull[s], 0, hq, x.t * kTile, x.b);
          tma_load_4d(sm.q[s] + kHalfBytes, &tm_q, &sm.qfull[s], 64, hq, x.t * kTile, x.b);
          tma_prefetch_4d(&tm_g, 0, hq, x.t * kTile, x.b);
          ++nq[s];
          ++n;
          if (h == 0) ok = load_kv(&tm_v, sm.v, sm.vfull, sm.vempty, nv, x.t, x, kSiteVEmpty);
        }
      }
      if (!ok) {
        // Drain the loads this thread issued before the CTA releases its memory.
        for (int s = 0; s < 2; ++s) {
          if (nk[s]) mbar_wait_drain(&sm.kfull[s], (nk[s] - 1) & 1);
          if (nv[s]) mbar_wait_drain(&sm.vfull[s], (nv[s] - 1) & 1);
          if (nq[s]) mbar_wait_drain(&sm.qfull[s], (nq[s] - 1) & 1);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t nkr[2] = {0, 0}, nvr[2] = {0, 0};
      bool ok = true;
      if (a.flags & SWA_FLAG_FORCE_TIMEOUT) ok = mbar_wait(&sm.never, 0, abort, a.err, kSiteForced);

      auto do_qk = [&](long long n) -> bool {
        const long long u = u0 + n / a.G;
        const int h = static_cast<int>(n % a.G);
        const Tile x = tile_at(a, u, u0, u1);
        const int sp = (x.t + 1) & 1, sc = x.t & 1;
        if (h == 0) {
          if (x.need_prev) {
            if (!mbar_wait(&sm.kready[sp], nkr[sp] & 1, abort, a.err, kSiteKReady)) return false;
            ++nkr[sp];
          }
          if (!mbar_wait(&sm.kready[sc], nkr[sc] & 1, abort, a.err, kSiteKReady)) return false;
          ++nkr[sc];
        }
        const int r = static_cast<int>(n & 1);
        const uint32_t c = static_cast<uint32_t>(n >> 1);
        if (!mbar_wait(&sm.qready[r], c & 1, abort, a.err, kSiteQReady)) return false;
        if (c > 0 && !mbar_wait(&sm.tfree[r], (c - 1) & 1, abort, a.err, kSiteTFree)) return false;
        tc_fence_after();
        const uint32_t s_base = tmem + r * 256;
        for (int blk = x.has_prev ? 0 : 1; blk < 2; ++blk) {
          const uint8_t* kt = sm.k[blk == 0 ? sp : sc];
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(s_base + blk * 128, desc_kmajor(sm.q[r], kk), desc_kmajor(kt, kk), kIdescQK,
                   kk > 0);
        }
        mma_commit(&sm.sfull[r]);
        mma_commit(&sm.qempty[r]);
        if (h == a.G - 1) {
          if (x.has_prev) mma_commit(&sm.kempty[sp]);
          if (x.seg_last) mma_commit(&sm.kempty[sc]);
        }
        return true;
      };

      auto do_pv = [&](long long n) -> bool {
        const long long u = u0 + n / a.G;
        const int h = static_cast<int>(n % a.G);
        const Tile x = tile_at(a, u, u0, u1);
        const int sp = (x.t + 1) & 1, sc = x.t & 1;
        if (h == 0) {
          if (x.need_prev) {
            if (!mbar_wait(&sm.vfull[sp], nvr[sp] & 1, abort, a.err, kSiteVFull)) return false;
            ++nvr[sp];
          }
          if (!mbar_wait(&sm.vfull[sc], nvr[sc] & 1, abort, a.err, kSiteVFull)) return false;
          ++nvr[sc];
        }
        const int r = static_cast<int>(n & 1);
        const uint32_t c = static_cast<uint32_t>(n >> 1);
        if (!mbar_wait(&sm.pfull[r], c & 1, abort, a.err, kSitePFull)) return false;
        tc_fence_after();
        const uint32_t p_base = tmem + r * 256;
        const uint32_t o_base = p_base + 128;
        bool first = true;
        for (int blk = x.has_prev ? 0 : 1; blk < 2; ++blk) {
          const uint8_t* vt = sm.v[blk == 0 ? sp : sc];
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            mma_ts(o_base, p_base + blk * 64 + kk * 8, desc_v(vt, kk), kIdescPV, first ? 0u : 1u);
            first = false;
          }
        }
        mma_commit(&sm.ofull[r]);
        if (h == a.G - 1) {
          if (x.has_prev) mma_commit(&sm.vempty[sp]);
          if (x.seg_last) mma_commit(&sm.vempty[sc]);
        }
        return true;
      };

      for (long long n = 0; n < n_heads && ok; n += 2) {
        ok = do_qk(n);
        if (ok && n + 1 < n_heads) ok = do_qk(n + 1);
        if (ok) ok = do_pv(n);
        if (ok && n + 1 < n_heads) ok = do_pv(n + 1);
      }
      if (!ok) {
        // No tcgen05.mma may still be running when TMEM is released.
        mma_commit(&sm.drain);
        mbar_wait_drain(&sm.drain, 0);
      }
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 8) {
    // ---------------------------------------------------------- transform
    const int row = tid - 128;
    uint32_t nk[2] = {0, 0};
    long long n = 0;
    bool ok = true;
    auto do_k = [&](int j) -> bool {
      const int s = j & 1;
      if (!mbar_wait(&sm.kfull[s], nk[s] & 1, abort, a.err, kSiteKFull)) return false;
      fill_cos_sin<kPairs>(sm, a, j, row);
      transform_row<kPairs>(sm.k[s], row, sm.wk, sm.cs, a.eps);
      fence_proxy_async_smem();
      mbar_arrive(&sm.kready[s]);
      ++nk[s];
      return true;
    };
    for (long long u = u0; u < u1 && ok; ++u) {
      const Tile x = tile_at(a, u, u0, u1);
      if (x.need_prev) ok = do_k(x.t - 1);
      if (ok) ok = do_k(x.t);  // leaves the cos/sin rows of tile t for the Q heads
      for (int h = 0; h < a.G && ok; ++h, ++n) {
        const int s = static_cast<int>(n & 1);
        if (!mbar_wait(&sm.qfull[s], static_cast<uint32_t>(n >> 1) & 1, abort, a.err, kSiteQFull)) {
          ok = false;
          break;
        }
        transform_row<kPairs>(sm.q[s], row, sm.wq, sm.cs, a.eps);
        fence_proxy_async_smem();
        mbar_arrive(&sm.qready[s]);
      }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------ softmax + epilogue
    const int r = (warp - 8) >> 2;  // TMEM region served by this warpgroup
    const int wq4 = warp & 3;       // TMEM lane quarter
    const int row = wq4 * 32 + lane;
    const uint32_t t_row = tmem + (static_cast<uint32_t>(wq4 * 32) << 16);
    const uint32_t s_cols = t_row + r * 256;
    const float sl2 = a.scale_log2;
    bool ok = true;
    for (long long n = r; n < n_heads && ok; n += 2) {
      const long long u = u0 + n / a.G;
      const int h = static_cast<int>(n % a.G);
      const Tile x = tile_at(a, u, u0, u1);
      const uint32_t c = static_cast<uint32_t>(n >> 1);
      const int hq = x.kvh * a.G + h;
      const long long pos = static_cast<long long>(x.t) * kTile + row;
      const bool valid = pos < a.T;
      const long long elem = ((static_cast<long long>(x.b) * a.T + (valid ? pos : 0)) * a.Hq + hq) *
                             kHeadDim;
      const uint4* gp = reinterpret_cast<const uint4*>(a.g + elem);

      if (!mbar_wait(&sm.sfull[r], c & 1, abort, a.err, kSiteSFull)) { ok = false; break; }
      tc_fence_after();

      // Pass 1: row maximum over the band.  Key tile t-1 contributes columns
      // c > row, key tile t columns c <= row; 32-column chunks entirely
      // outside the band are skipped.
      float m = -INFINITY;
      uint32_t v[32];
      if (x.has_prev) {
        for (int ch = wq4; ch < 4; ++ch) {
          tmem_ld32(s_cols + ch * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (ch * 32 + i > row) m = fmaxf(m, __uint_as_float(v[i]));
        }
      }
      for (int ch = 0; ch <= wq4; ++ch) {
        tmem_ld32(s_cols + 128 + ch * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (ch * 32 + i <= row) m = fmaxf(m, __uint_as_float(v[i]));
      }
      const float ms = m * sl2;

      // Pass 2: P = exp2(s*scale*log2e - max), packed bf16 over the first 128
      // columns of the region; row sum in fp32.
      float l = 0.f;
      uint32_t pk[16];
      if (x.has_prev) {
        for (int ch = 0; ch < 4; ++ch) {
          if (ch < wq4) {
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = 0u;
          } else {
            tmem_ld32(s_cols + ch * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float p0 = (ch * 32 + 2 * i > row)
                                   ? ex2_approx(fmaf(__uint_as_float(v[2 * i]), sl2, -ms)) : 0.f;
              const float p1 = (ch * 32 + 2 * i + 1 > row)
                                   ? ex2_approx(fmaf(__uint_as_float(v[2 * i + 1]), sl2, -ms)) : 0.f;
              l += p0 + p1;
              pk[i] = pack_bf16x2(p0, p1);
            }
          }
          tmem_st16(s_cols + ch * 16, pk);
        }
      }
      for (int ch = 0; ch < 4; ++ch) {
        if (ch > wq4) {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = 0u;
        } else {
          tmem_ld32(s_cols + 128 + ch * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = (ch * 32 + 2 * i <= row)
                                 ? ex2_approx(fmaf(__uint_as_float(v[2 * i]), sl2, -ms)) : 0.f;
            const float p1 = (ch * 32 + 2 * i + 1 <= row)
                                 ? ex2_approx(fmaf(__uint_as_float(v[2 * i + 1]), sl2, -ms)) : 0.f;
            l += p0 + p1;
            pk[i] = pack_bf16x2(p0, p1);
          }
        }
        tmem_st16(s_cols + 64 + ch * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.pfull[r]);

      if (a.lse != nullptr && valid)
        a.lse[(static_cast<long long>(x.b) * a.Hq + hq) * a.T + pos] =
            (ms + __log2f(l)) * 0.6931471805599453f;
      const float inv_l = 1.0f / l;

      // Epilogue: O / l * sigmoid(g), bf16, 16-byte stores of this row.
      uint4 gv[4];
      if (valid) {
#pragma unroll
        for (int i = 0; i < 4; ++i) gv[i] = __ldg(gp + i);
      }
      if (!mbar_wait(&sm.ofull[r], c & 1, abort, a.err, kSiteOFull)) { ok = false; break; }
      tc_fence_after();
      uint4* op = reinterpret_cast<uint4*>(a.o + elem);
      for (int ch = 0; ch < 4; ++ch) {
        tmem_ld32(s_cols + 128 + ch * 32, v);
        tmem_wait_ld();
        if (ch == 3) {
          tc_fence_before();
          mbar_arrive(&sm.tfree[r]);
        }
        uint4 gn[4];
        if (valid && ch < 3) {
#pragma unroll
          for (int i = 0; i < 4; ++i) gn[i] = __ldg(gp + 4 * (ch + 1) + i);
        }
        if (valid) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float gf[8], of[8];
            unpack8(gv[i], gf);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              of[e] = __uint_as_float(v[8 * i + e]) * inv_l * sigmoid_fast(gf[e]);
            __stcs(op + 4 * ch + i, pack8(of));
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) gv[i] = gn[i];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int kPairs>
int launch_impl(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                const CUtensorMap& tg, const FwdArgs& a, int num_sms, cudaStream_t stream) {
  const size_t smem = sizeof(Smem) + 1024;
  static int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(swa_fwd_kernel<kPairs>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return map_cuda_error(e);
    configured_device = dev;
  }
  const long long grid = a.total_tiles < num_sms ? a.total_tiles : num_sms;
  swa_fwd_kernel<kPairs><<<static_cast<unsigned>(grid), kThreads, smem, stream>>>(tq, tk, tv, tg,
                                                                                 a);
  return map_cuda_error(cudaGetLastError());
}

}  // namespace fwd

int launch_fwd(const swa_params_t* p, const CUtensorMap& tq, const CUtensorMap& tk,
               const CUtensorMap& tv, const CUtensorMap& tg, const FwdArgs& a,
               cudaStream_t stream) {
  DeviceInfo di;
  int rc = current_device_info(&di);
  if (rc != SWA_OK) return rc;
  switch (p->rot_dim) {
    case 0: return fwd::launch_impl<0>(tq, tk, tv, tg, a, di.num_sms, stream);
    case 32: return fwd::launch_impl<16>(tq, tk, tv, tg, a, di.num_sms, stream);
    case 42: return fwd::launch_impl<21>(tq, tk, tv, tg, a, di.num_sms, stream);
    case 48: return fwd::launch_impl<24>(tq, tk, tv, tg, a, di.num_sms, stream);
    default: return SWA_ERR_UNSUPPORTED;
  }
}

}  // namespace swa
