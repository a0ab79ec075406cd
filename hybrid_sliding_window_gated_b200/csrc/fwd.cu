// fwd.cu -- fused prefill forward of the gated sliding-window attention core
// for sm_100a: TMA loads and stores, QK-RMSNorm and partial RoPE in shared
// memory, tcgen05 QK^T and PV with TMEM accumulators, single-pass softmax over
// the 256-key band, and the sigmoid-gate epilogue.
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
// Roles (384 threads, three warpgroups; registers rebalanced with setmaxnreg):
//   warp 0      K and Q producer (lane 0 issues TMA; all lanes compute each
//               K tile's rotation table)
//   warp 1      TMEM allocator and tcgen05.mma issuer (one lane)
//   warp 3      V producer (one lane), so a V tile that waits for its slot
//               holds up no K or Q load
//   warps 4-7   region 0 (even head slots), warps 8-11 region 1 (odd).  For
//               each of its heads a region warpgroup normalises and rotates
//               the Q rows (and the K rows of a tile whose first head it owns)
//               in place in the 128-byte-swizzled tiles, runs the softmax, and
//               finally the epilogue: it copies O out of TMEM (freeing the
//               region for the next QK^T) and writes o = O/l * sigmoid(g).
//               One thread per row throughout, so 1/rms(q) and 1/l stay in
//               registers.
//
// Q slots.  Head n uses slot n % 3 of three.  The producer loads Q(n) there
// once the o store of head n-3 has read the slot; once QK^T(n) has read Q(n),
// the slot receives the gate tile g(n) by TMA (it lands while the softmax
// runs); the epilogue overwrites it in place with o(n), which leaves by TMA
// store, and the slot goes back to the producer.  With two heads in flight the
// third slot holds the next Q, so a region never waits for its Q load.  All
// bulk global traffic (q, k, v, g in; o out) moves by TMA: the load/store
// unit touches only shared memory, since a row-per-thread pattern on global
// memory touches 32 cache lines per warp instruction.
//
// TMEM (512 columns) holds two regions of 256 columns.  For a head in region
// r: S = Q [K_{t-1} K_t]^T fills all 256 columns (fp32); the softmax writes P
// as packed bf16 over the first 128 columns; PV accumulates O (fp32) into the
// last 128 columns; the epilogue reads O.  Regions alternate between heads so
// the tensor core works on one head while the softmax runs on the other.
//
// Scores without the q norm.  s = scale * q'.k' with q' = RoPE(q/rms(q) * wq).
// The MMA multiplies q'' = [RoPE(q * wq) on the rotated dims; raw q elsewhere]
// by k'' = [RoPE(k/rms(k) * wk); k/rms(k) * wk * wq elsewhere] (wq folded into
// the unrotated dims of K, where it commutes), and the softmax applies the
// per-row factor 1/rms(q).  So Q rows only need their sum of squares and the
// rotation of the first rot_dim dims.
//
// Softmax without a max pass.  After RMSNorm every row has sum(xhat^2) <= D,
// so |q'| <= sqrt(D) max|wq| and |k'| <= sqrt(D) max|wk| (RoPE keeps norms),
// hence every score s <= M = scale * D * max|wq| * max|wk|.  exp2((s - M) log2e)
// then never overflows, and it cannot underflow while 2 M log2e <= 120 (the
// smallest possible score is -M); softmax is invariant to the subtracted
// constant, so the result equals the max-subtracted form.  Weights outside
// that range fall back to an exact two-pass (row max first) softmax.
//
// Rotation angles.  Position p = 128 j + i: the rotation by p w is the
// product of a per-tile table rot(128 j w), computed by the producer's lanes
// for each K tile (fp64 reduction of the angle as a multiple of pi, then
// sincospif), and rot(i w) for the thread's own row i, which each region
// thread keeps in registers.
//
// Code size.  The region loop runs once per head on every SM, so its
// instructions are refetched all the time; when they miss the instruction
// cache, every SM fetches from L2 while L2 is busiest.  The chunk loops of the
// softmax and the epilogue therefore stay rolled, with one register buffer.
#include <cuda_fp8.h>

#include "launch.cuh"
#include "ptx.cuh"
#include "swa_internal.h"

namespace swa {

namespace fwd {

constexpr int kThreads = 384;
// Launch budget is 384 x 168 registers; the split below sums to at most that.
constexpr int kRegsLaunch = 168;
constexpr int kRegsControl = 56;   // producer + MMA warpgroup
constexpr int kRegsRegion = 224;   // each region warpgroup
static_assert(kRegsControl + 2 * kRegsRegion <= 3 * kRegsLaunch,
              "register split exceeds the launch budget");

constexpr int kHalfBytes = kTile * 64 * 2;  // 128 rows x 64 bf16 = 16 KiB (one TMA box)
constexpr int kTileBytes = 2 * kHalfBytes;  // a full 128 x 128 bf16 tile

struct alignas(1024) Smem {
  // K ring, [half][slot]: per 64-dim half the two slots' 128 rows lie one
  // after the other, so one N = 256 MMA per k-step reads both key tiles.
  uint8_t k[2][2][kHalfBytes];
  uint8_t v[2][kTileBytes];
  uint8_t q[3][kTileBytes];  // head n uses slot n % 3: Q(n), then g(n), then o(n)
  float2 rot_tile[2][kMaxPairs];  // rot(128 j * w_p) of the K tile in each slot
  float wq[kHeadDim];
  float wk[kHeadDim];
  float sc[3];  // FP8 inputs: dequantisation factors of q, k, v
  uint64_t kfull[2], kready[2], kempty[2];
  uint64_t vfull[2], vempty[2], vready[2];  // vready: FP8 V expanded to bf16
  uint64_t qfull[3], qready[2];
  uint64_t sfull[2], pfull[2], ofull[2], tfree[2];
  uint64_t gfull[3], ostore[2];  // gate tile landed (per slot) / o written (per region)
  uint64_t slotfree[3];          // the o store has read the slot: it may take the next Q
  uint64_t drain, never;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Smem) <= 232448, "shared memory over the 227 KiB per-CTA limit");

// Wait-site ids reported through the device error word.
enum Site {
  kSiteKEmpty = 1, kSiteVEmpty, kSiteOStore, kSiteKFull, kSiteQFull, kSiteKReady,
  kSiteQReady, kSiteTFree, kSiteVFull, kSitePFull, kSiteSFull, kSiteOFull, kSiteForced,
  kSiteGFull, kSiteSlotFree, kSiteAlign
};

// Position inside a CTA's contiguous run of tiles, advanced without division.
struct Cursor {
  int b, kvh, t;  // chain (batch row, KV head) and tile index in the chain
  int h;          // query head within the GQA group
  int u;          // tiles advanced since the start of the run
};

__device__ __forceinline__ Cursor cursor_at(const FwdArgs& a, int u0) {
  Cursor c;
  const int chain = u0 / a.tiles_per_chain;
  c.t = u0 - chain * a.tiles_per_chain;
  c.b = chain / a.Hkv;
  c.kvh = chain - c.b * a.Hkv;
  c.h = 0;
  c.u = 0;
  return c;
}
__device__ __forceinline__ void next_tile(Cursor& c, const FwdArgs& a) {
  ++c.u;
  if (++c.t == a.tiles_per_chain) {
    c.t = 0;
    if (++c.kvh == a.Hkv) {
      c.kvh = 0;
      ++c.b;
    }
  }
}
__device__ __forceinline__ void next_head(Cursor& c, const FwdArgs& a) {
  if (++c.h == a.G) {
    c.h = 0;
    next_tile(c, a);
  }
}
// Key tile t-1 exists (chain tile 0 has one when the previous chunk's halo
// is given: key tile -1) / must be loaded at this tile (the first tile of a
// run, or chain tile 0 with a halo, whose ring slot held another chain's tile).
__device__ __forceinline__ bool has_prev(const Cursor& c, const FwdArgs& a) {
  return c.t > 0 || a.halo;
}
__device__ __forceinline__ bool need_prev(const Cursor& c, const FwdArgs& a) {
  return has_prev(c, a) && (c.u == 0 || c.t == 0);
}
// Last tile of the run on its chain: its K/V tile is released after use.
__device__ __forceinline__ bool seg_last(const Cursor& c, const FwdArgs& a, int n_tiles) {
  return c.u == n_tiles - 1 || c.t == a.tiles_per_chain - 1;
}

// Offset of 16-byte chunk `chunk16` of row `row` inside one 128B-swizzled
// half tile (the layout TMA SWIZZLE_128B writes): chunk c lands at c ^ (row & 7).
__device__ __forceinline__ uint32_t sw_off(int row, int chunk16) {
  return static_cast<uint32_t>(row * 128 + ((chunk16 ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint4 pack8(const float* x) {
  uint4 u;
  u.x = pack_bf16x2(x[0], x[1]);
  u.y = pack_bf16x2(x[2], x[3]);
  u.z = pack_bf16x2(x[4], x[5]);
  u.w = pack_bf16x2(x[6], x[7]);
  return u;
}

__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t u) {
  return make_float2(bf16_lo(u), bf16_hi(u));
}

__device__ __forceinline__ float2 cmul(float2 x, float2 y) {
  return make_float2(x.x * y.x - x.y * y.y, x.x * y.y + x.y * y.x);
}

// Number of rotation factors a thread keeps (at least one, so the array exists).
template <int kPairs>
struct RowRot {
  float2 r[kPairs > 0 ? kPairs : 1];  // rot(row * w_p): fixed per thread
};

// Sum of squares of a 128-element bf16 row held in two swizzled halves.
__device__ __forceinline__ float row_sumsq(const uint8_t* h0, const uint8_t* h1, int row) {
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};  // independent chains for ILP
#pragma unroll 2
  for (int c = 0; c < 8; ++c) {
    const uint4 x = *reinterpret_cast<const uint4*>(h0 + sw_off(row, c));
    const uint4 y = *reinterpret_cast<const uint4*>(h1 + sw_off(row, c));
    const uint32_t w[8] = {x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 f = bf16x2_to_f2(w[i]);
      acc[i & 3] = __ffma2_rn(f, f, acc[i & 3]);
    }
  }
  const float2 s2 = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
  return s2.x + s2.y;
}

// Rotate the first 2*kPairs dims of a row in place: y = R(x * scale * wr),
// rotate-half pairs (p, p + kPairs).  Dims of the rotated chunks beyond
// 2*kPairs are multiplied by scale * wo * wo2, or left as they are (kKeepOthers).
template <int kPairs, bool kKeepOthers>
__device__ __forceinline__ void rope_chunks(uint8_t* h0, int row, float scale, const float* wr,
                                            const float* wo, const float* wo2, const float2* rtile,
                                            const RowRot<kPairs>& rr) {
  constexpr int kRopeChunks = (2 * kPairs + 7) / 8;
  float x[kRopeChunks * 8];
#pragma unroll
  for (int c = 0; c < kRopeChunks; ++c) {
    const uint4 u = *reinterpret_cast<const uint4*>(h0 + sw_off(row, c));
    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[8 * c + 2 * e] = bf16_lo(w4[e]);
      x[8 * c + 2 * e + 1] = bf16_hi(w4[e]);
    }
  }
#pragma unroll
  for (int d = 2 * kPairs; d < kRopeChunks * 8; ++d)
    if (!kKeepOthers) x[d] = x[d] * scale * wo[d] * wo2[d];
#pragma unroll
  for (int p = 0; p < kPairs; ++p) {
    const float2 t = cmul(rtile[p], rr.r[p]);  // rot((128 j + row) w_p)
    const float u = x[p] * scale * wr[p];
    const float v = x[p + kPairs] * scale * wr[p + kPairs];
    x[p] = u * t.x - v * t.y;            // x_p cos - x_{p+P} sin
    x[p + kPairs] = v * t.x + u * t.y;   // x_{p+P} cos + x_p sin
  }
#pragma unroll
  for (int c = 0; c < kRopeChunks; ++c)
    *reinterpret_cast<uint4*>(h0 + sw_off(row, c)) = pack8(x + 8 * c);
}

// Scale dims [8*c0, 128) of a row in place by scale * w[d] * w2[d] (f32x2 math).
__device__ __forceinline__ void scale_chunks(uint8_t* h0, uint8_t* h1, int row, int c0,
                                             float scale, const float* w, const float* w2) {
  const float2 sc = make_float2(scale, scale);
#pragma unroll 1
  for (int c = c0; c < 16; ++c) {
    uint8_t* p = (c < 8 ? h0 : h1) + sw_off(row, c & 7);
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const float4 wa1 = *reinterpret_cast<const float4*>(w + 8 * c);
    const float4 wb1 = *reinterpret_cast<const float4*>(w + 8 * c + 4);
    const float4 wa2 = *reinterpret_cast<const float4*>(w2 + 8 * c);
    const float4 wb2 = *reinterpret_cast<const float4*>(w2 + 8 * c + 4);
    const float4 wa = make_float4(wa1.x * wa2.x, wa1.y * wa2.y, wa1.z * wa2.z, wa1.w * wa2.w);
    const float4 wb = make_float4(wb1.x * wb2.x, wb1.y * wb2.y, wb1.z * wb2.z, wb1.w * wb2.w);
    const float2 y0 = __fmul2_rn(__fmul2_rn(bf16x2_to_f2(u.x), make_float2(wa.x, wa.y)), sc);
    const float2 y1 = __fmul2_rn(__fmul2_rn(bf16x2_to_f2(u.y), make_float2(wa.z, wa.w)), sc);
    const float2 y2 = __fmul2_rn(__fmul2_rn(bf16x2_to_f2(u.z), make_float2(wb.x, wb.y)), sc);
    const float2 y3 = __fmul2_rn(__fmul2_rn(bf16x2_to_f2(u.w), make_float2(wb.z, wb.w)), sc);
    uint4 o;
    o.x = pack_bf16x2(y0.x, y0.y);
    o.y = pack_bf16x2(y1.x, y1.y);
    o.z = pack_bf16x2(y2.x, y2.y);
    o.w = pack_bf16x2(y3.x, y3.y);
    *reinterpret_cast<uint4*>(p) = o;
  }
}

// K row: k'' = [RoPE(k / rms(k) * wk) on the rotated dims; k / rms(k) * wk * wq
// elsewhere].
template <int kPairs>
__device__ __forceinline__ void transform_k_row(uint8_t* h0, uint8_t* h1, int row, const Smem& sm,
                                                int kslot, const RowRot<kPairs>& rr, float eps) {
  const float rinv = rsqrtf(row_sumsq(h0, h1, row) * (1.0f / kHeadDim) + eps);
  constexpr int kRopeChunks = (2 * kPairs + 7) / 8;
  if constexpr (kRopeChunks > 0)
    rope_chunks<kPairs, false>(h0, row, rinv, sm.wk, sm.wk, sm.wq, sm.rot_tile[kslot], rr);
  scale_chunks(h0, h1, row, kRopeChunks, rinv, sm.wk, sm.wq);
}

// Q row: q'' = [RoPE(q * wq) on the rotated dims; q unchanged elsewhere].
// Returns 1/rms(q), which the softmax applies to the scores.
template <int kPairs>
__device__ __forceinline__ float transform_q_row(uint8_t* tile, int row, const Smem& sm,
                                                 int kslot, const RowRot<kPairs>& rr, float eps) {
  const float rinv = rsqrtf(row_sumsq(tile, tile + kHalfBytes, row) * (1.0f / kHeadDim) + eps);
  constexpr int kRopeChunks = (2 * kPairs + 7) / 8;
  if constexpr (kRopeChunks > 0)
    rope_chunks<kPairs, true>(tile, row, 1.0f, sm.wq, sm.wq, sm.wq, sm.rot_tile[kslot], rr);
  return rinv;
}

// ------------------------------------------------------- FP8 (E4M3) inputs
//
// An FP8 tile (128 rows x 128 one-byte dims, 128B-swizzled in 16-byte chunks
// of 16 dims) is loaded by TMA into the upper half of its 32 KiB slot.  Each
// thread expands its own row into the slot's two bf16 halves: it reads the
// whole 128-byte row first, so writing half 1 (the same bytes) is safe.
// Every E4M3 value is exact in bf16, and the per-tensor factor s (x = e4m3 *
// s) folds into per-row factors, so the operands carry no rounding that the
// bf16 path does not.

// Dims 16 c .. 16 c + 15 of an FP8 row, exactly, as floats.
__device__ __forceinline__ void e4m3x16_to_f32(const uint4& u, float (&x)[16]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(
          static_cast<__nv_fp8x2_storage_t>(w[i] >> (16 * h)), __NV_E4M3);
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&r));
      x[4 * i + 2 * h] = f.x;
      x[4 * i + 2 * h + 1] = f.y;
    }
  }
}

// The FP8 row as it landed: 128 bytes in the swizzled 16 KiB box at `src`.
__device__ __forceinline__ void load_row_fp8(const uint8_t* src, int row, uint4 (&u)[8]) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    u[c] = *reinterpret_cast<const uint4*>(src + sw_off(row, c));
}

__device__ __forceinline__ float row_sumsq_fp8(const uint4 (&u)[8]) {
  float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float x[16];
    e4m3x16_to_f32(u[c], x);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 f = make_float2(x[2 * i], x[2 * i + 1]);
      acc[i & 1] = __ffma2_rn(f, f, acc[i & 1]);
    }
  }
  const float2 s2 = __fadd2_rn(acc[0], acc[1]);
  return s2.x + s2.y;
}

// Write 64 dims of a row, given as floats, as bf16 into the half at `hp`.
__device__ __forceinline__ void store_half_bf16(uint8_t* hp, int row, const float* x) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4*>(hp + sw_off(row, c)) = pack8(x + 8 * c);
}

// The factor that takes an FP8 row x8 to RMSNorm's x / rms(x) for x = s x8:
// s / sqrt(s^2 mean(x8^2) + eps).
__device__ __forceinline__ float fp8_row_factor(float sumsq8, float s, float eps) {
  return s * rsqrtf(s * s * sumsq8 * (1.0f / kHeadDim) + eps);
}

// K row from FP8: k'' as transform_k_row writes it, from x8 and the factor.
template <int kPairs>
__device__ __forceinline__ void transform_k_row_fp8(uint8_t* h0, uint8_t* h1, int row,
                                                    const Smem& sm, int kslot,
                                                    const RowRot<kPairs>& rr, float eps) {
  uint4 u[8];
  load_row_fp8(h1, row, u);  // the FP8 box lands in the second half's bytes
  const float f = fp8_row_factor(row_sumsq_fp8(u), sm.sc[1], eps);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float x[64];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float y[16];
      e4m3x16_to_f32(u[4 * h + c], y);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int d = 64 * h + 16 * c + i;
        x[16 * c + i] = d < 2 * kPairs ? y[i] * f * sm.wk[d] : y[i] * f * sm.wk[d] * sm.wq[d];
      }
    }
    if (h == 0) {
#pragma unroll
      for (int p = 0; p < kPairs; ++p) {
        const float2 t = cmul(sm.rot_tile[kslot][p], rr.r[p]);
        const float a0 = x[p], b0 = x[p + kPairs];
        x[p] = a0 * t.x - b0 * t.y;
        x[p + kPairs] = b0 * t.x + a0 * t.y;
      }
    }
    store_half_bf16(h == 0 ? h0 : h1, row, x);
  }
}

// Q row from FP8: q'' = [RoPE(x8 * wq) on the rotated dims; x8 elsewhere],
// both exact in bf16 but for the rotation; returns the row's factor, which
// the softmax applies in place of 1/rms(q).
template <int kPairs>
__device__ __forceinline__ float transform_q_row_fp8(uint8_t* tile, int row, const Smem& sm,
                                                     int kslot, const RowRot<kPairs>& rr,
                                                     float eps) {
  uint4 u[8];
  load_row_fp8(tile + kHalfBytes, row, u);
  const float f = fp8_row_factor(row_sumsq_fp8(u), sm.sc[0], eps);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float x[64];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float y[16];
      e4m3x16_to_f32(u[4 * h + c], y);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int d = 64 * h + 16 * c + i;
        x[16 * c + i] = d < 2 * kPairs ? y[i] * sm.wq[d] : y[i];
      }
    }
    if (h == 0) {
#pragma unroll
      for (int p = 0; p < kPairs; ++p) {
        const float2 t = cmul(sm.rot_tile[kslot][p], rr.r[p]);
        const float a0 = x[p], b0 = x[p + kPairs];
        x[p] = a0 * t.x - b0 * t.y;
        x[p + kPairs] = b0 * t.x + a0 * t.y;
      }
    }
    store_half_bf16(tile + h * kHalfBytes, row, x);
  }
  return f;
}

// V row from FP8: x8 exactly as bf16 (the factor s_v enters with 1/l).
__device__ __forceinline__ void expand_v_row_fp8(uint8_t* tile, int row) {
  uint4 u[8];
  load_row_fp8(tile + kHalfBytes, row, u);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float x[64];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float y[16];
      e4m3x16_to_f32(u[4 * h + c], y);
#pragma unroll
      for (int i = 0; i < 16; ++i) x[16 * c + i] = y[i];
    }
    store_half_bf16(tile + h * kHalfBytes, row, x);
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

constexpr uint32_t kIdescQK = make_idesc_bf16(128, 256, false, false);  // both key tiles at once
// K-major descriptor of k-step kk of the K ring: 256 rows (slot 0's keys,
// then slot 1's) of one 64-dim half.
__device__ __forceinline__ uint64_t desc_kring(const uint8_t (*khalf)[2][kHalfBytes], int kk) {
  return make_desc_sw128(smem_u32(khalf[kk >> 2][0]) + (kk & 3) * 32, 16, 1024);
}
constexpr uint32_t kIdescPV = make_idesc_bf16(128, 128, false, true);

// Phase bookkeeping for a 2-slot ring: bit s of `par` is the parity of the
// next use of slot s; bit s of `used` says whether slot s was used before.
struct Ring {
  uint32_t par = 0, used = 0;
  __device__ __forceinline__ uint32_t parity(int s) const { return (par >> s) & 1u; }
  __device__ __forceinline__ bool was_used(int s) const { return (used >> s) & 1u; }
  __device__ __forceinline__ void advance(int s) {
    par ^= 1u << s;
    used |= 1u << s;
  }
};

template <int kPairs, bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
    swa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                   const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ CUtensorMap tm_kh,
                   const __grid_constant__ CUtensorMap tm_vh, const FwdArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];  // 128B-swizzled tiles need 1 KiB
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  if (smem_u32(smem_raw) & 1023u) {  // the layout above assumes the alignment; never copy into it otherwise
    if (tid == 0) atomicCAS(a.err, 0, kDevErrTimeoutBase + kSiteAlign);
    return;
  }

  const int u0 = static_cast<int>(a.total_tiles * blockIdx.x / gridDim.x);
  const int u1 = static_cast<int>(a.total_tiles * (blockIdx.x + 1) / gridDim.x);
  const int n_tiles = u1 - u0;
  const int n_heads = n_tiles * a.G;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.kfull[i], 2);  // the copy's expect_tx arrive + the rotation table
      mbar_init(&sm.kready[i], 128);
      mbar_init(&sm.kempty[i], 1);
      mbar_init(&sm.vfull[i], 1);
      mbar_init(&sm.vempty[i], 1);
      mbar_init(&sm.vready[i], 128);
      mbar_init(&sm.qready[i], 128);
      mbar_init(&sm.sfull[i], 1);
      mbar_init(&sm.pfull[i], 128);
      mbar_init(&sm.ofull[i], 1);
      mbar_init(&sm.tfree[i], 128);
      mbar_init(&sm.ostore[i], 128);
    }
    for (int i = 0; i < 3; ++i) {  // per Q slot
      mbar_init(&sm.qfull[i], 1);
      mbar_init(&sm.gfull[i], 1);
      mbar_init(&sm.slotfree[i], 1);
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
    prefetch_tensormap(&tm_o);
    if (a.halo) {
      prefetch_tensormap(&tm_kh);
      prefetch_tensormap(&tm_vh);
    }
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  // Launched as a programmatic dependent of the previous kernel on the
  // stream: the set-up above overlapped its tail; every global read or write
  // below (the weights included) waits for it to complete.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid < kHeadDim) {
    const float wq = a.wq[tid], wk = a.wk[tid];
    sm.wq[tid] = wq;
    sm.wk[tid] = wk;
  }
  if (tid < 3) sm.sc[tid] = kFp8 ? a.qkv_scale[tid] : 1.0f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp < 4) {
    regs_dec<kRegsControl>();
    if (warp == 0) {
      // -------------------------------------------------- K and Q producer
      Ring kr;
      bool ok = true;
      auto wait0 = [&](uint64_t* bar, uint32_t par, int site) -> bool {
        bool w = true;
        if (lane == 0) w = mbar_wait_inl(bar, par, abort, a.err, site);
        return __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
      };
      auto load_kv = [&](bool is_k, int j, const Cursor& c) -> bool {  // K tiles only
        (void)is_k;
        const int s = j & 1;
        if (kr.was_used(s) && !wait0(&sm.kempty[s], kr.parity(s) ^ 1u, kSiteKEmpty)) return false;
        if (lane == 0) {
          if (kFp8) {  // one 16 KiB box of bytes, into the slot's upper half
            mbar_arrive_expect_tx(&sm.kfull[s], kHalfBytes);
            tma_load_4d(sm.k[1][s], &tm_k, &sm.kfull[s], 0, c.kvh, j * kTile, c.b);
          } else {
            // key tile -1: the halo's 127 rows, from row -1 (zero-filled, never in the band)
            const CUtensorMap* map = j < 0 ? &tm_kh : &tm_k;
            const int y = j < 0 ? -1 : j * kTile;
            mbar_arrive_expect_tx(&sm.kfull[s], kTileBytes);
            tma_load_4d(sm.k[0][s], map, &sm.kfull[s], 0, c.kvh, y, c.b);
            tma_load_4d(sm.k[1][s], map, &sm.kfull[s], 64, c.kvh, y, c.b);
          }
        }
        // rot(128 j w_p) for this tile, then the second arrive on kfull.
        if (lane < kPairs) {
          float cv, sv;
          rope_cos_sin(static_cast<double>(a.pos0 + static_cast<long long>(j) * kTile),
                       a.inv_freq[lane], &cv, &sv);
          sm.rot_tile[s][lane] = make_float2(cv, sv);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.kfull[s]);
        kr.advance(s);
        return true;
      };
      // Q(n) goes into slot n % 3 as soon as the o store of head n-3 has read
      // it, so each region finds its next Q already loaded.
      int nq = 0;  // Q loads issued
      Cursor c = cursor_at(a, u0);
      for (int it = 0; it < n_tiles && ok; ++it, next_tile(c, a)) {
        if (need_prev(c, a)) ok = load_kv(true, c.t - 1, c);  // first tile of a run: key tile t-1 too
        ok = ok && load_kv(true, c.t, c);
        for (int h = 0; h < a.G && ok; ++h) {
          const int qs = nq % 3;
          if (nq >= 3 && !wait0(&sm.slotfree[qs], ((nq / 3) - 1) & 1, kSiteSlotFree)) {
            ok = false;
            break;
          }
          if (lane == 0) {
            const int hq = c.kvh * a.G + h;
            if (kFp8) {
              mbar_arrive_expect_tx(&sm.qfull[qs], kHalfBytes);
              tma_load_4d(sm.q[qs] + kHalfBytes, &tm_q, &sm.qfull[qs], 0, hq, c.t * kTile, c.b);
            } else {
              mbar_arrive_expect_tx(&sm.qfull[qs], kTileBytes);
              tma_load_4d(sm.q[qs], &tm_q, &sm.qfull[qs], 0, hq, c.t * kTile, c.b);
              tma_load_4d(sm.q[qs] + kHalfBytes, &tm_q, &sm.qfull[qs], 64, hq, c.t * kTile, c.b);
            }
            tma_prefetch_4d(&tm_g, 0, hq, c.t * kTile, c.b);  // warm L2 for the gate tile
            tma_prefetch_4d(&tm_g, 64, hq, c.t * kTile, c.b);
          }
          ++nq;
        }
      }
      if (!ok && lane == 0) {
        // Drain the loads this warp issued before the CTA releases its memory.
        for (int s = 0; s < 2; ++s)
          if (kr.was_used(s)) mbar_wait_drain(&sm.kfull[s], kr.parity(s) ^ 1u);
        for (int s = 0; s < 3; ++s) {
          const int cntq = (nq - s + 2) / 3;  // Q loads into slot s
          if (cntq > 0) mbar_wait_drain(&sm.qfull[s], static_cast<uint32_t>(cntq - 1) & 1);
        }
      }
    } else if (warp == 3 && lane == 0) {
      // -------------------------------------------------------- V producer
      // Its own thread: a V tile waits for the last PV of the tile before,
      // and no K or Q load should queue behind that.
      Ring vr;
      bool ok = true;
      Cursor c = cursor_at(a, u0);
      for (int it = 0; it < n_tiles && ok; ++it, next_tile(c, a)) {
        for (int j = need_prev(c, a) ? c.t - 1 : c.t; j <= c.t && ok; ++j) {
          const int s = j & 1;
          if (vr.was_used(s) &&
              !(ok = mbar_wait_inl(&sm.vempty[s], vr.parity(s) ^ 1u, abort, a.err, kSiteVEmpty)))
            break;
          if (kFp8) {
            mbar_arrive_expect_tx(&sm.vfull[s], kHalfBytes);
            tma_load_4d(sm.v[s] + kHalfBytes, &tm_v, &sm.vfull[s], 0, c.kvh, j * kTile, c.b);
          } else {
            const CUtensorMap* map = j < 0 ? &tm_vh : &tm_v;
            const int y = j < 0 ? -1 : j * kTile;
            mbar_arrive_expect_tx(&sm.vfull[s], kTileBytes);
            tma_load_4d(sm.v[s], map, &sm.vfull[s], 0, c.kvh, y, c.b);
            tma_load_4d(sm.v[s] + kHalfBytes, map, &sm.vfull[s], 64, c.kvh, y, c.b);
          }
          vr.advance(s);
        }
      }
      if (!ok) {
        for (int s = 0; s < 2; ++s)
          if (vr.was_used(s)) mbar_wait_drain(&sm.vfull[s], vr.parity(s) ^ 1u);
      }
    } else if (warp == 1 && lane == 0) {
      // -------------------------------------------------------- MMA issuer
      Ring kr, vr;  // readiness of K (after the transform) and V slots
      bool ok = true;
      if (a.flags & SWA_FLAG_FORCE_TIMEOUT) ok = mbar_wait_inl(&sm.never, 0, abort, a.err, kSiteForced);
      Cursor cq = cursor_at(a, u0), cp = cq;
      for (int n = 0; n < n_heads && ok; n += 2) {
        // QK^T for heads n and n+1, then PV for both (regions n&1 alternate).
        for (int i = 0; i < 2 && n + i < n_heads && ok; ++i, next_head(cq, a)) {
          const int m = n + i, r = m & 1;
          const uint32_t cnt = static_cast<uint32_t>(m >> 1);
          const int sp = (cq.t + 1) & 1, sc = cq.t & 1;
          if (cq.h == 0) {
            if (need_prev(cq, a)) {
              if (!mbar_wait_inl(&sm.kready[sp], kr.parity(sp), abort, a.err, kSiteKReady)) { ok = false; break; }
              kr.advance(sp);
            }
            if (!mbar_wait_inl(&sm.kready[sc], kr.parity(sc), abort, a.err, kSiteKReady)) { ok = false; break; }
            kr.advance(sc);
          }
          if (!mbar_wait_inl(&sm.qready[r], cnt & 1, abort, a.err, kSiteQReady)) { ok = false; break; }
          if (cnt > 0 && !mbar_wait_inl(&sm.tfree[r], (cnt - 1) & 1, abort, a.err, kSiteTFree)) { ok = false; break; }
          tc_fence_after();
          const uint32_t s_base = tmem + r * 256;
          // S = Q' [K slot 0; K slot 1]^T: columns 0..127 hold the keys of the
          // tile in slot 0, 128..255 those in slot 1 (key tile t-1 and t in
          // either order; without a tile t-1 that half is never read).
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(s_base, desc_kmajor(sm.q[m % 3], kk), desc_kring(sm.k, kk), kIdescQK, kk > 0);
          mma_commit(&sm.sfull[r]);
          if (cq.h == a.G - 1) {
            if (has_prev(cq, a)) mma_commit(&sm.kempty[sp]);
            if (seg_last(cq, a, n_tiles)) mma_commit(&sm.kempty[sc]);
          }
        }
        for (int i = 0; i < 2 && n + i < n_heads && ok; ++i, next_head(cp, a)) {
          const int m = n + i, r = m & 1;
          const uint32_t cnt = static_cast<uint32_t>(m >> 1);
          const int sp = (cp.t + 1) & 1, sc = cp.t & 1;
          if (cp.h == 0) {
            // FP8 V is read once a region warpgroup has expanded it to bf16
            uint64_t* vb = kFp8 ? sm.vready : sm.vfull;
            if (need_prev(cp, a)) {
              if (!mbar_wait_inl(&vb[sp], vr.parity(sp), abort, a.err, kSiteVFull)) { ok = false; break; }
              vr.advance(sp);
            }
            if (!mbar_wait_inl(&vb[sc], vr.parity(sc), abort, a.err, kSiteVFull)) { ok = false; break; }
            vr.advance(sc);
          }
          if (!mbar_wait_inl(&sm.pfull[r], cnt & 1, abort, a.err, kSitePFull)) { ok = false; break; }
          tc_fence_after();
          const uint32_t p_base = tmem + r * 256;
          const bool hp = has_prev(cp, a);
          uint32_t acc = 0;
          for (int blk = hp ? 0 : 1; blk < 2; ++blk) {
            const int slot = blk == 0 ? sp : sc;  // P sits over the S columns of its slot
            const uint8_t* vt = sm.v[slot];
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              mma_ts(p_base + 128, p_base + slot * 64 + kk * 8, desc_v(vt, kk), kIdescPV, acc);
              acc = 1;
            }
          }
          mma_commit(&sm.ofull[r]);
          if (cp.h == a.G - 1) {
            if (hp) mma_commit(&sm.vempty[sp]);
            if (seg_last(cp, a, n_tiles)) mma_commit(&sm.vempty[sc]);
          }
        }
      }
      if (!ok) {
        // No tcgen05.mma may still be running when TMEM is released.
        mma_commit(&sm.drain);
        mbar_wait_drain(&sm.drain, 0);
      }
    }
    __syncwarp();
  } else {
    // --------------------------------------------------------------- region
    // Warpgroup r serves TMEM region r: heads n = r, r+2, ...  Per head: the
    // transform T(n) (the tile's K when this is its first head, then Q(n)),
    // the softmax S(n) once QK^T(n) is done, then the epilogue E(n) once
    // PV(n) is.
    regs_inc<kRegsRegion>();
    const int r = (warp - 4) >> 2;
    const int wq4 = warp & 3;  // TMEM lane quarter
    const int row = wq4 * 32 + lane;
    const uint32_t t_row = tmem + (static_cast<uint32_t>(wq4 * 32) << 16) + r * 256;
    // rot(row w_p): this thread's row never changes, so its factor of every
    // rotation stays in registers; the tile factor rot(128 j w_p) comes with
    // each K tile.
    RowRot<kPairs> rr;
#pragma unroll
    for (int p = 0; p < kPairs; ++p) {
      float cv, sv;
      rope_cos_sin(static_cast<double>(row), a.inv_freq[p], &cv, &sv);
      rr.r[p] = make_float2(cv, sv);
    }
    const float sl2 = a.scale_log2;
    float wmq = 0.f, wmk = 0.f;
    for (int d = 0; d < kHeadDim; ++d) {
      wmq = fmaxf(wmq, fabsf(sm.wq[d]));
      wmk = fmaxf(wmk, fabsf(sm.wk[d]));
    }
    // Score bound in log2 units, with a 1/64 margin for the bf16 rounding of q', k'.
    const float bound = sl2 * kHeadDim * wmq * wmk * (1.0f + 1.0f / 64.0f);
    const bool exact = !(2.0f * bound <= 120.0f);
    bool ok = true;

    // K loads are accounted in order by both warpgroups (the same sequence the
    // producer issues); the warpgroup that owns the first head of a tile
    // transforms that tile's K loads, right before its Q.
    Ring kr;
    int acct = 0;  // tiles accounted so far
    Cursor kc = cursor_at(a, u0);
    auto account = [&](int upto, bool transform_last) -> bool {
      while (acct <= upto) {
        for (int j = need_prev(kc, a) ? kc.t - 1 : kc.t; j <= kc.t; ++j) {
          const int s = j & 1;
          if (transform_last && acct == upto) {
            if (!mbar_wait_inl(&sm.kfull[s], kr.parity(s), abort, a.err, kSiteKFull)) return false;
            if constexpr (kFp8)
              transform_k_row_fp8<kPairs>(sm.k[0][s], sm.k[1][s], row, sm, s, rr, a.eps);
            else
              transform_k_row<kPairs>(sm.k[0][s], sm.k[1][s], row, sm, s, rr, a.eps);
            fence_proxy_async_smem();
            mbar_arrive(&sm.kready[s]);
            if constexpr (kFp8) {  // V of the same tile (vfull has the K ring's phase)
              if (!mbar_wait_inl(&sm.vfull[s], kr.parity(s), abort, a.err, kSiteVFull)) return false;
              expand_v_row_fp8(sm.v[s], row);
              fence_proxy_async_smem();
              mbar_arrive(&sm.vready[s]);
            }
          } else if (acct == upto && j == kc.t) {
            // The Q rows of this tile use its rotation table, which the
            // producer publishes with kfull.  The slot cannot be refilled
            // before every QK^T of tile t+1, which waits for this warpgroup,
            // so the phase seen here is the current one.
            if (!mbar_wait_inl(&sm.kfull[s], kr.parity(s), abort, a.err, kSiteKFull)) return false;
          }
          kr.advance(s);
        }
        next_tile(kc, a);
        ++acct;
      }
      return true;
    };
    // Row 0 of the warpgroup issues its copies through head n's slot n % 3:
    // g(n) in, o(n) out, then releases the slot to the producer.
    const bool elected = row == 0;
    // Gate copies this thread issued into each slot, and the barrier phase of
    // the last one (slots are shared by both regions), for the drain.
    int g_issued[3] = {0, 0, 0};
    uint32_t last_g_phase[3] = {0u, 0u, 0u};

    Cursor c = cursor_at(a, u0);
    if (r == 1) next_head(c, a);
    for (int n = r; n < n_heads && ok; n += 2) {
      const uint32_t cnt = static_cast<uint32_t>(n >> 1);
      const int qs = n % 3;                                   // this head's slot
      const uint32_t qph = static_cast<uint32_t>(n / 3) & 1;  // its use of that slot
      const int hq = c.kvh * a.G + c.h;
      const long long pos = static_cast<long long>(c.t) * kTile + row;

      // ---- transform T(n): the K tiles of a tile whose first head this is,
      // then Q(n).  rot_hi of slot t&1 stays valid until K_{t+2} is loaded,
      // after every QK^T of tile t+1.
      if (!account(c.u, c.h == 0)) { ok = false; break; }
      if (!mbar_wait_inl(&sm.qfull[qs], qph, abort, a.err, kSiteQFull)) { ok = false; break; }
      float rinv;
      if constexpr (kFp8)
        rinv = transform_q_row_fp8<kPairs>(sm.q[qs], row, sm, c.t & 1, rr, a.eps);
      else
        rinv = transform_q_row<kPairs>(sm.q[qs], row, sm, c.t & 1, rr, a.eps);
      fence_proxy_async_smem();
      mbar_arrive(&sm.qready[r]);


      // ---- softmax S(n)
      if (!mbar_wait_inl(&sm.sfull[r], cnt & 1, abort, a.err, kSiteSFull)) { ok = false; break; }
      tc_fence_after();
      if (elected) {  // QK^T(n) has read Q(n): the slot takes the gate tile now
        mbar_arrive_expect_tx(&sm.gfull[qs], kTileBytes);
        tma_load_4d(sm.q[qs], &tm_g, &sm.gfull[qs], 0, hq, c.t * kTile, c.b);
        tma_load_4d(sm.q[qs] + kHalfBytes, &tm_g, &sm.gfull[qs], 64, hq, c.t * kTile, c.b);
        ++g_issued[qs];
        last_g_phase[qs] = qph;
      }
      // The MMA saw unnormalised q rows; 1/rms(q) enters with the softmax scale.
      const float rs = sl2 * rinv;
      const bool hp = has_prev(c, a);
      // Key tile t sits in K slot t & 1 and key tile t-1 (logical block 0) in
      // the other: block b's S is in columns slot_of(b) * 128, its P goes over
      // columns slot_of(b) * 64.
      const int st = c.t & 1;
      auto slot_of = [&](int blk) { return blk == 1 ? st : st ^ 1; };
      float ms = bound;
      if (exact) {
        // Row maximum over the band: key tile t-1 gives columns c > row, key
        // tile t columns c <= row; pieces entirely outside the band are skipped.
        float m = -INFINITY;
#pragma unroll 1
        for (int blk = hp ? 0 : 1; blk < 2; ++blk) {
#pragma unroll 1
          for (int pc = 0; pc < 4; ++pc) {
            const bool none = blk == 0 ? (pc < wq4) : (pc > wq4);
            if (none) continue;
            uint32_t v[32];
            tmem_ld32(t_row + slot_of(blk) * 128 + pc * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const bool in = blk == 0 ? (pc * 32 + i > row) : (pc * 32 + i <= row);
              if (in) m = fmaxf(m, __uint_as_float(v[i]));
            }
          }
        }
        ms = m * rs;
      }
      // P = exp2(s * rs - ms), packed bf16 over the first 128 columns of the
      // region; fp32 row sum.  Key tile t-1 keeps columns c > row, key tile t
      // columns c <= row.  For this warp's 32 rows, 32-column chunk pc of key
      // tile t-1 is empty for pc < wq4 and full for pc > wq4; of key tile t
      // full for pc < wq4 and empty for pc > wq4; only pc == wq4 straddles
      // the band edge.  The tile in slot 0 is taken first: the other tile's
      // P lands over S columns 64..127 of slot 0, which must be read by then.
      const int na = hp ? 4 - wq4 : 0;  // chunks of key tile t-1 in the band
      const int nt = wq4 + 1;           // chunks of key tile t
      const int nch = na + nt;
      const int b_first = st == 0 ? 1 : 0;  // the logical tile in slot 0
      const int n_first = b_first == 0 ? na : nt;
      float2 l2 = make_float2(0.f, 0.f);
      const float2 rs2 = make_float2(rs, rs), nms2 = make_float2(-ms, -ms);
      {
        // Chunk i of the band: 32 columns of S in, 16 columns of packed P out.
        // Loops stay rolled (two chunk bodies per variant): the region code
        // is refetched by every head, so its size decides instruction-cache
        // hits.
        auto chunk_blk = [&](int i) { return i < n_first ? b_first : 1 - b_first; };
        auto chunk_pc = [&](int i) {
          const int k = i < n_first ? i : i - n_first;
          return chunk_blk(i) == 0 ? wq4 + k : k;
        };
        auto chunk_col = [&](int i) { return slot_of(chunk_blk(i)) * 128 + chunk_pc(i) * 32; };
        auto chunk = [&](const uint32_t(&x)[32], int i) {
          const int blk = chunk_blk(i);
          const int pc = chunk_pc(i);
          uint32_t pk[16];
          if (pc != wq4) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float2 z = __ffma2_rn(
                  make_float2(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1])), rs2, nms2);
              const float2 p = make_float2(ex2_approx(z.x), ex2_approx(z.y));
              l2 = __fadd2_rn(l2, p);
              pk[e] = pack_bf16x2(p.x, p.y);
            }
          } else {  // the diagonal chunk: mask per column
            const int c0 = pc * 32;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int cc = c0 + 2 * e;
              const bool in0 = blk == 0 ? (cc > row) : (cc <= row);
              const bool in1 = blk == 0 ? (cc + 1 > row) : (cc + 1 <= row);
              const float2 z = __ffma2_rn(
                  make_float2(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1])), rs2, nms2);
              const float2 p =
                  make_float2(in0 ? ex2_approx(z.x) : 0.f, in1 ? ex2_approx(z.y) : 0.f);
              l2 = __fadd2_rn(l2, p);
              pk[e] = pack_bf16x2(p.x, p.y);
            }
          }
          tmem_st16(t_row + slot_of(blk) * 64 + pc * 16, pk);
        };
        // One register buffer: while a warp waits for its chunk, the SM runs
        // the other warps; the smaller loop keeps the region code in cache.
#pragma unroll 1
        for (int i = 0; i < nch; ++i) {
          uint32_t va[32];
          tmem_ld32(t_row + chunk_col(i), va);
          tmem_wait_ld();
          chunk(va, i);
        }
      }
      {
        // Zero the empty chunks last: P columns alias S columns that the
        // chunks above still had to read.
        const uint32_t zero16[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u,
                                     0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        for (int pc = 0; pc < 4; ++pc) {
          if (hp && pc < wq4) tmem_st16(t_row + slot_of(0) * 64 + pc * 16, zero16);
          if (pc > wq4) tmem_st16(t_row + slot_of(1) * 64 + pc * 16, zero16);
        }
      }
      const float l = l2.x + l2.y;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.pfull[r]);
      if (a.lse != nullptr && pos < a.T)
        a.lse[(static_cast<long long>(c.b) * a.Hq + hq) * a.T + pos] =
            (ms + __log2f(l)) * 0.6931471805599453f;

      // ---- epilogue E(n): o = A/l * sigmoid(g), written over g(n) in Q slot r,
      // 32 columns per step.
      if (!mbar_wait_inl(&sm.ofull[r], cnt & 1, abort, a.err, kSiteOFull)) { ok = false; break; }
      if (!mbar_wait_inl(&sm.gfull[qs], qph, abort, a.err, kSiteGFull)) { ok = false; break; }
      tc_fence_after();
      const float il = sm.sc[2] / l;  // FP8 V: its factor s_v enters here
      const float2 il2 = make_float2(il, il);
      {
        // Chunk ch: 32 columns of O, written over the same columns of g.
        auto gate = [&](const uint32_t(&ov)[32], int ch) {
          uint8_t* half = sm.q[qs] + (ch >> 1) * kHalfBytes;
#pragma unroll
          for (int i = 0; i < 4; ++i) {  // four 16-byte pieces of this chunk
            uint4* gp = reinterpret_cast<uint4*>(half + sw_off(row, (ch & 1) * 4 + i));
            const uint4 gv = *gp;
            const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
            uint32_t ow[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 sg = sigmoid2(bf16x2_to_f2(gw[e]));
              const float2 acc = __fmul2_rn(make_float2(__uint_as_float(ov[8 * i + 2 * e]),
                                                        __uint_as_float(ov[8 * i + 2 * e + 1])),
                                            il2);
              const float2 o2 = __fmul2_rn(acc, sg);
              ow[e] = pack_bf16x2(o2.x, o2.y);
            }
            *gp = make_uint4(ow[0], ow[1], ow[2], ow[3]);
          }
        };
#pragma unroll 1
        for (int ch = 0; ch < kHeadDim / 32; ++ch) {
          uint32_t oa[32];
          tmem_ld32(t_row + 128 + ch * 32, oa);
          tmem_wait_ld();
          if (ch + 1 == kHeadDim / 32) {
            tc_fence_before();
            mbar_arrive(&sm.tfree[r]);  // region r may take the next QK^T now
          }
          gate(oa, ch);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&sm.ostore[r]);

      Cursor cn = c;
      next_head(cn, a);
      next_head(cn, a);
      if (elected) {
        // o(n) out of the slot (rows past T are clipped by the copy); once the
        // store has read it the slot goes back to the producer.
        if (!mbar_wait_inl(&sm.ostore[r], cnt & 1, abort, a.err, kSiteOStore)) { ok = false; break; }
        tma_store_4d(&tm_o, sm.q[qs], 0, hq, c.t * kTile, c.b);
        tma_store_4d(&tm_o, sm.q[qs] + kHalfBytes, 64, hq, c.t * kTile, c.b);
        bulk_commit();
        bulk_wait_read<0>();
        mbar_arrive(&sm.slotfree[qs]);
      }
      c = cn;
    }
    if (elected) {
      if (!ok) {
        // Drain this thread's loads before the CTA releases its memory.
        for (int s2 = 0; s2 < 3; ++s2)
          if (g_issued[s2] > 0) mbar_wait_drain(&sm.gfull[s2], last_g_phase[s2]);
      }
      bulk_wait_all();  // every store complete before the CTA exits
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int kPairs, bool kFp8>
int launch_impl(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                const CUtensorMap& tg, const CUtensorMap& to, const CUtensorMap& tkh,
                const CUtensorMap& tvh, const FwdArgs& a, int num_sms, cudaStream_t stream) {
  const size_t smem = sizeof(Smem);
  static int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    // The register split (setmaxnreg) assumes the kernel was built with the
    // full launch budget per thread; refuse to launch otherwise.
    cudaFuncAttributes attr;
    cudaError_t e = cudaFuncGetAttributes(&attr, swa_fwd_kernel<kPairs, kFp8>);
    if (e != cudaSuccess) return map_cuda_error(e);
    if (attr.numRegs != kRegsLaunch) return SWA_ERR_UNSUPPORTED;
    e = cudaFuncSetAttribute(swa_fwd_kernel<kPairs, kFp8>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return map_cuda_error(e);
    configured_device = dev;
  }
  const long long grid = a.total_tiles < num_sms ? a.total_tiles : num_sms;
  return launch_dependent(swa_fwd_kernel<kPairs, kFp8>, static_cast<unsigned>(grid), kThreads,
                          smem, stream, tq, tk, tv, tg, to, tkh, tvh, a);
}

template <bool kFp8>
int launch_rot(int rot_dim, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
               const CUtensorMap& tg, const CUtensorMap& to, const CUtensorMap& tkh,
               const CUtensorMap& tvh, const FwdArgs& a, int num_sms, cudaStream_t stream) {
  switch (rot_dim) {
    case 0: return launch_impl<0, kFp8>(tq, tk, tv, tg, to, tkh, tvh, a, num_sms, stream);
    case 32: return launch_impl<16, kFp8>(tq, tk, tv, tg, to, tkh, tvh, a, num_sms, stream);
    case 42: return launch_impl<21, kFp8>(tq, tk, tv, tg, to, tkh, tvh, a, num_sms, stream);
    case 48: return launch_impl<24, kFp8>(tq, tk, tv, tg, to, tkh, tvh, a, num_sms, stream);
    default: return SWA_ERR_UNSUPPORTED;
  }
}

}  // namespace fwd

int launch_fwd(const swa_params_t* p, const CUtensorMap& tq, const CUtensorMap& tk,
               const CUtensorMap& tv, const CUtensorMap& tg, const CUtensorMap& to,
               const CUtensorMap& tkh, const CUtensorMap& tvh, const FwdArgs& a,
               cudaStream_t stream) {
  DeviceInfo di;
  int rc = current_device_info(&di);
  if (rc != SWA_OK) return rc;
  if (a.total_tiles > (1ll << 30)) return SWA_ERR_UNSUPPORTED;
  if (a.qkv_scale != nullptr && a.halo) return SWA_ERR_UNSUPPORTED;  // FP8 takes no halo
  return a.qkv_scale != nullptr
             ? fwd::launch_rot<true>(p->rot_dim, tq, tk, tv, tg, to, tkh, tvh, a, di.num_sms,
                                     stream)
             : fwd::launch_rot<false>(p->rot_dim, tq, tk, tv, tg, to, tkh, tvh, a, di.num_sms,
                                      stream);
}

}  // namespace swa
