// bwd.cu -- backward of the gated sliding-window attention core for sm_100a.
//
// Forward (ZGCM-1 pages: onedev.kr summary, "어떻게 동작하나"; jaehun.me review,
// "How Gated SWA Behaves"): q' = RoPE(RMSNorm(q; wq)), k' = RoPE(RMSNorm(k; wk)),
// s_ij = scale q'_i.k'_j on the band j in [i-127, i], P = softmax(s), A = P V,
// O = A (*) sigmoid(g).  Given dO and the forward's lse, the chain rule gives
//   dg = dO (*) A (*) sig (1 - sig),   dA = dO (*) sig,   D_i = dA_i . A_i,
//   dP = dA V^T,   dS = scale P (*) (dP - D),
//   dq' = dS k',   dk' = dS^T q',   dv = P^T dA,
// then RoPE^-1 (rotation by -theta) and the RMSNorm Jacobian
//   dx = (w (*) dy - xhat mean(xhat (*) w (*) dy)) / r,   dw += dy (*) xhat.
//
// Two kernels, both on the tensor cores with TMEM accumulators:
//   swa_bwd_q_kernel (query-major, one 128-row query tile and head at a time,
//     key tiles t-1 and t resident): recomputes S and P (from lse) and
//     A = P V, writes dg and the workspace rows dA (fp16) and D (fp32), then
//     dP = dA V^T, dS per key tile into shared memory, dQ = dS K' and dq.
//   swa_bwd_kv_kernel (key-major, one key tile at a time, query tiles j and
//     j+1 and every head of the group): S^T = K' Q'^T and dP^T = V dA^T,
//     P^T and dS^T packed in TMEM, dV += P^T dA and dK += dS^T Q' accumulated
//     in TMEM across the 2G (query tile, head) pairs, then dk and dv.
// Every dq row and every dk/dv row is complete inside one CTA: no atomics
// except the per-CTA sums of dwq and dwk.
//
// Roles: warp 0 TMA producer (its lanes also compute rotation tables), warp 1
// TMEM allocator and MMA issuer, and in the query-major pass warps 2-3 the Q
// transform, a head ahead; both passes run 384 threads with registers
// rebalanced by setmaxnreg and two compute warpgroups, warps 4-7 and 8-11,
// thread r of each on tile row r.  In the query-major pass they share every
// row: each takes half of the row's columns and they exchange the row sums
// through shared memory.  In the key-major pass the (query tile, head) pairs
// alternate between them, so that one transforms the next pair's Q while the
// other turns the current pair's S^T and dP^T into P^T and dS^T; the dk and dv
// rows are split by halves.  Waits are bounded as in the forward (inlined:
// ptxas places no calls under setmaxnreg).
#include <cuda_fp16.h>

#include "bwd_internal.h"
#include "launch.cuh"
#include "ptx.cuh"

namespace swa {
namespace bwd {

// Both passes: a control warpgroup and two compute warpgroups, launch budget
// 384 x 168 registers, rebalanced with setmaxnreg between them.
constexpr int kThreads = 384;
constexpr int kRegsLaunch = 168;
constexpr int kRegsControl = 56;
constexpr int kRegsCompute = 224;
static_assert(kRegsControl + 2 * kRegsCompute <= 3 * kRegsLaunch, "register split");
constexpr int kHalfBytes = kTile * 64 * 2;  // 128 rows x 64 bf16 (one TMA box)
constexpr int kTileBytes = 2 * kHalfBytes;
constexpr float kLog2e = 1.4426950408889634f;

enum Site {
  kSiteKFull = 0x60, kSiteKEmpty, kSiteVFull, kSiteVEmpty, kSiteQFull, kSiteQEmpty, kSiteQReady,
  kSiteKReady, kSiteSFull, kSitePFull, kSiteAFull, kSiteDAFull, kSiteDPFull, kSiteDSFull,
  kSiteDQ0, kSiteDQFull, kSiteTFree, kSiteTables, kSiteDKVFull, kSiteKVEmpty, kSiteStaged,
  kSiteMmaDone, kSiteForced, kSiteXchg, kSiteKVReady, kSiteVReady
};

// ---------------------------------------------------------------- helpers

// Offset of 16-byte chunk `c` (0..7) of row `row` in a 128B-swizzled half tile.
__device__ __forceinline__ uint32_t sw_off(int row, int c) {
  return static_cast<uint32_t>(row * 128 + ((c ^ (row & 7)) << 4));
}
__device__ __forceinline__ float2 bf2(uint32_t u) { return make_float2(bf16_lo(u), bf16_hi(u)); }
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ float2 f16x2(uint32_t u) {
  return __half22float2(*reinterpret_cast<const __half2*>(&u));
}
// 32 bytes of one row per thread in one access (rows are 32-byte aligned):
// a warp's row-per-thread access then touches each 32-byte sector once.  The
// rows stream through once, so loads and stores both skip L1: with the
// shared memory these kernels take, L1 keeps about 28 KB, which the register
// spills need.
__device__ __forceinline__ void ld32B(const void* p, uint32_t (&r)[8]) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "l"(p));
}
__device__ __forceinline__ void st32B(void* p, const uint32_t (&r)[8]) {
  asm volatile("st.global.L1::no_allocate.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(r[0]), "r"(r[1]),
               "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// bf16 magnitude bits of the largest value the fp16 staging of V carries:
// 0x477F is 65280, and the next bf16 value, 65536, is past the fp16 maximum.
constexpr uint32_t kF16MaxBits = 0x477Fu;

// Row `row` of a [128 x 128] bf16 tile (two 128-byte-row halves) converted to
// fp16 in place: every backward contraction runs fp16 x fp16, three more
// mantissa bits than bf16.  Returns the row's largest magnitude as bf16 bits
// (NaN compares above every finite value).
// `hs` is the distance between the tile's two halves (the query-major pass
// keeps its two key tiles interleaved by half).
__device__ __forceinline__ uint32_t row_to_f16(uint8_t* tile, int row, int hs = kHalfBytes) {
  uint32_t m = 0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      // chunk c of the row in its swizzled place: the 32 rows of a warp then
      // spread over all banks (row-linear order would put every lane's access
      // in the same four)
      uint4* p = reinterpret_cast<uint4*>(tile + h * hs + sw_off(row, c));
      const uint4 u = *p;
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        m = __vmaxu2(m, w[e] & 0x7FFF7FFFu);
        const float2 f = bf2(w[e]);
        o[e] = pack_f16x2(f.x, f.y);
      }
      *p = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  return max(m & 0xFFFFu, m >> 16);
}

// Scale exponents of the fp16 staging.  Every exponent lies in
// [-kExpLimit, kExpLimit], so a sum of two is still a normal fp32 power of two.
constexpr int kExpLimit = 62;
__device__ __forceinline__ float pow2f(int e) {  // 2^e for e in [-126, 127]
  return __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
}
// Exponent e of a row of dA: 2^e max|dO| lies in [1, 2), so dA 2^e (|dA| <=
// |dO|) keeps fp16's full precision whatever the gradient's scale.  `m` is
// max|dO| as bf16 magnitude bits; an all-zero row takes the largest exponent,
// which leaves every minimum over rows to the rows that carry a gradient.
__device__ __forceinline__ int row_exponent(uint32_t m) {
  const int E = static_cast<int>(m >> 7);  // biased bf16 exponent
  if (E == 0) return kExpLimit;
  return max(-kExpLimit, min(kExpLimit, 127 - E));
}
// Exponent k of dS for a query tile whose keys' values satisfy |v| <= vmax.
// With |dA 2^e| <= 2: |dP| <= 2 D vmax and |D_i| <= 2 D vmax (A_i is a convex
// combination of v rows), so |dS 2^(e+k)| <= scale 4 D vmax 2^k <= 2^15:
// inside fp16's range by construction, and values of typical size land near
// 1 rather than among fp16's subnormals when v is small.
__device__ __forceinline__ int ds_exponent(float scale, uint32_t vmax_bits) {
  const float bound = scale * (4.0f * kHeadDim) * __uint_as_float(vmax_bits << 16);
  const uint32_t Eb = (__float_as_uint(bound) >> 23) & 0xFFu;
  if (!(bound > 0.0f) || Eb == 0xFFu) return 0;  // zero, NaN or inf
  if (Eb == 0) return kExpLimit;
  return max(-kExpLimit, min(kExpLimit, 141 - static_cast<int>(Eb)));  // bound < 2^(Eb-126)
}
// Largest bf16 exponent field of dO the staging takes (|dO| < 2^63); beyond
// it, short of inf or NaN, the call reports kDevErrRange.
constexpr int kMaxDoExpField = 127 + kExpLimit;
__device__ __forceinline__ float2 cmul(float2 x, float2 y) {
  return make_float2(x.x * y.x - x.y * y.y, x.x * y.y + x.y * y.x);
}

// A bounded wait whose outcome is the same on every lane of the warp, so the
// warp-collective tcgen05 loads and stores that follow never run divergent.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int* err, int site) {
  return __all_sync(0xffffffffu, mbar_wait_inl(bar, parity, abort, err, site));
}

struct RotTables {
  float2 lo[kMaxPairs][16];  // rot(b w_p), b = 0..15
};

// Rotation of position 128 j + row for pair p: hi[p][row/16] is rot((128 j +
// 16 a) w_p) for the tile, lo the per-CTA table.
__device__ __forceinline__ float2 rot_at(const float2 (*hi)[8], const RotTables& t, int p, int row) {
  return cmul(hi[p][row >> 4], t.lo[p][row & 15]);
}

__device__ __forceinline__ float row_sumsq(const uint8_t* tile, int row, int hs = kHalfBytes) {
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 x = *reinterpret_cast<const uint4*>(tile + sw_off(row, c));
    const uint4 y = *reinterpret_cast<const uint4*>(tile + hs + sw_off(row, c));
    const uint32_t w[8] = {x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 f = bf2(w[i]);
      acc[i & 3] = __ffma2_rn(f, f, acc[i & 3]);
    }
  }
  const float2 s = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
  return s.x + s.y;
}

// In place: bf16 row <- RoPE(row / rms(row) * w) as fp16 (the true normalised,
// rotated operand; fp16 keeps 3 more mantissa bits than bf16 for the score and
// gradient contractions whose operands are all computed here).  Returns 1/rms.
template <int kPairs>
__device__ __forceinline__ float norm_rope_row(uint8_t* tile, int row, const float* w,
                                               const float2 (*hi)[8], const RotTables& t,
                                               float eps, int hs = kHalfBytes) {
  const float rinv = rsqrtf(row_sumsq(tile, row, hs) * (1.0f / kHeadDim) + eps);
  float x[kHeadDim / 2];  // the first half (dims 0..63): it holds every rotated pair
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 u = *reinterpret_cast<const uint4*>(tile + sw_off(row, c));
    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[8 * c + 2 * e] = bf16_lo(w4[e]) * rinv * w[8 * c + 2 * e];
      x[8 * c + 2 * e + 1] = bf16_hi(w4[e]) * rinv * w[8 * c + 2 * e + 1];
    }
  }
#pragma unroll
  for (int p = 0; p < kPairs; ++p) {
    const float2 r = rot_at(hi, t, p, row);
    const float a = x[p], b = x[p + kPairs];
    x[p] = a * r.x - b * r.y;
    x[p + kPairs] = b * r.x + a * r.y;
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 u;
    u.x = pack_f16x2(x[8 * c], x[8 * c + 1]);
    u.y = pack_f16x2(x[8 * c + 2], x[8 * c + 3]);
    u.z = pack_f16x2(x[8 * c + 4], x[8 * c + 5]);
    u.w = pack_f16x2(x[8 * c + 6], x[8 * c + 7]);
    *reinterpret_cast<uint4*>(tile + sw_off(row, c)) = u;
  }
  uint8_t* h1 = tile + hs;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 u = *reinterpret_cast<const uint4*>(h1 + sw_off(row, c));
    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
    uint32_t o4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int d = 64 + 8 * c + 2 * e;
      o4[e] = pack_f16x2(bf16_lo(w4[e]) * rinv * w[d], bf16_hi(w4[e]) * rinv * w[d + 1]);
    }
    *reinterpret_cast<uint4*>(h1 + sw_off(row, c)) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
  }
  return rinv;
}

// Dim d of row `row` in a [128 x 128] 16-bit tile (two halves, 128B swizzle).
__device__ __forceinline__ uint16_t* tile_elem(uint8_t* tile, int row, int d) {
  return reinterpret_cast<uint16_t*>(tile + (d >> 6) * kHalfBytes + sw_off(row, (d >> 3) & 7) +
                                     (d & 7) * 2);
}
__device__ __forceinline__ uint16_t f16_bits(float x) {
  return static_cast<uint16_t>(pack_f16x2(x, 0.f) & 0xFFFFu);
}

// norm_rope_row for warps with few registers: the same operand, with each
// rotated pair (p, p + kPairs) taken on its own and the rest of the row by
// 16-byte chunks.  Every value is read once before it is rewritten.
template <int kPairs>
__device__ __forceinline__ float norm_rope_row_lean(uint8_t* tile, int row, const float* w,
                                                    const float2 (*hi)[8], const RotTables& t,
                                                    float eps) {
  const float rinv = rsqrtf(row_sumsq(tile, row) * (1.0f / kHeadDim) + eps);
#pragma unroll 1
  for (int p = 0; p < kPairs; ++p) {
    uint16_t* pa = tile_elem(tile, row, p);
    uint16_t* pb = tile_elem(tile, row, p + kPairs);
    const float a = bf16_lo(*pa) * rinv * w[p];
    const float b = bf16_lo(*pb) * rinv * w[p + kPairs];
    const float2 r = rot_at(hi, t, p, row);
    *pa = f16_bits(a * r.x - b * r.y);
    *pb = f16_bits(b * r.x + a * r.y);
  }
  constexpr int kFirstChunk = (2 * kPairs + 7) / 8;  // the first chunk with no rotated dim
#pragma unroll 1
  for (int d = 2 * kPairs; d < 8 * kFirstChunk; ++d) {
    uint16_t* pd = tile_elem(tile, row, d);
    *pd = f16_bits(bf16_lo(*pd) * rinv * w[d]);
  }
#pragma unroll 1
  for (int c = kFirstChunk; c < 16; ++c) {
    uint4* pc = reinterpret_cast<uint4*>(tile + (c >> 3) * kHalfBytes + sw_off(row, c & 7));
    const uint4 u = *pc;
    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
    uint32_t o4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int d = 8 * c + 2 * e;
      o4[e] = pack_f16x2(bf16_lo(w4[e]) * rinv * w[d], bf16_hi(w4[e]) * rinv * w[d + 1]);
    }
    *pc = make_uint4(o4[0], o4[1], o4[2], o4[3]);
  }
  return rinv;
}

// Sum a 64-value per-thread vector over the warp; lane l gets dims 2l, 2l+1.
__device__ __forceinline__ float2 warp_reduce_scatter64(float (&v)[64], int lane) {
#pragma unroll
  for (int m = 16, n = 32; m >= 1; m >>= 1, n >>= 1) {
    const bool up = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < n; ++i) {
      const float keep = up ? v[n + i] : v[i];
      const float send = up ? v[i] : v[n + i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
    }
  }
  return make_float2(v[0], v[1]);
}

__device__ __forceinline__ uint64_t desc_kmajor(const uint8_t* tile, int kk) {
  return desc_advance(make_desc_sw128(smem_u32(tile), 16, 1024), (kk >> 2) * kHalfBytes + (kk & 3) * 32);
}
__device__ __forceinline__ uint64_t desc_mn(const uint8_t* tile, int kk) {
  return desc_advance(make_desc_sw128(smem_u32(tile), kHalfBytes, 1024), kk * 2048);
}
// One dA tile of the workspace, which is tile-major: [B, Hq, tiles] tiles of
// 128 rows x 128 fp16 in the swizzled MMA operand layout, 32 KiB each, so the
// query-major pass stores and the key-major pass loads a tile in one copy.
__device__ __forceinline__ uint16_t* da_tile(const BwdArgs& a, int b, int hq, int t) {
  return a.ws_da + ((static_cast<long long>(b) * a.Hq + hq) * a.tiles_per_chain + t) *
                       (kTileBytes / 2);
}
// 1-D bulk copies (16-byte aligned, sizes multiples of 16).
__device__ __forceinline__ void bulk_store(void* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
               "r"(smem_u32(ssrc)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_load(void* sdst, const void* gsrc, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(sdst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// K-major descriptor of k-step kk over both slots of a ring (256 rows).
__device__ __forceinline__ uint64_t desc_ring(const uint8_t (*ring)[2][kHalfBytes], int kk) {
  return desc_advance(make_desc_sw128(smem_u32(ring[kk >> 2][0]), 16, 1024), (kk & 3) * 32);
}
// K-major descriptor of one slot of a ring (128 rows) for k-step kk.
__device__ __forceinline__ uint64_t desc_ring_slot(const uint8_t (*ring)[2][kHalfBytes], int slot,
                                                   int kk) {
  return desc_advance(make_desc_sw128(smem_u32(ring[kk >> 2][slot]), 16, 1024), (kk & 3) * 32);
}
// MN-major descriptor of one slot of a ring for k-step kk (its halves 32 KiB apart).
__device__ __forceinline__ uint64_t desc_mn_ring(const uint8_t (*ring)[2][kHalfBytes], int slot,
                                                 int kk) {
  return desc_advance(make_desc_sw128(smem_u32(ring[0][slot]), 2 * kHalfBytes, 1024), kk * 2048);
}
constexpr uint32_t kIdescKK = make_idesc_bf16(128, 128, false, false);  // A, B K-major
constexpr uint32_t kIdescKM = make_idesc_bf16(128, 128, false, true);   // B MN-major
// The same shapes with fp16 A and B (format fields 0): Q', K' and dS operands.
constexpr uint32_t kF16 = ~((1u << 7) | (1u << 10));
constexpr uint32_t kIdescKK16 = kIdescKK & kF16;
constexpr uint32_t kIdescKM16 = kIdescKM & kF16;
constexpr uint32_t kIdescKK16x256 = make_idesc_bf16(128, 256, false, false) & kF16;  // both key tiles
// fp16 holds the normalised operands while max|w| * sqrt(head_dim) stays well
// inside its range; larger weights are refused (device error code below).
constexpr float kMaxWeight = 4096.0f;

// Contiguous per-CTA ranges of tiles over (batch row, KV head, tile).
struct Cursor {
  int b, kvh, t, u;
};
__device__ __forceinline__ Cursor cursor_at(const BwdArgs& a, int u0) {
  Cursor c;
  const int chain = u0 / a.tiles_per_chain;
  c.t = u0 - chain * a.tiles_per_chain;
  c.b = chain / a.Hkv;
  c.kvh = chain - c.b * a.Hkv;
  c.u = 0;
  return c;
}
__device__ __forceinline__ void next_tile(Cursor& c, const BwdArgs& a) {
  ++c.u;
  if (++c.t == a.tiles_per_chain) {
    c.t = 0;
    if (++c.kvh == a.Hkv) {
      c.kvh = 0;
      ++c.b;
    }
  }
}
// Key tile t-1 exists (chain tile 0 has one with a halo: key tile -1) / must
// be loaded (the first tile of a run, or chain tile 0 with a halo).
__device__ __forceinline__ bool has_prev(const Cursor& c, const BwdArgs& a) {
  return c.t > 0 || a.halo;
}
__device__ __forceinline__ bool need_prev(const Cursor& c, const BwdArgs& a) {
  return has_prev(c, a) && (c.u == 0 || c.t == 0);
}
// The key-major pass walks key tiles -halo .. tiles-1 of each chain.
__device__ __forceinline__ Cursor cursor_at_kv(const BwdArgs& a, int u0) {
  Cursor c;
  const int chain = u0 / a.kv_tiles;
  c.t = u0 - chain * a.kv_tiles - a.halo;
  c.b = chain / a.Hkv;
  c.kvh = chain - c.b * a.Hkv;
  c.u = 0;
  return c;
}
__device__ __forceinline__ void next_tile_kv(Cursor& c, const BwdArgs& a) {
  ++c.u;
  if (++c.t == a.tiles_per_chain) {
    c.t = -a.halo;
    if (++c.kvh == a.Hkv) {
      c.kvh = 0;
      ++c.b;
    }
  }
}
// TMA of key tile j of a chain: tile -1 is the halo's rows from row -1 (that
// row zero-filled and never in the band).
__device__ __forceinline__ void load_key_tile(uint8_t* dst, const CUtensorMap* map,
                                              const CUtensorMap* map_halo, uint64_t* bar, int j,
                                              int kvh, int b, int hs = kHalfBytes) {
  const CUtensorMap* m = j < 0 ? map_halo : map;
  const int y = j < 0 ? -1 : j * kTile;
  tma_load_4d(dst, m, bar, 0, kvh, y, b);
  tma_load_4d(dst + hs, m, bar, 64, kvh, y, b);
}

// Rotation table rot((128 j + 16 a) w_p), a = 0..7, computed by a warp.
template <int kPairs>
__device__ __forceinline__ void fill_rot_hi(float2 (*hi)[8], int j, const BwdArgs& a, int lane) {
  for (int e = lane; e < kPairs * 8; e += 32) {
    const int p = e >> 3, ai = e & 7;
    float cv, sv;
    rope_cos_sin(static_cast<double>(a.pos0 + static_cast<long long>(j) * kTile) + 16.0 * ai,
                 a.inv_freq[p], &cv, &sv);
    hi[p][ai] = make_float2(cv, sv);
  }
}

// ===================================================== pass 1: query-major

struct alignas(1024) SmemQ {
  // K and V rings, [half][slot]: per 64-dim half the two slots' 128 rows lie
  // one after the other, so one N = 256 MMA reads both key tiles.
  uint8_t k[2][2][kHalfBytes];
  uint8_t v[2][2][kHalfBytes];
  // Head n works in slot n & 1: Q', then dA, then dS of each key tile, each
  // written once the MMA reading its predecessor is done; the other slot
  // receives Q of head n+1 meanwhile.
  uint8_t slot[2][kTileBytes];
  RotTables rot;
  float2 rot_hi[2][kMaxPairs][8];  // per K slot
  float2 qrot_hi[kMaxPairs][8];    // the Q transform's (each of its warps fills its rows' entries)
  float wq[kHeadDim], wk[kHeadDim], dw[kHeadDim];
  uint64_t kfull[2], kready[2], kempty[2], vfull[2], vready[2], vempty[2];
  uint64_t qfull[2], qempty[2];
  uint64_t qready[2];  // per Q slot
  uint64_t sfull, pfull, afull, dafull, dpfull, dsfull, dq0, dqfull;
  uint64_t tables, drain, never;  // never: completed by nothing (forced timeouts)
  // Row-sum exchanges between the two compute warpgroups (l with the dA row
  // exponent, D, the dq dot).
  uint64_t xlb, xdb, xtb;
  float xl[2][kTile], xd[2][kTile], xt[2][kTile];
  int xe[2][kTile];     // each half row's dA exponent (exchanged with l)
  int xew[2][2][4];     // [head parity][warpgroup][warp]: minimum of those exponents
  uint32_t vmax[2][4];  // per V slot and converting warp: largest |v| (bf16 bits)
  float rinvq[3][kTile];  // 1/rms of each Q row, head n in n % 3
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(SmemQ) + 1024 <= 232448, "pass 1 shared memory");

template <int kPairs>
__global__ void __launch_bounds__(kThreads, 1)
    swa_bwd_q_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_kh,
                     const __grid_constant__ CUtensorMap tm_vh, const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  SmemQ& sm = *reinterpret_cast<SmemQ*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                        ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u0 = static_cast<int>(a.total_tiles * blockIdx.x / gridDim.x);
  const int u1 = static_cast<int>(a.total_tiles * (blockIdx.x + 1) / gridDim.x);
  int n_tiles = u1 - u0;

  if (tid < kHeadDim) sm.dw[tid] = 0.f;
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.kfull[i], 2);
      mbar_init(&sm.kready[i], 128);
      mbar_init(&sm.kempty[i], 1);
      mbar_init(&sm.vfull[i], 1);
      mbar_init(&sm.vready[i], 128);
      mbar_init(&sm.vempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.qfull[i], 1);
      mbar_init(&sm.qempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) mbar_init(&sm.qready[i], 64);
    mbar_init(&sm.sfull, 1);
    mbar_init(&sm.pfull, 256);
    mbar_init(&sm.afull, 1);
    mbar_init(&sm.dafull, 256);
    mbar_init(&sm.dpfull, 1);
    mbar_init(&sm.dsfull, 256);
    mbar_init(&sm.dq0, 1);
    mbar_init(&sm.dqfull, 1);
    mbar_init(&sm.tables, 256);
    mbar_init(&sm.xlb, 256);
    mbar_init(&sm.xdb, 256);
    mbar_init(&sm.xtb, 256);
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.never, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  // A programmatic dependent of the previous kernel on the stream: every
  // global access below (the weights included) waits for it to complete.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid < kHeadDim) {
    sm.wq[tid] = a.wq[tid];
    sm.wk[tid] = a.wk[tid];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  // Weights whose normalised operands could leave the fp16 range are refused
  // (uniformly: every thread sees the same shared copy).
  {
    bool wbad = false;
    for (int d = 0; d < kHeadDim; ++d)
      wbad |= !(fabsf(sm.wq[d]) <= kMaxWeight && fabsf(sm.wk[d]) <= kMaxWeight);
    if (wbad) {
      if (tid == 0 && blockIdx.x == 0) atomicCAS(a.err, 0, kDevErrBadWeights);
      n_tiles = 0;
    }
  }
  const int n_heads = n_tiles * a.G;

  if (warp < 4) regs_dec<kRegsControl>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint32_t kpar = 0, vpar = 0, kused = 0, vused = 0;  // per-slot parity / used bits
    bool ok = true;
    int nq = 0;
    auto wait0 = [&](uint64_t* bar, uint32_t par, int site) -> bool {
      bool w = true;
      if (lane == 0) w = mbar_wait_inl(bar, par, abort, a.err, site);
      return __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
    };
    auto load_kv = [&](bool is_k, int j, const Cursor& c) -> bool {
      const int s = j & 1;
      uint32_t& par = is_k ? kpar : vpar;
      uint32_t& used = is_k ? kused : vused;
      uint64_t* full = is_k ? &sm.kfull[s] : &sm.vfull[s];
      uint64_t* empty = is_k ? &sm.kempty[s] : &sm.vempty[s];
      if (((used >> s) & 1u) &&
          !wait0(empty, ((par >> s) & 1u) ^ 1u, is_k ? kSiteKEmpty : kSiteVEmpty))
        return false;
      if (lane == 0) {
        uint8_t* dst = is_k ? sm.k[0][s] : sm.v[0][s];
        mbar_arrive_expect_tx(full, kTileBytes);
        load_key_tile(dst, is_k ? &tm_k : &tm_v, is_k ? &tm_kh : &tm_vh, full, j, c.kvh, c.b,
                      2 * kHalfBytes);
      }
      if (is_k) {
        fill_rot_hi<kPairs>(sm.rot_hi[s], j, a, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(full);
      }
      par ^= 1u << s;
      used |= 1u << s;
      return true;
    };
    auto load_q = [&](const Cursor& c, int h) -> bool {
      const int b = nq & 1;
      if (nq >= 2 && !wait0(&sm.qempty[b], ((nq >> 1) - 1) & 1, kSiteQEmpty)) return false;
      if (lane == 0) {
        const int hq = c.kvh * a.G + h;
        mbar_arrive_expect_tx(&sm.qfull[b], kTileBytes);
        tma_load_4d(sm.slot[b], &tm_q, &sm.qfull[b], 0, hq, c.t * kTile, c.b);
        tma_load_4d(sm.slot[b] + kHalfBytes, &tm_q, &sm.qfull[b], 64, hq, c.t * kTile, c.b);
      }
      ++nq;
      return true;
    };
    Cursor c = cursor_at(a, u0);
    for (int it = 0; it < n_tiles && ok; ++it, next_tile(c, a)) {
      // The tile's first Q goes ahead of its key tiles: its slot frees a head
      // earlier than theirs, and its transform needs no key tile.
      ok = load_q(c, 0);
      if (ok && need_prev(c, a))
        ok = load_kv(true, c.t - 1, c) && load_kv(false, c.t - 1, c);
      ok = ok && load_kv(true, c.t, c) && load_kv(false, c.t, c);
      for (int h = 1; h < a.G && ok; ++h) ok = load_q(c, h);
    }
    if (!ok && lane == 0) {
      for (int s = 0; s < 2; ++s) {
        if ((kused >> s) & 1u) mbar_wait_drain(&sm.kfull[s], ((kpar >> s) & 1u) ^ 1u);
        if ((vused >> s) & 1u) mbar_wait_drain(&sm.vfull[s], ((vpar >> s) & 1u) ^ 1u);
      }
      for (int b = 0; b < 2; ++b) {
        const int cnt = (nq - b + 1) / 2;  // loads issued into slot b
        if (cnt > 0) mbar_wait_drain(&sm.qfull[b], (cnt - 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t kpar = 0, vpar = 0;
      bool ok = true;
      int nds = 0;  // dS tiles consumed so far
      Cursor c = cursor_at(a, u0);
      int h = 0;
      auto W = [&](uint64_t* bar, uint32_t par, int site) {
        if (ok) ok = mbar_wait_inl(bar, par, abort, a.err, site);
        return ok;
      };
      if (a.flags & SWA_FLAG_FORCE_TIMEOUT) W(&sm.never, 0, kSiteForced);  // for the tests
      for (int n = 0; n < n_heads && ok; ++n) {
        const uint32_t ph = n & 1;
        const bool hp = has_prev(c, a);
        const int sp = (c.t + 1) & 1, sc = c.t & 1;
        if (h == 0) {
          if (need_prev(c, a)) {
            if (!W(&sm.kready[sp], (kpar >> sp) & 1u, kSiteKReady)) break;
            kpar ^= 1u << sp;
          }
          if (!W(&sm.kready[sc], (kpar >> sc) & 1u, kSiteKReady)) break;
          kpar ^= 1u << sc;
        }
        if (!W(&sm.qready[n & 1], (n >> 1) & 1u, kSiteQReady)) break;
        tc_fence_after();
        // TMEM of head n, with tb = 0 or 256 by the parity of n and tw the
        // other half: S in tb .. tb + 255, then A and later dQ over its second
        // half; P in tw .. tw + 127; dP of ring slot 0 in tb .. tb + 127 and of
        // slot 1 in tw + 128 .. tw + 255.  This head's S overwrites only what
        // the previous head's dS phase has read (its P and slot-1 dP), not its
        // dQ, so it goes right behind the previous dQ; everything else of this
        // head is written after the compute warps' previous dq epilogue.
        const uint32_t tb = (n & 1) * 256u, tw = 256u - tb;
        // S = Q' [K' slot 0; K' slot 1]^T into columns tb .. tb + 255, one
        // N = 256 MMA per k-step: columns tb + 128 s .. hold the key tile in
        // slot s (t-1 and t in either order; without a tile t-1 that half is
        // never read).
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + tb, desc_kmajor(sm.slot[n & 1], kk), desc_ring(sm.k, kk), kIdescKK16x256,
                 kk > 0);
        mma_commit(&sm.sfull);
        if (h == 0) {
          if (need_prev(c, a)) {
            if (!W(&sm.vready[sp], (vpar >> sp) & 1u, kSiteVFull)) break;
            vpar ^= 1u << sp;
          }
          if (!W(&sm.vready[sc], (vpar >> sc) & 1u, kSiteVFull)) break;
          vpar ^= 1u << sc;
        }
        // A = P V into columns tb + 128 .. tb + 255, which S's second half held
        // (P packed in columns tw .. tw + 127)
        if (!W(&sm.pfull, ph, kSitePFull)) break;
        tc_fence_after();
        {
          uint32_t acc = 0;
          for (int blk = hp ? 0 : 1; blk < 2; ++blk)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {  // P of the tile in slot s: columns tw + 64 s ..
              const int slot = blk ? sc : sp;
              mma_ts(tmem + tb + 128, tmem + tw + slot * 64 + kk * 8, desc_mn_ring(sm.v, slot, kk),
                     kIdescKM16, acc);
              acc = 1;
            }
        }
        mma_commit(&sm.afull);
        // dP = dA V^T per key tile: ring slot 0's into columns tb .. tb + 127
        // (S's first half), slot 1's into tw + 128 .. tw + 255, clear of P and
        // A.  The dA tile goes to the workspace (for the key-major pass) while
        // the MMAs read it too; dS overwrites it after dpfull, which follows
        // the store's read.
        if (!W(&sm.dafull, ph, kSiteDAFull)) break;
        tc_fence_after();
        bulk_store(da_tile(a, c.b, c.kvh * a.G + h, c.t), sm.slot[n & 1], kTileBytes);
        bulk_commit();
        for (int blk = hp ? 0 : 1; blk < 2; ++blk) {
          const int s = blk ? sc : sp;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tmem + (s == 0 ? tb : tw + 128), desc_kmajor(sm.slot[n & 1], kk),
                   desc_ring_slot(sm.v, s, kk), kIdescKK16, kk > 0);
        }
        bulk_wait_read<0>();
        mma_commit(&sm.dpfull);
        // dQ = sum over key tiles of dS K' into columns tb + 128 .. tb + 255
        {
          uint32_t acc = 0;
          for (int blk = hp ? 0 : 1; blk < 2; ++blk) {
            if (!W(&sm.dsfull, nds & 1, kSiteDSFull)) break;
            ++nds;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              mma_ss(tmem + tb + 128, desc_kmajor(sm.slot[n & 1], kk),
                     desc_mn_ring(sm.k, blk ? sc : sp, kk), kIdescKM16, acc);
              acc = 1;
            }
            mma_commit(blk == 0 ? &sm.dq0 : &sm.dqfull);
          }
          if (!ok) break;
        }
        mma_commit(&sm.qempty[n & 1]);
        if (h == a.G - 1) {
          if (hp) {
            mma_commit(&sm.kempty[sp]);
            mma_commit(&sm.vempty[sp]);
          }
          if (c.u == n_tiles - 1 || c.t == a.tiles_per_chain - 1) {
            mma_commit(&sm.kempty[sc]);
            mma_commit(&sm.vempty[sc]);
          }
        }
        if (++h == a.G) {
          h = 0;
          next_tile(c, a);
        }
      }
      if (!ok) {
        mma_commit(&sm.drain);
        mbar_wait_drain(&sm.drain, 0);
      }
      bulk_wait_all();  // every dA tile written before the CTA exits
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------ Q transform (warps 2, 3)
    // Q' of head n in place in its slot, two rows per thread, while the
    // compute warpgroups still work on head n-1: head n's QK^T then follows
    // head n-1's dQ on the tensor core.
    bool ok = warp_wait(&sm.tables, 0, abort, a.err, kSiteTables);
    const int wsel = warp - 2;  // rows 32 wsel + 64 i + (0..31): hi entries 2 wsel + 4 i + (0, 1)
    Cursor c = cursor_at(a, u0);
    int h = 0;
    for (int n = 0; n < n_heads && ok; ++n) {
      if (h == 0) {  // rotation of the query tile's positions, this warp's entries
        for (int e = lane; e < kPairs * 4; e += 32) {
          const int p = e >> 2, ai = 2 * wsel + (e & 1) + 4 * ((e >> 1) & 1);
          float cv, sv;
          rope_cos_sin(static_cast<double>(a.pos0 + static_cast<long long>(c.t) * kTile) +
                           16.0 * ai, a.inv_freq[p], &cv, &sv);
          sm.qrot_hi[p][ai] = make_float2(cv, sv);
        }
        __syncwarp();
      }
      if (!(ok = warp_wait(&sm.qfull[n & 1], (n >> 1) & 1, abort, a.err, kSiteQFull))) break;
      for (int r = tid - 64; r < kTile; r += 64)
        sm.rinvq[n % 3][r] = norm_rope_row_lean<kPairs>(sm.slot[n & 1], r, sm.wq, sm.qrot_hi,
                                                        sm.rot, a.eps);
      fence_proxy_async_smem();
      mbar_arrive(&sm.qready[n & 1]);
      if (++h == a.G) {
        h = 0;
        next_tile(c, a);
      }
    }
  } else {
    // --------------------------------------------------- compute warpgroups
    // Two warpgroups share every query row: thread r of each owns row r
    // (TMEM lane r).  Warpgroup cg takes
    //   - the K transform (cg 0) or the V conversion (cg 1) of a new key tile,
    //     and cg 0 the Q transform;
    //   - chunks i = cg, cg + 2, ... of P over the band;
    //   - columns [64 cg, 64 cg + 64) of the gate/dA phase, of dS and of the
    //     dq epilogue.
    // Row sums (l, D and the dq Jacobian's dot) are exchanged through shared
    // memory, each under a bounded mbarrier wait that both warpgroups arrive on.
    regs_inc<kRegsCompute>();
    const int cg = (warp - 4) >> 2;
    const int row = (tid - 128) & 127;
    const int wq4 = warp & 3;
    const uint32_t t_row = tmem + (static_cast<uint32_t>(wq4 * 32) << 16);
    for (int e = tid - 128; e < kPairs * 16; e += 256) {
      const int p = e >> 4, bi = e & 15;
      float cv, sv;
      rope_cos_sin(static_cast<double>(bi), a.inv_freq[p], &cv, &sv);
      sm.rot.lo[p][bi] = make_float2(cv, sv);
    }
    mbar_arrive(&sm.tables);
    bool ok = warp_wait(&sm.tables, 0, abort, a.err, kSiteTables);
    uint32_t kpar = 0, vpar = 0;
    bool in_range = true;  // v and dO within the fp16 staging range
    int ndq0 = 0;
    int kt = 0;  // dS exponent of the current query tile
    // Publish this warpgroup's partial of a row sum and add the partner's.
    auto exchange = [&](uint64_t* bar, float (*buf)[kTile], float v, uint32_t par, int site,
                        float& total) -> bool {
      buf[cg][row] = v;
      mbar_arrive(bar);
      if (!warp_wait(bar, par, abort, a.err, site)) return false;
      total = v + buf[cg ^ 1][row];
      return true;
    };
    Cursor c = cursor_at(a, u0);
    int h = 0;
    for (int n = 0; n < n_heads && ok; ++n) {
      const uint32_t ph = n & 1;
      const bool hp = has_prev(c, a);
      const int sc = c.t & 1;
      const int hq = c.kvh * a.G + h;
      const long long pos = static_cast<long long>(c.t) * kTile + row;
      const bool valid_row = pos < a.T;
      const long long tok = (static_cast<long long>(c.b) * a.T + pos) * a.Hq + hq;  // row of q/g/dO
      const long long lrow = (static_cast<long long>(c.b) * a.Hq + hq) * a.T + pos;  // lse / D

      // ---- K' (cg 0) and V in fp16 (cg 1) of this tile's new key tiles
      if (h == 0) {
        for (int j = need_prev(c, a) ? c.t - 1 : c.t; j <= c.t && ok; ++j) {
          const int s = j & 1;
          if (cg == 0) {
            ok = warp_wait(&sm.kfull[s], (kpar >> s) & 1u, abort, a.err, kSiteKFull);
            if (!ok) break;
            norm_rope_row<kPairs>(sm.k[0][s], row, sm.wk, sm.rot_hi[s], sm.rot, a.eps,
                                  2 * kHalfBytes);
            fence_proxy_async_smem();
            mbar_arrive(&sm.kready[s]);
            kpar ^= 1u << s;
          } else {
            ok = warp_wait(&sm.vfull[s], (vpar >> s) & 1u, abort, a.err, kSiteVFull);
            if (!ok) break;
            const uint32_t m = row_to_f16(sm.v[0][s], row, 2 * kHalfBytes);
            in_range &= m <= kF16MaxBits;
            const uint32_t wm = __reduce_max_sync(0xffffffffu, m);
            if (lane == 0) sm.vmax[s][wq4] = wm;
            fence_proxy_async_smem();
            mbar_arrive(&sm.vready[s]);
          }
        }
        if (!ok) break;
      }
      uint8_t* slot = sm.slot[n & 1];
      const uint8_t* grow = reinterpret_cast<const uint8_t*>(a.g + tok * kHeadDim) + 128 * cg;
      const uint8_t* dorow = reinterpret_cast<const uint8_t*>(a.dO + tok * kHeadDim) + 128 * cg;
      // Rows past T take lse = +inf: their P is exactly 0 with no mask.
      const float lse_r = valid_row ? a.lse[lrow] : INFINITY;  // loaded once, used twice
      const float lse2 = lse_r * kLog2e;
      // this warpgroup's 64 columns of g and dO, in flight during P
      uint32_t gc[32], dc[32];  // this warpgroup's 64 columns of g and dO
      if (valid_row) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          ld32B(grow + 32 * i, *reinterpret_cast<uint32_t(*)[8]>(gc + 8 * i));
          ld32B(dorow + 32 * i, *reinterpret_cast<uint32_t(*)[8]>(dc + 8 * i));
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) gc[i] = dc[i] = 0u;
      }

      // ---- P = exp(s - lse) on the band.  The in-band 32-column chunks are
      // key tile t-1's wq4..3 (when it exists), then key tile t's 0..wq4;
      // this warpgroup takes every other one.  A key tile's S sits at the
      // columns of its ring slot (tb + 128 s ..), its P at tw + 64 s .., clear
      // of S: each chunk's P is stored as soon as it is computed, and PV may
      // start before the row sums are exchanged.
      if (!(ok = warp_wait(&sm.sfull, ph, abort, a.err, kSiteSFull))) break;
      tc_fence_after();
      // Q' done.  Its 1/rms, read in the dq epilogue, stays until head n+3's
      // transform, which waits (through its slot) for head n+1's dS.
      if (!(ok = warp_wait(&sm.qready[n & 1], (n >> 1) & 1, abort, a.err, kSiteQReady))) break;
      const uint32_t tb = (n & 1) * 256u, tw = 256u - tb;  // TMEM halves, as the MMA lane's
      const int na = hp ? 4 - wq4 : 0;  // chunks of key tile t-1 in the band
      const int nch = na + wq4 + 1;
      const int sp = sc ^ 1;  // ring slot of key tile t-1
      const float2 sc2 = make_float2(a.scale_log2, a.scale_log2), nl2 = make_float2(-lse2, -lse2);
      float2 lsum2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const int i = cg + 2 * k;
        if (i < nch) {
          const int blk = i < na ? 0 : 1;
          const int pc = blk == 0 ? wq4 + i : i - na;
          uint32_t x[32], pk[16];
          tmem_ld32(t_row + tb + (blk ? sc : sp) * 128 + pc * 32, x);
          tmem_wait_ld();
          if (pc != wq4) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float2 z = __ffma2_rn(
                  make_float2(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1])), sc2, nl2);
              pk[e] = pack_f16x2(ex2_approx(z.x), ex2_approx(z.y));
              lsum2 = __fadd2_rn(lsum2, f16x2(pk[e]));  // the values the MMAs see
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int c0 = pc * 32 + 2 * e;
              const bool in0 = blk == 0 ? c0 > row : c0 <= row;
              const bool in1 = blk == 0 ? c0 + 1 > row : c0 + 1 <= row;
              const float2 z = __ffma2_rn(
                  make_float2(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1])), sc2, nl2);
              pk[e] = pack_f16x2(in0 ? ex2_approx(z.x) : 0.f, in1 ? ex2_approx(z.y) : 0.f);
              lsum2 = __fadd2_rn(lsum2, f16x2(pk[e]));
            }
          }
          tmem_st16(t_row + tw + (blk ? sc : sp) * 64 + pc * 16, pk);
        }
      }
      {
        // chunks outside the band: key tile t-1's below wq4 (or all of it
        // when it does not exist) by cg 0, key tile t's above wq4 by cg 1
        const uint32_t zero16[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u,
                                     0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        for (int pc = 0; pc < 4; ++pc) {
          if (cg == 0 && (!hp || pc < wq4)) tmem_st16(t_row + tw + sp * 64 + pc * 16, zero16);
          if (cg == 1 && pc > wq4) tmem_st16(t_row + tw + sc * 64 + pc * 16, zero16);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.pfull);
      // The row's dA exponent e: each warpgroup takes it from its 64 values of
      // dO and the two are exchanged with l (the row takes the smaller).  Each
      // warp's minimum goes to shared memory too, for the tile's minimum.
      float lsum;
      int ei;
      {
        uint32_t m2 = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) m2 = __vmaxu2(m2, dc[i] & 0x7FFF7FFFu);
        const uint32_t mh = max(m2 & 0xFFFFu, m2 >> 16);
        const int ef = static_cast<int>(mh >> 7);
        in_range &= !(ef > kMaxDoExpField && ef < 0xFF);
        const int eh = row_exponent(mh);
        const int ew = __reduce_min_sync(0xffffffffu, eh);
        if (lane == 0) sm.xew[ph][cg][wq4] = ew;
        sm.xl[cg][row] = lsum2.x + lsum2.y;
        sm.xe[cg][row] = eh;
        mbar_arrive(&sm.xlb);
        if (!(ok = warp_wait(&sm.xlb, ph, abort, a.err, kSiteXchg))) break;
        lsum = lsum2.x + lsum2.y + sm.xl[cg ^ 1][row];
        ei = min(eh, sm.xe[cg ^ 1][row]);
        if (cg == 1 && row == 0) {  // the key-major pass's common scale starts here
          int mn = kExpLimit;
#pragma unroll
          for (int w = 0; w < 8; ++w) mn = min(mn, sm.xew[ph][w >> 2][w & 3]);
          a.ws_ee[(static_cast<long long>(c.b) * a.Hq + hq) * a.tiles_per_chain + c.t] = mn;
        }
      }
      // The forward's lse came from its own rounding of the scores; these rows
      // are renormalised to sum to exactly 1 under this pass's scores, and the
      // corrected normaliser goes to the key-major pass.
      const float inv_l = lsum > 0.f ? 1.0f / lsum : 0.f;
      // in log2 units, with the row's exponent added (the key-major pass
      // subtracts its common exponent and so scales P^T column by column)
      // (warpgroup 1 writes the row's workspace entries: it has the fewer P chunks)
      if (cg == 1 && valid_row)
        a.ws_lse[lrow] = (lse_r + __logf(lsum)) * kLog2e + static_cast<float>(ei);

      // ---- dA = dO sigma(g) 2^e over this warpgroup's 64 columns, into the
      // Q slot (QK^T has read it): dA needs no A, so the dP MMAs start on it
      // while A = P V is still on its way.  dO sigma'(g) waits for A in
      // registers.
      const float2 il2 = make_float2(inv_l, inv_l);
      const float2 si2 = make_float2(pow2f(ei), pow2f(ei));  // dA is staged as dA 2^e
      float2 dgf[32];    // dO sigma (1 - sigma) per column pair
      uint32_t dao[32];  // dA 2^e as the MMAs see it (fp16)
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float2 gg = bf2(gc[e]), dd = bf2(dc[e]);
        float2 ds;                            // sigma (1 - sigma), without cancellation
        const float2 sg = sigmoid2(gg, &ds);  // one MUFU op per element
        dgf[e] = __fmul2_rn(dd, ds);
        const float2 dav = __fmul2_rn(__fmul2_rn(dd, sg), si2);
        dao[e] = pack_f16x2(dav.x, dav.y);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        // dA into the MMA operand tile (row-major over dims, 128B swizzle)
        const int c16 = 8 * cg + i;  // 16-byte piece of the row
        *reinterpret_cast<uint4*>(slot + (c16 >> 3) * kHalfBytes + sw_off(row, c16 & 7)) =
            make_uint4(dao[4 * i], dao[4 * i + 1], dao[4 * i + 2], dao[4 * i + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sm.dafull);

      // ---- dg and D = sum dA A over the same columns (TMEM chunks 2 cg,
      // 2 cg + 1 of A)
      if (!(ok = warp_wait(&sm.afull, ph, abort, a.err, kSiteAFull))) break;
      tc_fence_after();
      float2 dsum2 = make_float2(0.f, 0.f);
      {
        uint8_t* dgrow = reinterpret_cast<uint8_t*>(a.dg + tok * kHeadDim) + 128 * cg;
#pragma unroll
        for (int hc = 0; hc < 2; ++hc) {
          uint32_t x[32];
          tmem_ld32(t_row + tb + 128 + (2 * cg + hc) * 32, x);
          tmem_wait_ld();
          uint32_t dgo[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 av = __fmul2_rn(
                make_float2(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1])), il2);  // A / l
            const float2 dgv = __fmul2_rn(dgf[16 * hc + e], av);
            dgo[e] = pack_bf16x2(dgv.x, dgv.y);
            dsum2 = __ffma2_rn(f16x2(dao[16 * hc + e]), av, dsum2);  // D uses the rounded dA
          }
          if (valid_row) {
            st32B(dgrow + 64 * hc, *reinterpret_cast<const uint32_t(*)[8]>(dgo));
            st32B(dgrow + 64 * hc + 32, *reinterpret_cast<const uint32_t(*)[8]>(dgo + 8));
          }
        }
      }
      float dsum;
      if (!(ok = exchange(&sm.xdb, sm.xd, dsum2.x + dsum2.y, ph, kSiteXchg, dsum))) break;
      if (cg == 1 && valid_row) a.ws_d[lrow] = dsum;

      // ---- dS = scale P (dP - D) per key tile into the Q slot (this
      // warpgroup's 64 columns), then dQ
      uint32_t xq[32];  // this warpgroup's half of the raw q row, loaded while dS and dQ run
      if (valid_row) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          ld32B(reinterpret_cast<const uint8_t*>(a.q + tok * kHeadDim) + 128 * cg + 32 * i,
                *reinterpret_cast<uint32_t(*)[8]>(xq + 8 * i));
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) xq[i] = 0u;
      }
      // dS exponent of this query tile, from the largest |v| of its key
      // tiles: both warpgroups read the V conversion's maxima once per tile.
      if (h == 0) {
        for (int j = need_prev(c, a) ? c.t - 1 : c.t; j <= c.t && ok; ++j) {
          const int s = j & 1;
          ok = warp_wait(&sm.vready[s], (vpar >> s) & 1u, abort, a.err, kSiteVReady);
          vpar ^= 1u << s;
        }
        if (!ok) break;
        uint32_t vm = 0;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          vm = max(vm, sm.vmax[sc][w]);
          if (hp) vm = max(vm, sm.vmax[sc ^ 1][w]);
        }
        kt = ds_exponent(a.scale, vm);
        if (cg == 0 && row == 0)
          a.ws_ek[(static_cast<long long>(c.b) * a.Hkv + c.kvh) * a.tiles_per_chain + c.t] = kt;
      }
      if (!(ok = warp_wait(&sm.dpfull, ph, abort, a.err, kSiteDPFull))) break;
      tc_fence_after();
      // dS 2^(e+k) = scale 2^k P / l (dP 2^e - D 2^e)
      const float dsc = a.scale * inv_l * pow2f(kt);
      const float2 sl2 = make_float2(dsc, dsc), nd2 = make_float2(-dsum, -dsum);
      for (int blk = hp ? 0 : 1; blk < 2 && ok; ++blk) {
        if (blk == 1 && hp) {  // the MMA has read dS of key tile t-1 from the slot
          if (!(ok = warp_wait(&sm.dq0, ndq0 & 1, abort, a.err, kSiteDQ0))) break;
          ++ndq0;
        }
        // both chunks' P and dP in flight at once, then one wait
        uint32_t pkc[2][16], dp[2][32];
#pragma unroll
        for (int hc = 0; hc < 2; ++hc) {
          const int s = blk ? sc : sc ^ 1;  // the key tile's ring slot
          tmem_ld16(t_row + tw + s * 64 + (2 * cg + hc) * 16, pkc[hc]);
          tmem_ld32(t_row + (s == 0 ? tb : tw + 128) + (2 * cg + hc) * 32, dp[hc]);
        }
        tmem_wait_ld();
#pragma unroll
        for (int hc = 0; hc < 2; ++hc) {
          const int pc = 2 * cg + hc;
          uint32_t ds[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 v = __fmul2_rn(
                __fmul2_rn(f16x2(pkc[hc][e]), sl2),
                __fadd2_rn(make_float2(__uint_as_float(dp[hc][2 * e]),
                                       __uint_as_float(dp[hc][2 * e + 1])),
                           nd2));
            ds[e] = pack_f16x2(v.x, v.y);
          }
          uint8_t* half = slot + (pc >> 1) * kHalfBytes;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint4*>(half + sw_off(row, (pc & 1) * 4 + i)) =
                make_uint4(ds[4 * i], ds[4 * i + 1], ds[4 * i + 2], ds[4 * i + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sm.dsfull);
      }
      if (!ok) break;

      // ---- dq through RoPE^-1 and the RMSNorm Jacobian, over this
      // warpgroup's half of the row (the rotated dims are all in half 0)
      if (!(ok = warp_wait(&sm.dqfull, ph, abort, a.err, kSiteDQFull))) break;
      tc_fence_after();
      {
        const float rinv = sm.rinvq[n % 3][row];
        const float2 rinv2 = make_float2(rinv, rinv);
        float y[64];
        {
          uint32_t r[32], r2[32];
          tmem_ld32(t_row + tb + 128 + cg * 64, r);
          tmem_ld32(t_row + tb + 128 + cg * 64 + 32, r2);
          tmem_wait_ld();
          const float2 un2 = make_float2(pow2f(-(ei + kt)), pow2f(-(ei + kt)));  // undo 2^(e+k)
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 y0 = __fmul2_rn(make_float2(__uint_as_float(r[2 * i]),
                                                     __uint_as_float(r[2 * i + 1])), un2);
            const float2 y1 = __fmul2_rn(make_float2(__uint_as_float(r2[2 * i]),
                                                     __uint_as_float(r2[2 * i + 1])), un2);
            y[2 * i] = y0.x;
            y[2 * i + 1] = y0.y;
            y[32 + 2 * i] = y1.x;
            y[32 + 2 * i + 1] = y1.y;
          }
        }
        if (cg == 0) {  // RoPE^-1 on the rotated pairs, all in the first half
#pragma unroll
          for (int p = 0; p < kPairs; ++p) {
            const float2 rcp = rot_at(sm.rot_hi[sc], sm.rot, p, row);
            const float a0 = y[p], b0 = y[p + kPairs];
            y[p] = a0 * rcp.x + b0 * rcp.y;  // R^T: (a, b) -> (a cos + b sin, b cos - a sin)
            y[p + kPairs] = b0 * rcp.x - a0 * rcp.y;
          }
        }
        float2 dot2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 xh = __fmul2_rn(bf2(xq[i]), rinv2);  // xhat
          const int d = 64 * cg + 2 * i;
          dot2 = __ffma2_rn(__fmul2_rn(make_float2(y[2 * i], y[2 * i + 1]),
                                       make_float2(sm.wq[d], sm.wq[d + 1])),
                            xh, dot2);
        }
        float dot;
        if (!(ok = exchange(&sm.xtb, sm.xt, dot2.x + dot2.y, ph, kSiteXchg, dot))) break;
        dot *= 1.0f / kHeadDim;
        const float2 ndot2 = make_float2(-dot, -dot);
        uint8_t* out = reinterpret_cast<uint8_t*>(a.dq + tok * kHeadDim) + 128 * cg;
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {  // dx = rinv (w dy - xhat dot), 16 dims at a time
          uint32_t o[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int i = 8 * i4 + e;
            const float2 xh = __fmul2_rn(bf2(xq[i]), rinv2);
            const int d = 64 * cg + 2 * i;
            const float2 yv = make_float2(y[2 * i], y[2 * i + 1]);
            const float2 g = __fmul2_rn(
                rinv2, __ffma2_rn(xh, ndot2, __fmul2_rn(yv, make_float2(sm.wq[d], sm.wq[d + 1]))));
            o[e] = pack_bf16x2(g.x, g.y);
            const float2 cv = __fmul2_rn(yv, xh);  // dw contribution dy * xhat, in place
            y[2 * i] = cv.x;
            y[2 * i + 1] = cv.y;
          }
          if (valid_row) st32B(out + 32 * i4, o);
        }
        const float2 sw = warp_reduce_scatter64(y, lane);
        atomicAdd(sm.dw + 64 * cg + 2 * lane, sw.x);
        atomicAdd(sm.dw + 64 * cg + 2 * lane + 1, sw.y);
      }
      if (++h == a.G) {
        h = 0;
        next_tile(c, a);
      }
    }
    if (!in_range) atomicCAS(a.err, 0, kDevErrRange);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // per-CTA dwq into the caller's accumulator
  if (tid >= 128 && tid < 256 && !*abort) atomicAdd(a.dwq + (tid - 128), sm.dw[tid - 128]);
}

// ======================================================= pass 2: key-major

struct alignas(1024) SmemKV {
  uint8_t k[kTileBytes];   // K'_j
  uint8_t v[kTileBytes];   // V_j
  uint8_t q[2][kTileBytes];   // Q'_i of (query tile, head) pair nq, in buffer nq & 1
  uint8_t da[2][kTileBytes];  // dA_i
  RotTables rot;
  float2 rot_hi[2][2][kMaxPairs][8];  // [key tile parity][tile j, j+1]
  float lse2[2][2][kTile], dd[2][2][kTile];  // per query column: [warpgroup][its pair parity]
  float wq[kHeadDim], wk[kHeadDim], dw[kHeadDim];
  float rinvk[kTile];   // 1/rms of each K row (cg 0 computes it; both use it)
  float xt[2][kTile];   // per-warpgroup halves of each dk row's Jacobian dot
  uint64_t kfull, vfull, kvempty, qfull[2], qempty[2], kvready, dkvfull, tfree, xtb;
  uint64_t qready[2], staged[2], sfull[2], pfull[2];  // per warpgroup: pair nq is warpgroup nq & 1's
  uint64_t tables, drain, never;  // never: completed by nothing (forced timeouts)
  uint32_t tmem_base;
  int abort;
};
static_assert(offsetof(SmemKV, lse2) % 16 == 0 && offsetof(SmemKV, dd) % 16 == 0,
              "per-column lse / D are read as float4");
static_assert(sizeof(SmemKV) + 1024 <= 232448, "pass 2 shared memory");

template <int kPairs>
__global__ void __launch_bounds__(kThreads, 1)
    swa_bwd_kv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_kh,
                      const __grid_constant__ CUtensorMap tm_vh, const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  SmemKV& sm = *reinterpret_cast<SmemKV*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                          ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u0 = static_cast<int>(a.kv_total_tiles * blockIdx.x / gridDim.x);
  const int u1 = static_cast<int>(a.kv_total_tiles * (blockIdx.x + 1) / gridDim.x);
  int n_tiles = u1 - u0;

  if (tid < kHeadDim) sm.dw[tid] = 0.f;
  if (tid == 0) {
    mbar_init(&sm.kfull, 2);
    mbar_init(&sm.vfull, 1);
    mbar_init(&sm.kvempty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.qfull[i], 1);
      mbar_init(&sm.qempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.qready[i], 128);
      mbar_init(&sm.staged[i], 128);
      mbar_init(&sm.sfull[i], 1);
      mbar_init(&sm.pfull[i], 128);
    }
    mbar_init(&sm.kvready, 256);
    mbar_init(&sm.dkvfull, 1);
    mbar_init(&sm.tfree, 256);
    mbar_init(&sm.xtb, 256);
    mbar_init(&sm.tables, 256);
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.never, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  // A programmatic dependent of the previous kernel on the stream: every
  // global access below (the weights included) waits for it to complete.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid < kHeadDim) {
    sm.wq[tid] = a.wq[tid];
    sm.wk[tid] = a.wk[tid];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  // Weights whose normalised operands could leave the fp16 range are refused
  // (uniformly: every thread sees the same shared copy).
  {
    bool wbad = false;
    for (int d = 0; d < kHeadDim; ++d)
      wbad |= !(fabsf(sm.wq[d]) <= kMaxWeight && fabsf(sm.wk[d]) <= kMaxWeight);
    if (wbad) {
      if (tid == 0 && blockIdx.x == 0) atomicCAS(a.err, 0, kDevErrBadWeights);
      n_tiles = 0;
    }
  }
  // (query tiles, heads) a key tile meets: tiles j and j+1 (when they exist) x G;
  // the halo's key tile -1 meets only query tile 0
  auto n_iters = [&](const Cursor& c) {
    return ((c.t >= 0 ? 1 : 0) + (c.t + 1 < a.tiles_per_chain ? 1 : 0)) * a.G;
  };
  auto dt0 = [&](const Cursor& c) { return c.t < 0 ? 1 : 0; };  // first query tile j + dt0

  if (warp < 4) regs_dec<kRegsControl>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    bool ok = true;
    int nq = 0, nkv = 0;
    auto wait0 = [&](uint64_t* bar, uint32_t par, int site) -> bool {
      bool w = true;
      if (lane == 0) w = mbar_wait_inl(bar, par, abort, a.err, site);
      return __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
    };
    Cursor c = cursor_at_kv(a, u0);
    for (int it = 0; it < n_tiles && ok; ++it, next_tile_kv(c, a)) {
      if (it > 0 && !(ok = wait0(&sm.kvempty, (it - 1) & 1, kSiteKVEmpty))) break;
      ++nkv;
      if (lane == 0) {
        mbar_arrive_expect_tx(&sm.kfull, kTileBytes);
        load_key_tile(sm.k, &tm_k, &tm_kh, &sm.kfull, c.t, c.kvh, c.b);
        mbar_arrive_expect_tx(&sm.vfull, kTileBytes);
        load_key_tile(sm.v, &tm_v, &tm_vh, &sm.vfull, c.t, c.kvh, c.b);
      }
      fill_rot_hi<kPairs>(sm.rot_hi[it & 1][0], c.t, a, lane);
      fill_rot_hi<kPairs>(sm.rot_hi[it & 1][1], c.t + 1, a, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.kfull);
      const int ni = n_iters(c);
      for (int i = 0; i < ni && ok; ++i, ++nq) {
        const int b = nq & 1;
        if (nq >= 2 && !(ok = wait0(&sm.qempty[b], ((nq >> 1) - 1) & 1, kSiteQEmpty))) break;
        if (lane == 0) {
          const int qt = c.t + dt0(c) + i / a.G, hq = c.kvh * a.G + i % a.G;
          mbar_arrive_expect_tx(&sm.qfull[b], 2 * kTileBytes);
          tma_load_4d(sm.q[b], &tm_q, &sm.qfull[b], 0, hq, qt * kTile, c.b);
          tma_load_4d(sm.q[b] + kHalfBytes, &tm_q, &sm.qfull[b], 64, hq, qt * kTile, c.b);
          bulk_load(sm.da[b], da_tile(a, c.b, hq, qt), kTileBytes, &sm.qfull[b]);
        }
      }
    }
    if (!ok && lane == 0) {
      // every copy issued so far has completed or is drained here
      if (nkv > 0) {
        mbar_wait_drain(&sm.kfull, (nkv - 1) & 1);
        mbar_wait_drain(&sm.vfull, (nkv - 1) & 1);
      }
      for (int b = 0; b < 2; ++b) {
        const int cnt = (nq - b + 1) / 2;  // loads issued into buffer b
        if (cnt > 0) mbar_wait_drain(&sm.qfull[b], (cnt - 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = true;
      int nq = 0;
      auto W = [&](uint64_t* bar, uint32_t par, int site) {
        if (ok) ok = mbar_wait_inl(bar, par, abort, a.err, site);
        return ok;
      };
      if (a.flags & SWA_FLAG_FORCE_TIMEOUT) W(&sm.never, 0, kSiteForced);  // for the tests
      Cursor c = cursor_at_kv(a, u0);
      for (int it = 0; it < n_tiles && ok; ++it, next_tile_kv(c, a)) {
        const int ni = n_iters(c);
        for (int i = 0; i < ni && ok; ++i, ++nq) {
          const int cg = nq & 1, ph = (nq >> 1) & 1;  // the pair's warpgroup, its phase
          if (i == 0) {
            if (!W(&sm.kvready, it & 1, kSiteKVReady)) break;
            if (it > 0 && !W(&sm.tfree, (it - 1) & 1, kSiteTFree)) break;
          }
          if (!W(&sm.qready[cg], ph, kSiteQReady)) break;
          // S^T and dP^T of this pair overwrite the columns that dV and dK of
          // the previous pair read as their A operands (P^T, dS^T); the tensor
          // core runs one thread's MMAs in issue order, so they go right
          // behind them.
          tc_fence_after();
          // S^T = K' Q'^T (columns 256..383), dP^T = V dA^T (384..511)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tmem + 256, desc_kmajor(sm.k, kk), desc_kmajor(sm.q[nq & 1], kk), kIdescKK16,
                   kk > 0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tmem + 384, desc_kmajor(sm.v, kk), desc_kmajor(sm.da[nq & 1], kk), kIdescKK16,
                   kk > 0);
          mma_commit(&sm.sfull[cg]);
          if (!W(&sm.pfull[cg], ph, kSitePFull)) break;
          tc_fence_after();
          // dV += P^T dA (0..127), dK += dS^T Q' (128..255)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem, tmem + 256 + kk * 8, desc_mn(sm.da[nq & 1], kk), kIdescKM16,
                   (i > 0 || kk > 0));
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + 128, tmem + 384 + kk * 8, desc_mn(sm.q[nq & 1], kk), kIdescKM16,
                   (i > 0 || kk > 0));
          mma_commit(&sm.qempty[nq & 1]);
        }
        if (!ok) break;
        mma_commit(&sm.dkvfull);
        mma_commit(&sm.kvempty);
      }
      if (!ok) {
        mma_commit(&sm.drain);
        mbar_wait_drain(&sm.drain, 0);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // --------------------------------------------------- compute warpgroups
    // Two warpgroups, each with thread r on key row r (TMEM lane r).  Per key
    // tile cg 0 transforms K and cg 1 converts V; the (query tile, head) pairs
    // alternate between them (pair nq is warpgroup nq & 1's: its Q transform,
    // lse / D staging and P^T / dS^T), so one warpgroup transforms the next
    // pair's Q while the other works on the current pair's scores; dk and dv
    // are split by halves of the row.
    regs_inc<kRegsCompute>();
    const int cg = (warp - 4) >> 2;
    const int row = (tid - 128) & 127;
    const int wq4 = warp & 3;
    const uint32_t t_row = tmem + (static_cast<uint32_t>(wq4 * 32) << 16);
    for (int e = tid - 128; e < kPairs * 16; e += 256) {
      const int p = e >> 4, bi = e & 15;
      float cv, sv;
      rope_cos_sin(static_cast<double>(bi), a.inv_freq[p], &cv, &sv);
      sm.rot.lo[p][bi] = make_float2(cv, sv);
    }
    mbar_arrive(&sm.tables);
    bool ok = warp_wait(&sm.tables, 0, abort, a.err, kSiteTables);
    bool in_range = true;  // v within the fp16 staging range
    int nq = 0;
    Cursor c = cursor_at_kv(a, u0);
    for (int it = 0; it < n_tiles && ok; ++it, next_tile_kv(c, a)) {
      const long long kpos = static_cast<long long>(c.t) * kTile + row;  // this thread's key
      // Common scale of this key tile's dV and dK accumulators: e_c, the
      // smallest dA exponent among the (query tile, head) pairs it meets, and
      // k_c, the smaller dS exponent of the two query tiles (their key tiles
      // j-1 .. j+1 bound every D_i the pairs bring).  Column i of P^T and dS^T
      // is scaled by 2^(e_c - e_i) <= 1 through its staged lse, so the
      // accumulators hold dV 2^e_c and dK 2^(e_c + k_c).
      int ec = kExpLimit, kc = kExpLimit;
      {
        const bool own = c.t >= 0, next = c.t + 1 < a.tiles_per_chain;
        const long long chain = static_cast<long long>(c.b) * a.Hkv + c.kvh;
        if (own) kc = min(kc, __ldg(a.ws_ek + chain * a.tiles_per_chain + c.t));
        if (next) kc = min(kc, __ldg(a.ws_ek + chain * a.tiles_per_chain + c.t + 1));
        for (int h2 = 0; h2 < a.G; ++h2) {
          const long long base =
              (static_cast<long long>(c.b) * a.Hq + c.kvh * a.G + h2) * a.tiles_per_chain;
          if (own) ec = min(ec, __ldg(a.ws_ee + base + c.t));
          if (next) ec = min(ec, __ldg(a.ws_ee + base + c.t + 1));
        }
      }
      // ---- K'_j (cg 0) and V_j in fp16 (cg 1), published to the MMA by kvready
      // (kfull also publishes the tile's rotation tables, which both use)
      if (!(ok = warp_wait(&sm.kfull, it & 1, abort, a.err, kSiteKFull))) break;
      if (cg == 0) {
        sm.rinvk[row] = norm_rope_row<kPairs>(sm.k, row, sm.wk, sm.rot_hi[it & 1][0], sm.rot, a.eps);
      } else {
        if (!(ok = warp_wait(&sm.vfull, it & 1, abort, a.err, kSiteVFull))) break;
        in_range &= row_to_f16(sm.v, row) <= kF16MaxBits;
      }
      fence_proxy_async_smem();
      mbar_arrive(&sm.kvready);
      const int ni = n_iters(c);
      for (int i = 0; i < ni && ok; ++i, ++nq) {
        if ((nq & 1) != cg) continue;  // the other warpgroup's pair
        const int ph = (nq >> 1) & 1;   // phase of this warpgroup's barriers
        const int dt = dt0(c) + i / a.G;  // query tile j + dt
        const int hq = c.kvh * a.G + i % a.G;
        const long long qpos = static_cast<long long>(c.t + dt) * kTile + row;  // query row `row`
        // ---- Q'_i, and lse / D of its rows for the column-wise softmax (their
        // loads go out first, so the transform hides their latency)
        const long long lrow = (static_cast<long long>(c.b) * a.Hq + hq) * a.T + qpos;
        const float lse_i = qpos < a.T ? __ldg(a.ws_lse + lrow) : 0.f;
        const float d_i = qpos < a.T ? __ldg(a.ws_d + lrow) : 0.f;
        if (!(ok = warp_wait(&sm.qfull[cg], ph, abort, a.err, kSiteQFull))) break;
        norm_rope_row<kPairs>(sm.q[cg], row, sm.wq, sm.rot_hi[it & 1][dt], sm.rot, a.eps);
        float* l2 = sm.lse2[cg][ph];
        float* dd = sm.dd[cg][ph];
        l2[row] = lse_i - static_cast<float>(ec);  // log2 lse_i + e_i - e_c
        dd[row] = d_i;                           // D_i 2^e_i
        fence_proxy_async_smem();
        mbar_arrive(&sm.qready[cg]);
        mbar_arrive(&sm.staged[cg]);  // lse2 / dd of this pair visible to the warpgroup
        if (!(ok = warp_wait(&sm.staged[cg], ph, abort, a.err, kSiteStaged))) break;
        // ---- P^T and dS^T for key row `row` against the 128 query columns
        if (!(ok = warp_wait(&sm.sfull[cg], ph, abort, a.err, kSiteSFull))) break;
        tc_fence_after();
        // Query columns past T (the last, partial tile) and key rows past T
        // are outside; only chunk wq4 straddles the band edge.
        const int col_end = static_cast<int>(min(static_cast<long long>(kTile),
                                                 a.T - static_cast<long long>(c.t + dt) * kTile));
        const float2 kval2 = kpos < a.T ? make_float2(1.f, 1.f) : make_float2(0.f, 0.f);
        const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
        const float dss = a.scale * pow2f(kc);  // dS^T 2^(e_c + k_c)
        const float2 scale2 = make_float2(dss, dss);
#pragma unroll 1
        for (int pc = 0; pc < 4; ++pc) {
          // query tile j keeps columns >= row, tile j+1 columns < row
          // (warp-uniform: tcgen05.ld is warp-collective).
          const bool any = dt == 0 ? (pc >= wq4) : (pc <= wq4);
          uint32_t pk[16], dk[16];
          if (any) {
            uint32_t sv[32], dp[32];
            tmem_ld32(t_row + 256 + pc * 32, sv);
            tmem_ld32(t_row + 384 + pc * 32, dp);
            tmem_wait_ld();
            const bool edge = pc == wq4 || pc * 32 + 32 > col_end;
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {  // four columns per step
              const float4 l4 = *reinterpret_cast<const float4*>(l2 + pc * 32 + 4 * e4);
              const float4 d4 = *reinterpret_cast<const float4*>(dd + pc * 32 + 4 * e4);
#pragma unroll
              for (int h2 = 0; h2 < 2; ++h2) {
                const int e = 2 * e4 + h2;
                const float2 nl = h2 == 0 ? make_float2(-l4.x, -l4.y) : make_float2(-l4.z, -l4.w);
                const float2 dv2 = h2 == 0 ? make_float2(d4.x, d4.y) : make_float2(d4.z, d4.w);
                const float2 z = __ffma2_rn(
                    make_float2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), sc2, nl);
                float2 p = __fmul2_rn(make_float2(ex2_approx(z.x), ex2_approx(z.y)), kval2);
                if (edge) {
                  const int col = pc * 32 + 2 * e;
                  const bool in0 = col < col_end && (dt == 0 ? col >= row : col < row);
                  const bool in1 = col + 1 < col_end && (dt == 0 ? col + 1 >= row : col + 1 < row);
                  p = make_float2(in0 ? p.x : 0.f, in1 ? p.y : 0.f);
                }
                const float2 dsv = __fmul2_rn(
                    __fmul2_rn(scale2, p),
                    __fadd2_rn(make_float2(__uint_as_float(dp[2 * e]), __uint_as_float(dp[2 * e + 1])),
                               make_float2(-dv2.x, -dv2.y)));
                pk[e] = pack_f16x2(p.x, p.y);
                dk[e] = pack_f16x2(dsv.x, dsv.y);
              }
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = dk[e] = 0u;
          }
          // packed over S^T / dP^T columns this thread has already read
          tmem_st16(t_row + 256 + pc * 16, pk);
          tmem_st16(t_row + 384 + pc * 16, dk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sm.pfull[cg]);
      }
      if (!ok) break;
      // ---- dk (RoPE^-1, RMSNorm Jacobian) and dv of key tile j, over this
      // warpgroup's half of the row (the rotated dims are all in half 0)
      const long long krow = (static_cast<long long>(c.b) * a.T + kpos) * a.Hkv + c.kvh;
      // the key's raw row: an own row, or (key tile -1) halo row `row - 1`;
      // row 0 of the halo tile is the zero-filled row before the halo
      const bool own_row = c.t >= 0 && kpos < a.T;
      const long long hrow =
          (static_cast<long long>(c.b) * (kWindow - 1) + (row - 1)) * a.Hkv + c.kvh;
      const uint16_t* ksrc = own_row ? a.k + krow * kHeadDim
                                     : (c.t < 0 && row >= 1 ? a.k_halo + hrow * kHeadDim : nullptr);
      uint32_t xk[32];  // this warpgroup's half of the raw k row, loaded while dK is computed
      if (ksrc != nullptr) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          ld32B(reinterpret_cast<const uint8_t*>(ksrc) + 128 * cg + 32 * i,
                *reinterpret_cast<uint32_t(*)[8]>(xk + 8 * i));
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) xk[i] = 0u;
      }
      if (!(ok = warp_wait(&sm.dkvfull, it & 1, abort, a.err, kSiteDKVFull))) break;
      tc_fence_after();
      {
        // cg 0 published 1/rms of the K rows with kvready of this tile
        if (cg == 1 && !(ok = warp_wait(&sm.kvready, it & 1, abort, a.err, kSiteKVReady))) break;
        const float rinv = sm.rinvk[row];
        const float2 rinv2 = make_float2(rinv, rinv);
        // dK 2^(e_c + k_c) and dV 2^e_c are unscaled in the epilogue: dk is
        // linear in dK, so its factor goes into 1/rms (and the dwk sums)
        const float unk = pow2f(-(ec + kc)), unv = pow2f(-ec);
        const float2 rinvu2 = make_float2(rinv * unk, rinv * unk);
        const float2 unv2 = make_float2(unv, unv);
        // Edge rows (the first n_lo and the last n_hi keys of each sequence)
        // also go out in fp32, [B, n, Hkv, {dk, dv}, D]: a caller that sums
        // partial gradients of the same keys from two calls (sequence
        // sharding) then rounds the sum once.
        float* edge = nullptr;
        if (c.t < 0)  // the halo keys: this chunk's share, always in fp32
          edge = row >= 1 ? a.dkv_halo + hrow * 2 * kHeadDim : nullptr;
        else if (kpos < a.n_lo)
          edge = a.edge_lo +
                 ((static_cast<long long>(c.b) * a.n_lo + kpos) * a.Hkv + c.kvh) * 2 * kHeadDim;
        else if (kpos < a.T && kpos >= a.T - a.n_hi)
          edge = a.edge_hi + ((static_cast<long long>(c.b) * a.n_hi + (kpos - (a.T - a.n_hi))) *
                                  a.Hkv + c.kvh) * 2 * kHeadDim;
        float y[64];
        uint32_t dvw[32];
        {
          uint32_t r[32], r2[32];
          tmem_ld32(t_row + 128 + cg * 64, r);
          tmem_ld32(t_row + 128 + cg * 64 + 32, r2);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            y[i] = __uint_as_float(r[i]);
            y[32 + i] = __uint_as_float(r2[i]);
          }
          tmem_ld32(t_row + cg * 64, r);
          tmem_ld32(t_row + cg * 64 + 32, r2);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 v0 = __fmul2_rn(
                make_float2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1])), unv2);
            const float2 v1 = __fmul2_rn(
                make_float2(__uint_as_float(r2[2 * e]), __uint_as_float(r2[2 * e + 1])), unv2);
            dvw[e] = pack_bf16x2(v0.x, v0.y);
            dvw[16 + e] = pack_bf16x2(v1.x, v1.y);
            if (edge != nullptr) {
              *reinterpret_cast<float2*>(edge + kHeadDim + 64 * cg + 2 * e) = v0;
              *reinterpret_cast<float2*>(edge + kHeadDim + 64 * cg + 32 + 2 * e) = v1;
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&sm.tfree);  // dK and dV have been read from TMEM
        if (own_row) {
          uint8_t* dvrow = reinterpret_cast<uint8_t*>(a.dv + krow * kHeadDim) + 128 * cg;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            st32B(dvrow + 32 * i, *reinterpret_cast<const uint32_t(*)[8]>(dvw + 8 * i));
        }
        if (cg == 0) {  // RoPE^-1 on the rotated pairs, all in the first half
#pragma unroll
          for (int p = 0; p < kPairs; ++p) {
            const float2 rcp = rot_at(sm.rot_hi[it & 1][0], sm.rot, p, row);
            const float a0 = y[p], b0 = y[p + kPairs];
            y[p] = a0 * rcp.x + b0 * rcp.y;  // R^T: (a, b) -> (a cos + b sin, b cos - a sin)
            y[p + kPairs] = b0 * rcp.x - a0 * rcp.y;
          }
        }
        float2 dot2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 xh = __fmul2_rn(bf2(xk[i]), rinv2);  // xhat
          const int d = 64 * cg + 2 * i;
          dot2 = __ffma2_rn(__fmul2_rn(make_float2(y[2 * i], y[2 * i + 1]),
                                       make_float2(sm.wk[d], sm.wk[d + 1])),
                            xh, dot2);
        }
        sm.xt[cg][row] = dot2.x + dot2.y;
        mbar_arrive(&sm.xtb);
        if (!(ok = warp_wait(&sm.xtb, it & 1, abort, a.err, kSiteXchg))) break;
        const float dot = (dot2.x + dot2.y + sm.xt[cg ^ 1][row]) * (1.0f / kHeadDim);
        const float2 ndot2 = make_float2(-dot, -dot);
        uint8_t* out = reinterpret_cast<uint8_t*>(a.dk + krow * kHeadDim) + 128 * cg;
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {  // dx = rinv (w dy - xhat dot), 16 dims at a time
          uint32_t o[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int i = 8 * i4 + e;
            const float2 xh = __fmul2_rn(bf2(xk[i]), rinv2);
            const int d = 64 * cg + 2 * i;
            const float2 yv = make_float2(y[2 * i], y[2 * i + 1]);
            const float2 g = __fmul2_rn(
                rinvu2, __ffma2_rn(xh, ndot2, __fmul2_rn(yv, make_float2(sm.wk[d], sm.wk[d + 1]))));
            o[e] = pack_bf16x2(g.x, g.y);
            if (edge != nullptr) *reinterpret_cast<float2*>(edge + d) = g;
            const float2 cv = __fmul2_rn(yv, xh);  // dw contribution dy * xhat, in place
            y[2 * i] = cv.x;
            y[2 * i + 1] = cv.y;
          }
          if (own_row) st32B(out + 32 * i4, o);
        }
        const float2 sw = warp_reduce_scatter64(y, lane);
        atomicAdd(sm.dw + 64 * cg + 2 * lane, sw.x * unk);
        atomicAdd(sm.dw + 64 * cg + 2 * lane + 1, sw.y * unk);
      }
    }
    if (!in_range) atomicCAS(a.err, 0, kDevErrRange);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (tid >= 128 && tid < 256 && !*abort) atomicAdd(a.dwk + (tid - 128), sm.dw[tid - 128]);
}

template <int kPairs>
int launch_impl(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                const CUtensorMap& tkh, const CUtensorMap& tvh,
                const BwdArgs& a, int num_sms, cudaStream_t stream) {
  const size_t smem_q = sizeof(SmemQ) + 1024, smem_kv = sizeof(SmemKV) + 1024;
  static int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    // The register split (setmaxnreg) assumes each kernel was built with the
    // full launch budget per thread; refuse otherwise.
    cudaFuncAttributes attr, attr_kv;
    cudaError_t e = cudaFuncGetAttributes(&attr, swa_bwd_q_kernel<kPairs>);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&attr_kv, swa_bwd_kv_kernel<kPairs>);
    if (e != cudaSuccess) return map_cuda_error(e);
    if (attr.numRegs != kRegsLaunch || attr_kv.numRegs != kRegsLaunch) return SWA_ERR_UNSUPPORTED;
    e = cudaFuncSetAttribute(swa_bwd_q_kernel<kPairs>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem_q));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(swa_bwd_kv_kernel<kPairs>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_kv));
    if (e != cudaSuccess) return map_cuda_error(e);
    configured_device = dev;
  }
  const long long grid = a.total_tiles < num_sms ? a.total_tiles : num_sms;
  int rc = launch_dependent(swa_bwd_q_kernel<kPairs>, static_cast<unsigned>(grid), kThreads,
                            smem_q, stream, tq, tk, tv, tkh, tvh, a);
  if (rc != SWA_OK) return rc;
  const long long grid_kv = a.kv_total_tiles < num_sms ? a.kv_total_tiles : num_sms;
  return launch_dependent(swa_bwd_kv_kernel<kPairs>, static_cast<unsigned>(grid_kv), kThreads,
                          smem_kv, stream, tq, tk, tv, tkh, tvh, a);
}

}  // namespace bwd

int launch_bwd(const swa_params_t* p, const CUtensorMap& tq, const CUtensorMap& tk,
               const CUtensorMap& tv, const CUtensorMap& tkh, const CUtensorMap& tvh,
               const BwdArgs& a, cudaStream_t stream) {
  DeviceInfo di;
  int rc = current_device_info(&di);
  if (rc != SWA_OK) return rc;
  switch (p->rot_dim) {
    case 0: return bwd::launch_impl<0>(tq, tk, tv, tkh, tvh, a, di.num_sms, stream);
    case 32: return bwd::launch_impl<16>(tq, tk, tv, tkh, tvh, a, di.num_sms, stream);
    case 42: return bwd::launch_impl<21>(tq, tk, tv, tkh, tvh, a, di.num_sms, stream);
    case 48: return bwd::launch_impl<24>(tq, tk, tv, tkh, tvh, a, di.num_sms, stream);
    default: return SWA_ERR_UNSUPPORTED;
  }
}

}  // namespace swa
