// global.cu -- the global causal GQA layers of the hybrid stack, for sm_100a.
//
// ZGCM-1 interleaves its 27 gated sliding-window layers with 5 global layers
// (layers 6, 12, 18, 24, 30: onedev.kr summary, "어떻게 동작하나"): the same
// QK-RMSNorm and partial RoPE on q and k and GQA with 32 query and 8 KV heads
// of dim 128, but every query attends over the whole causal context and
// there is no output gate (jaehun.me review, "How Gated SWA Behaves": global
// layers skip the gate).  They keep every token's K and V ("Why the KV Cache
// Shrinks by 6.4x": the global layers store the whole sequence), so the
// decode step reads a full-length cache.
//
//   q' = RoPE(RMSNorm(q; wq)),  k' = RoPE(RMSNorm(k; wk)),
//   s_ij = scale q'_i . k'_j for j <= i,  O_i = softmax_j(s_i) V.
//
// Four kernels:
//   global_kv_kernel      writes k' (bf16) and v into slots of the caches
//                         [B, Hkv, cap, D]: every prefill token, or each
//                         sequence's new token at its decode position.
//   global_fwd_kernel     causal prefill attention on the tensor cores: reads
//                         K' and V from the caches the kernel above wrote.
//   global_decode_kernel  one decode step, split over chunks of the cache.
//   global_combine_kernel sums the chunks' partial softmax results.
//
// Prefill attention.  A work unit is (query tile t, batch row, KV head, pair
// of query heads); it runs key tiles 0..t.  Persistent CTAs take units in
// order of decreasing t, dealt out in a snake over the CTAs so the long and
// short units even out.  Roles mirror the sliding-window forward: a K and a
// V producer warp (TMA), a Q producer warp (TMA, plus the tile's rotation
// table), one MMA-issuing thread, and two region warpgroups, one per head of
// the pair, each with 256 TMEM columns: S = Q K_j^T (128 columns), P packed
// bf16 over S, O += P V_j (128 columns).  The tensor core alternates between
// the regions: PV_j and QK_{j+1} of one head run while the other head's
// softmax runs.  Q slots, o written over Q and stored by TMA, as there.
//
// Softmax without a running maximum.  After RMSNorm |q'| <= sqrt(D) max|wq|
// and |k'| <= sqrt(D) max|wk|, so every score is below M = scale D max|wq|
// max|wk|; exp2((s - M) log2 e) cannot overflow, and the largest term of a
// row cannot underflow while 2 M log2 e <= 120.  With no running maximum, O
// accumulates across key tiles with no rescaling at all.  Larger weights
// take an exact two-pass form: a first pass over the key tiles finds each
// row's maximum (QK^T only), the second uses it.
#include "decode_internal.h"
#include "global_internal.h"
#include "launch.cuh"
#include "ptx.cuh"
#include "rowops.cuh"
#include "warp_mma.cuh"

namespace swa {
namespace glb {

// ------------------------------------------------------------ KV-cache writer

// One warp per token row: the row's rotation is computed once for its KV
// heads, whose 256-byte rows lie next to each other.
__global__ void __launch_bounds__(256) global_kv_kernel(const GlobalKvArgs a, long long rows) {
  __shared__ __align__(16) float scratch[8][kHeadDim];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long r = static_cast<long long>(blockIdx.x) * 8 + warp;
  if (r >= rows) return;  // warp-uniform
  long long b, t, slot;
  bool zero = false;      // a slot past the prefill in its last tile: zero-filled
  if (a.pos != nullptr) {  // decode: row n, slot pos[n]
    b = r;
    t = r;
    slot = a.pos[r];
    if (slot < 0 || slot >= a.cap) {
      if (lane == 0) atomicCAS(a.err, 0, kDevErrBadPosition);
      return;
    }
  } else {  // prefill: rows (b, t) for t < round_up(T, 128), clipped to the cache
    const long long per = ((a.T + kTile - 1) / kTile) * kTile;
    b = r / per;
    t = r - b * per;
    slot = t;
    if (slot >= a.cap) return;
    zero = t >= a.T;
  }
  float cs = 1.0f, sn = 0.0f;
  if (!zero && lane < a.half_rot)
    rope_cos_sin(static_cast<double>(slot), a.inv_freq[lane], &cs, &sn);
  for (int h = 0; h < a.Hkv; ++h) {
    const long long crow = ((b * a.Hkv + h) * a.cap + slot) * kHeadDim;
    if (zero) {
      *reinterpret_cast<uint2*>(a.k_cache + crow + 4 * lane) = make_uint2(0u, 0u);
      *reinterpret_cast<uint2*>(a.v_cache + crow + 4 * lane) = make_uint2(0u, 0u);
      continue;
    }
    const long long row = (a.pos != nullptr ? (b * a.Hkv + h) : ((b * a.T + t) * a.Hkv + h)) *
                          kHeadDim;
    float x[4];
    load4(a.k + row + 4 * lane, x);
    const uint2 vv = *reinterpret_cast<const uint2*>(a.v + row + 4 * lane);
    norm_rope_row(x, a.wk, a.eps, scratch[warp], lane, a.half_rot, cs, sn);
    *reinterpret_cast<uint2*>(a.k_cache + crow + 4 * lane) =
        make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]));
    *reinterpret_cast<uint2*>(a.v_cache + crow + 4 * lane) = vv;
  }
}

// --------------------------------------------------------- prefill attention

constexpr int kThreads = 384;
constexpr int kRegsLaunch = 168;
constexpr int kRegsControl = 96;   // the producers' and MMA issuer's loops need more than 56
constexpr int kRegsRegion = 200;
static_assert(kRegsControl + 2 * kRegsRegion <= 3 * kRegsLaunch, "register split");
constexpr int kHalfBytes = kTile * 64 * 2;
constexpr int kTileBytes = 2 * kHalfBytes;

struct alignas(1024) Smem {
  uint8_t k[2][kTileBytes];
  uint8_t v[2][kTileBytes];
  uint8_t q[3][kTileBytes];       // head n uses slot n % 3: Q(n), then o(n)
  float2 rot_q[3][kMaxPairs];     // rot(128 t w_p) of the query tile in each Q slot
  float wq[kHeadDim], wk[kHeadDim];
  uint64_t kfull[2], kempty[2], vfull[2], vempty[2];
  uint64_t qfull[3], slotfree[3];
  uint64_t qready[2], sfull[2], pfull[2], ofull[2], ostore[2];
  uint64_t drain, never;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Smem) <= 232448, "shared memory over the 227 KiB per-CTA limit");

enum Site {
  kSiteKEmpty = 0x80, kSiteVEmpty, kSiteSlotFree, kSiteKFull, kSiteVFull, kSiteQFull,
  kSiteQReady, kSiteSFull, kSitePFull, kSiteOFull, kSiteOStore, kSiteForced, kSiteAlign
};

__device__ __forceinline__ uint32_t sw_off(int row, int chunk16) {
  return static_cast<uint32_t>(row * 128 + ((chunk16 ^ (row & 7)) << 4));
}
__device__ __forceinline__ float2 cmul(float2 x, float2 y) {
  return make_float2(x.x * y.x - x.y * y.y, x.x * y.y + x.y * y.x);
}
__device__ __forceinline__ uint64_t desc_kmajor(const uint8_t* tile, int kk) {
  return desc_advance(make_desc_sw128(smem_u32(tile), 16, 1024), (kk >> 2) * kHalfBytes + (kk & 3) * 32);
}
__device__ __forceinline__ uint64_t desc_v(const uint8_t* tile, int kk) {
  return desc_advance(make_desc_sw128(smem_u32(tile), kHalfBytes, 1024), kk * 2048);
}
constexpr uint32_t kIdescQK = make_idesc_bf16(128, 128, false, false);
constexpr uint32_t kIdescPV = make_idesc_bf16(128, 128, false, true);

// A work unit and its place in the CTA's sequence.
struct Unit {
  int b, kvh, t, pair;
};
// The k-th unit of CTA c: units are numbered in order of decreasing query
// tile and dealt in a snake (round k goes to c, or grid-1-c when k is odd).
__device__ __forceinline__ long long unit_index(int k, int c, int grid) {
  return static_cast<long long>(k) * grid + ((k & 1) ? grid - 1 - c : c);
}
__device__ __forceinline__ Unit unit_at(const GlobalFwdArgs& a, long long u) {
  const long long per_t = static_cast<long long>(a.B) * a.Hkv * a.pairs;
  Unit x;
  const long long ti = u / per_t;
  long long rem = u - ti * per_t;
  x.t = a.tiles - 1 - static_cast<int>(ti);
  x.pair = static_cast<int>(rem % a.pairs);
  rem /= a.pairs;
  x.kvh = static_cast<int>(rem % a.Hkv);
  x.b = static_cast<int>(rem / a.Hkv);
  return x;
}
// Query head of region r in unit x; a group with an odd head count repeats
// its last head in the second region and drops that copy's output.
__device__ __forceinline__ int unit_head(const GlobalFwdArgs& a, const Unit& x, int r) {
  return x.kvh * a.G + min(2 * x.pair + r, a.G - 1);
}
__device__ __forceinline__ bool unit_head_real(const GlobalFwdArgs& a, const Unit& x, int r) {
  return 2 * x.pair + r < a.G;
}

template <int kPairs>
struct RowRot {
  float2 r[kPairs > 0 ? kPairs : 1];
};

// Q row in place: q' = RoPE(q / rms(q) * wq), all 128 dims (the K side comes
// from the cache already normalised and rotated).
template <int kPairs>
__device__ __forceinline__ void transform_q_row(uint8_t* tile, int row, const float* wq,
                                                const float2* rtile, const RowRot<kPairs>& rr,
                                                float eps) {
  uint8_t* h0 = tile;
  uint8_t* h1 = tile + kHalfBytes;
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};
#pragma unroll 2
  for (int c = 0; c < 8; ++c) {
    const uint4 x = *reinterpret_cast<const uint4*>(h0 + sw_off(row, c));
    const uint4 y = *reinterpret_cast<const uint4*>(h1 + sw_off(row, c));
    const uint32_t w[8] = {x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 f = make_float2(bf16_lo(w[i]), bf16_hi(w[i]));
      acc[i & 3] = __ffma2_rn(f, f, acc[i & 3]);
    }
  }
  const float2 s2 = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
  const float rinv = rsqrtf((s2.x + s2.y) * (1.0f / kHeadDim) + eps);
  constexpr int kRopeChunks = (2 * kPairs + 7) / 8;
  if constexpr (kRopeChunks > 0) {
    float x[kRopeChunks * 8];
#pragma unroll
    for (int c = 0; c < kRopeChunks; ++c) {
      const uint4 u = *reinterpret_cast<const uint4*>(h0 + sw_off(row, c));
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[8 * c + 2 * e] = bf16_lo(w4[e]) * rinv * wq[8 * c + 2 * e];
        x[8 * c + 2 * e + 1] = bf16_hi(w4[e]) * rinv * wq[8 * c + 2 * e + 1];
      }
    }
#pragma unroll
    for (int p = 0; p < kPairs; ++p) {
      const float2 t = cmul(rtile[p], rr.r[p]);  // rot((128 t + row) w_p)
      const float u = x[p], v = x[p + kPairs];
      x[p] = u * t.x - v * t.y;
      x[p + kPairs] = v * t.x + u * t.y;
    }
#pragma unroll
    for (int c = 0; c < kRopeChunks; ++c) {
      uint4 o;
      o.x = pack_bf16x2(x[8 * c], x[8 * c + 1]);
      o.y = pack_bf16x2(x[8 * c + 2], x[8 * c + 3]);
      o.z = pack_bf16x2(x[8 * c + 4], x[8 * c + 5]);
      o.w = pack_bf16x2(x[8 * c + 6], x[8 * c + 7]);
      *reinterpret_cast<uint4*>(h0 + sw_off(row, c)) = o;
    }
  }
  const float2 rv = make_float2(rinv, rinv);
#pragma unroll 1
  for (int c = kRopeChunks; c < 16; ++c) {
    uint8_t* p = (c < 8 ? h0 : h1) + sw_off(row, c & 7);
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const float4 wa = *reinterpret_cast<const float4*>(wq + 8 * c);
    const float4 wb = *reinterpret_cast<const float4*>(wq + 8 * c + 4);
    const float2 y0 = __fmul2_rn(__fmul2_rn(make_float2(bf16_lo(u.x), bf16_hi(u.x)),
                                            make_float2(wa.x, wa.y)), rv);
    const float2 y1 = __fmul2_rn(__fmul2_rn(make_float2(bf16_lo(u.y), bf16_hi(u.y)),
                                            make_float2(wa.z, wa.w)), rv);
    const float2 y2 = __fmul2_rn(__fmul2_rn(make_float2(bf16_lo(u.z), bf16_hi(u.z)),
                                            make_float2(wb.x, wb.y)), rv);
    const float2 y3 = __fmul2_rn(__fmul2_rn(make_float2(bf16_lo(u.w), bf16_hi(u.w)),
                                            make_float2(wb.z, wb.w)), rv);
    uint4 o;
    o.x = pack_bf16x2(y0.x, y0.y);
    o.y = pack_bf16x2(y1.x, y1.y);
    o.z = pack_bf16x2(y2.x, y2.y);
    o.w = pack_bf16x2(y3.x, y3.y);
    *reinterpret_cast<uint4*>(p) = o;
  }
}

template <int kPairs>
__global__ void __launch_bounds__(kThreads, 1)
    global_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_o, const GlobalFwdArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_u32(smem_raw) & 1023u) {
    if (tid == 0) atomicCAS(a.err, 0, kDevErrTimeoutBase + kSiteAlign);
    return;
  }
  const int grid = static_cast<int>(gridDim.x), cta = static_cast<int>(blockIdx.x);
  int n_units = 0;  // units of this CTA: the snake's rounds until the first past the end
  while (unit_index(n_units, cta, grid) < a.units) ++n_units;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.kfull[i], 1);
      mbar_init(&sm.kempty[i], 1);
      mbar_init(&sm.vfull[i], 1);
      mbar_init(&sm.vempty[i], 1);
      mbar_init(&sm.qready[i], 128);
      mbar_init(&sm.sfull[i], 1);
      mbar_init(&sm.pfull[i], 128);
      mbar_init(&sm.ofull[i], 1);
      mbar_init(&sm.ostore[i], 128);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&sm.qfull[i], 2);  // the copy's expect_tx arrive + the rotation table
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
    prefetch_tensormap(&tm_o);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  // A programmatic dependent of the cache writer before it on the stream:
  // every global access below waits for it to complete.
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

  // Every role derives the same bound and the same pass count.
  float wmq = 0.f, wmk = 0.f;
  for (int d = 0; d < kHeadDim; ++d) {
    wmq = fmaxf(wmq, fabsf(sm.wq[d]));
    wmk = fmaxf(wmk, fabsf(sm.wk[d]));
  }
  // in log2 units, with a 1/64 margin for the bf16 rounding of q' and k'
  const float bound = a.scale_log2 * kHeadDim * wmq * wmk * (1.0f + 1.0f / 64.0f);
  const int passes = (2.0f * bound <= 120.0f) ? 1 : 2;

  if (warp < 4) {
    regs_dec<kRegsControl>();
    if ((warp == 0 || warp == 3) && lane == 0) {
      // ---------------------------------------------- K (warp 0) / V (warp 3)
      const bool is_k = warp == 0;
      uint64_t* full = is_k ? sm.kfull : sm.vfull;
      uint64_t* empty = is_k ? sm.kempty : sm.vempty;
      const CUtensorMap* map = is_k ? &tm_k : &tm_v;
      uint8_t(*ring)[kTileBytes] = is_k ? sm.k : sm.v;
      long long cnt = 0;  // tiles loaded
      bool ok = true;
      for (int k = 0; k < n_units && ok; ++k) {
        const Unit x = unit_at(a, unit_index(k, cta, grid));
        const int np = is_k ? passes : 1;  // V serves only the last pass
        for (int pass = 0; pass < np && ok; ++pass) {
          for (int j = 0; j <= x.t; ++j, ++cnt) {
            const int s = static_cast<int>(cnt & 1);
            if (cnt >= 2 && !(ok = mbar_wait_inl(&empty[s], static_cast<uint32_t>((cnt >> 1) - 1) & 1,
                                                 abort, a.err, is_k ? kSiteKEmpty : kSiteVEmpty)))
              break;
            mbar_arrive_expect_tx(&full[s], kTileBytes);
            tma_load_4d(ring[s], map, &full[s], 0, j * kTile, x.kvh, x.b);
            tma_load_4d(ring[s] + kHalfBytes, map, &full[s], 64, j * kTile, x.kvh, x.b);
          }
        }
      }
      if (!ok) {  // drain the copies issued into each slot
        for (int s = 0; s < 2; ++s) {
          const long long issued = (cnt - s + 1) / 2;
          if (issued > 0) mbar_wait_drain(&full[s], static_cast<uint32_t>(issued - 1) & 1);
        }
      }
    } else if (warp == 2) {
      // ------------------------------------------------------- Q producer
      bool ok = true;
      int nq = 0;
      auto wait0 = [&](uint64_t* bar, uint32_t par, int site) -> bool {
        bool w = true;
        if (lane == 0) w = mbar_wait_inl(bar, par, abort, a.err, site);
        return __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
      };
      for (int k = 0; k < n_units && ok; ++k) {
        const Unit x = unit_at(a, unit_index(k, cta, grid));
        for (int r = 0; r < 2 && ok; ++r, ++nq) {
          const int qs = nq % 3;
          if (nq >= 3 && !(ok = wait0(&sm.slotfree[qs], ((nq / 3) - 1) & 1, kSiteSlotFree))) break;
          if (lane == 0) {
            const int hq = unit_head(a, x, r);
            mbar_arrive_expect_tx(&sm.qfull[qs], kTileBytes);
            tma_load_4d(sm.q[qs], &tm_q, &sm.qfull[qs], 0, hq, x.t * kTile, x.b);
            tma_load_4d(sm.q[qs] + kHalfBytes, &tm_q, &sm.qfull[qs], 64, hq, x.t * kTile, x.b);
          }
          if (lane < kPairs) {
            float cv, sv;
            rope_cos_sin(static_cast<double>(x.t) * kTile, a.inv_freq[lane], &cv, &sv);
            sm.rot_q[qs][lane] = make_float2(cv, sv);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.qfull[qs]);
        }
      }
      if (!ok && lane == 0) {
        for (int s = 0; s < 3; ++s) {
          const int cntq = (nq - s + 2) / 3;
          if (cntq > 0) mbar_wait_drain(&sm.qfull[s], static_cast<uint32_t>(cntq - 1) & 1);
        }
      }
      __syncwarp();
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------- MMA issuer
      bool ok = true;
      if (a.flags & SWA_FLAG_FORCE_TIMEOUT) ok = mbar_wait_inl(&sm.never, 0, abort, a.err, kSiteForced);
      long long kc = 0, vc = 0;  // K and V tiles consumed
      int pc[2] = {0, 0};        // P (or S consumed) completions per region
      auto W = [&](uint64_t* bar, uint32_t par, int site) {
        if (ok) ok = mbar_wait_inl(bar, par, abort, a.err, site);
        return ok;
      };
      auto qk = [&](int r, int qslot) {
        const uint8_t* kt = sm.k[kc & 1];
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + r * 256, desc_kmajor(sm.q[qslot], kk), desc_kmajor(kt, kk), kIdescQK,
                 kk > 0);
        mma_commit(&sm.sfull[r]);
      };
      for (int k = 0; k < n_units && ok; ++k) {
        const Unit x = unit_at(a, unit_index(k, cta, grid));
        const int q0 = (2 * k) % 3, q1 = (2 * k + 1) % 3;
        for (int pass = 0; pass < passes && ok; ++pass) {
          const bool last = pass == passes - 1;
          if (!W(&sm.kfull[kc & 1], static_cast<uint32_t>(kc >> 1) & 1, kSiteKFull)) break;
          // each region's Q is waited for on its own, so region 0 never waits
          // on region 1's epilogue of the unit before
          if (pass == 0 && !W(&sm.qready[0], k & 1, kSiteQReady)) break;
          tc_fence_after();
          qk(0, q0);
          if (pass == 0 && !W(&sm.qready[1], k & 1, kSiteQReady)) break;
          tc_fence_after();
          qk(1, q1);
          mma_commit(&sm.kempty[kc & 1]);
          ++kc;
          for (int j = 0; j <= x.t && ok; ++j) {
            for (int r = 0; r < 2 && ok; ++r) {
              if (!W(&sm.pfull[r], pc[r] & 1, kSitePFull)) break;
              ++pc[r];
              tc_fence_after();
              if (last) {
                if (r == 0 && !W(&sm.vfull[vc & 1], static_cast<uint32_t>(vc >> 1) & 1, kSiteVFull))
                  break;
                tc_fence_after();
                const uint8_t* vt = sm.v[vc & 1];
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                  mma_ts(tmem + r * 256 + 128, tmem + r * 256 + kk * 8, desc_v(vt, kk), kIdescPV,
                         (j > 0 || kk > 0) ? 1u : 0u);
                if (j == x.t) mma_commit(&sm.ofull[r]);
                if (r == 1) {
                  mma_commit(&sm.vempty[vc & 1]);
                  ++vc;
                }
              }
              if (j < x.t) {
                if (r == 0 && !W(&sm.kfull[kc & 1], static_cast<uint32_t>(kc >> 1) & 1, kSiteKFull))
                  break;
                tc_fence_after();
                qk(r, r == 0 ? q0 : q1);
                if (r == 1) {
                  mma_commit(&sm.kempty[kc & 1]);
                  ++kc;
                }
              }
            }
          }
        }
      }
      if (!ok) {
        mma_commit(&sm.drain);
        mbar_wait_drain(&sm.drain, 0);
      }
    }
    __syncwarp();
  } else {
    // ----------------------------------------------------------- regions
    regs_inc<kRegsRegion>();
    const int r = (warp - 4) >> 2;
    const int wq4 = warp & 3;
    const int row = wq4 * 32 + lane;
    const uint32_t t_row = tmem + (static_cast<uint32_t>(wq4 * 32) << 16) + r * 256;
    RowRot<kPairs> rr;
#pragma unroll
    for (int p = 0; p < kPairs; ++p) {
      float cv, sv;
      rope_cos_sin(static_cast<double>(row), a.inv_freq[p], &cv, &sv);
      rr.r[p] = make_float2(cv, sv);
    }
    const float sl2 = a.scale_log2;
    const bool elected = row == 0;
    bool ok = true;
    int scnt = 0;  // S tiles consumed by this region
    const uint32_t zero16[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u,
                                 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    for (int k = 0; k < n_units && ok; ++k) {
      const Unit x = unit_at(a, unit_index(k, cta, grid));
      const int n = 2 * k + r;
      const int qs = n % 3;
      const uint32_t qph = static_cast<uint32_t>(n / 3) & 1;
      const int hq = unit_head(a, x, r);
      const long long pos = static_cast<long long>(x.t) * kTile + row;

      // ---- Q(n): normalised, scaled and rotated in place
      if (!(ok = mbar_wait_inl(&sm.qfull[qs], qph, abort, a.err, kSiteQFull))) break;
      transform_q_row<kPairs>(sm.q[qs], row, sm.wq, sm.rot_q[qs], rr, a.eps);
      fence_proxy_async_smem();
      mbar_arrive(&sm.qready[r]);

      float ms = bound;  // subtracted in log2 units (the row maximum in the exact form)
      float2 l2 = make_float2(0.f, 0.f);
      for (int pass = 0; pass < passes && ok; ++pass) {
        const bool last = pass == passes - 1;
        float m = -INFINITY;
        const float2 sc2 = make_float2(sl2, sl2), nms2 = make_float2(-ms, -ms);
        for (int j = 0; j <= x.t; ++j) {
          if (!(ok = mbar_wait_inl(&sm.sfull[r], scnt & 1, abort, a.err, kSiteSFull))) break;
          ++scnt;
          tc_fence_after();
          const bool diag = j == x.t;
          const int nch = diag ? wq4 + 1 : 4;  // chunks that reach the causal edge
#pragma unroll 1
          for (int pc = 0; pc < nch; ++pc) {
            uint32_t v[32];
            tmem_ld32(t_row + pc * 32, v);
            tmem_wait_ld();
            const bool edge = diag && pc == wq4;
            if (!last) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (!edge || pc * 32 + i <= row) m = fmaxf(m, __uint_as_float(v[i]));
            } else {
              uint32_t pk[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const float2 z = __ffma2_rn(
                    make_float2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1])), sc2,
                    nms2);
                float2 p = make_float2(ex2_approx(z.x), ex2_approx(z.y));
                if (edge) {
                  const int c0 = pc * 32 + 2 * e;
                  p = make_float2(c0 <= row ? p.x : 0.f, c0 + 1 <= row ? p.y : 0.f);
                }
                l2 = __fadd2_rn(l2, p);
                pk[e] = pack_bf16x2(p.x, p.y);
              }
              // P over S's first 64 columns: chunk pc lands in columns this
              // thread has already read (16 pc .. 16 pc + 15 < 32 (pc + 1)).
              tmem_st16(t_row + pc * 16, pk);
            }
          }
          if (last) {
            for (int pc = nch; pc < 4; ++pc) tmem_st16(t_row + pc * 16, zero16);
            tmem_wait_st();
          }
          tc_fence_before();
          mbar_arrive(&sm.pfull[r]);
        }
        if (!last) ms = m * sl2;
      }
      if (!ok) break;

      // ---- epilogue: o = O / l over Q(n)'s slot, stored by TMA
      if (!(ok = mbar_wait_inl(&sm.ofull[r], k & 1, abort, a.err, kSiteOFull))) break;
      tc_fence_after();
      const float l = l2.x + l2.y;
      const float il = 1.0f / l;
      if (a.lse != nullptr && pos < a.T && unit_head_real(a, x, r))
        a.lse[(static_cast<long long>(x.b) * a.Hq + hq) * a.T + pos] =
            (ms + __log2f(l)) * 0.6931471805599453f;
      const float2 il2 = make_float2(il, il);
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t ov[32];
        tmem_ld32(t_row + 128 + ch * 32, ov);
        tmem_wait_ld();
        uint8_t* half = sm.q[qs] + (ch >> 1) * kHalfBytes;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 o2 = __fmul2_rn(make_float2(__uint_as_float(ov[8 * i + 2 * e]),
                                                     __uint_as_float(ov[8 * i + 2 * e + 1])),
                                         il2);
            w[e] = pack_bf16x2(o2.x, o2.y);
          }
          *reinterpret_cast<uint4*>(half + sw_off(row, (ch & 1) * 4 + i)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(&sm.ostore[r]);
      if (elected) {
        if (!(ok = mbar_wait_inl(&sm.ostore[r], k & 1, abort, a.err, kSiteOStore))) break;
        if (unit_head_real(a, x, r)) {
          tma_store_4d(&tm_o, sm.q[qs], 0, hq, x.t * kTile, x.b);
          tma_store_4d(&tm_o, sm.q[qs] + kHalfBytes, 64, hq, x.t * kTile, x.b);
          bulk_commit();
          bulk_wait_read<0>();
        }
        mbar_arrive(&sm.slotfree[qs]);
      }
    }
    if (elected) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ decode

constexpr int kDecThreads = 160;                // producer warp + 4 consumer warps
constexpr int kDecStages = 3;
constexpr int kRingHalf = kTile * 64 * 2;       // 128 keys x 64 dims bf16 (one TMA box)
constexpr int kQStride = 68;                    // words per packed q' row (bank padding)
constexpr int kOStride = 136;                   // floats per partial-O row (padding)

struct alignas(1024) DecStage {
  uint8_t k[2][kRingHalf];
  uint8_t v[2][kRingHalf];
};
struct alignas(1024) DecSmem {
  DecStage st[kDecStages];
  uint32_t qa[kGlobalMaxGroup][kQStride];
  float scratch[4][kHeadDim];
  float mw[4][kGlobalMaxGroup], lw[4][kGlobalMaxGroup];
  uint64_t full[kDecStages], empty[kDecStages];
  uint64_t never;
  int abort;
};
static_assert(4 * kGlobalMaxGroup * kOStride * 4 <= sizeof(DecStage), "partial O");
static_assert(sizeof(DecSmem) + 1024 <= 232448, "decode shared memory");

enum DecSite { kSiteDFull = 0xA0, kSiteDEmpty, kSiteDForced };

__device__ __forceinline__ uint32_t ring_off(int s, int c) {
  return static_cast<uint32_t>((c >> 3) * kRingHalf + s * 128 + (((c & 7) ^ (s & 7)) << 4));
}

// Barrier over the 128 consumer threads (named barrier 1).
__device__ __forceinline__ void consumers_sync() { named_sync(1, 128); }

// One CTA per (sequence, KV head, chunk of kGlobalChunk keys).  The chunk's
// keys [c0, min(c0 + chunk, pos + 1)) arrive in tiles of 128 by TMA; warp w
// scores keys 32 w .. 32 w + 31 of each tile with mma.sync (the group's query
// heads are the M rows, padded to 16), keeps a running maximum, rescales its
// partial O, and the four warps' partials are merged at the end into the
// chunk's (max, sum, O) in the workspace.
__global__ void __launch_bounds__(kDecThreads, 1)
    global_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const GlobalDecArgs a) {
  extern __shared__ uint8_t smem_raw[];
  DecSmem& sm = *reinterpret_cast<DecSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long item = blockIdx.x;
  const int c = static_cast<int>(item % a.chunks);
  const long long nk = item / a.chunks;
  const int kvh = static_cast<int>(nk % a.Hkv);
  const int n = static_cast<int>(nk / a.Hkv);
  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.never, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort = &sm.abort;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const long long p = a.pos[n];
  const long long c0 = static_cast<long long>(c) * kGlobalChunk;
  if (p < 0 || p >= a.cap) {  // reported by the cache writer before this kernel
    return;
  }
  if (c0 > p) return;  // the whole CTA: no key of this chunk is in the context
  const long long c1 = min(c0 + kGlobalChunk, p + 1);  // keys [c0, c1)
  const int ntile = static_cast<int>((c1 - c0 + kTile - 1) / kTile);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      bool ok = true;
      int i = 0;
      for (; i < ntile; ++i) {
        const int s = i % kDecStages;
        if (i >= kDecStages &&
            !(ok = mbar_wait(&sm.empty[s], ((i / kDecStages) - 1) & 1, abort, a.err, kSiteDEmpty)))
          break;
        const int key = static_cast<int>(c0) + i * kTile;
        mbar_arrive_expect_tx(&sm.full[s], 4 * kRingHalf);
        tma_load_4d(sm.st[s].k[0], &tm_k, &sm.full[s], 0, key, kvh, n);
        tma_load_4d(sm.st[s].k[1], &tm_k, &sm.full[s], 64, key, kvh, n);
        tma_load_4d(sm.st[s].v[0], &tm_v, &sm.full[s], 0, key, kvh, n);
        tma_load_4d(sm.st[s].v[1], &tm_v, &sm.full[s], 64, key, kvh, n);
      }
      if (!ok) {
        for (int s = 0; s < kDecStages; ++s) {
          const int issued = (i - s + kDecStages - 1) / kDecStages;
          if (issued > 0) mbar_wait_drain(&sm.full[s], (issued - 1) & 1);
        }
      }
    }
    __syncwarp();
    return;
  }
  // ------------------------------------------------------------- consumers
  const int lw = warp - 1;
  // q' for heads lw, lw + 4 at position p
  {
    float cs = 1.0f, sn = 0.0f;
    if (lane < a.half_rot) rope_cos_sin(static_cast<double>(p), a.inv_freq[lane], &cs, &sn);
    for (int h = lw; h < a.G; h += 4) {
      float x[4];
      load4(a.q + (static_cast<long long>(n) * a.Hq + kvh * a.G + h) * kHeadDim + 4 * lane, x);
      norm_rope_row(x, a.wq, a.eps, sm.scratch[lw], lane, a.half_rot, cs, sn);
      sm.qa[h][2 * lane] = pack_bf16x2(x[0], x[1]);
      sm.qa[h][2 * lane + 1] = pack_bf16x2(x[2], x[3]);
    }
  }
  bool ok = true;
  if (a.flags & SWA_FLAG_FORCE_TIMEOUT) ok = mbar_wait(&sm.never, 0, abort, a.err, kSiteDForced);
  consumers_sync();  // q' visible to every consumer warp
  const int grp = lane >> 2, tig = lane & 3;
  const bool row_ok = grp < a.G;
  float m = -INFINITY, l = 0.0f;  // this lane's head row grp, over this warp's keys
  float oacc[16][4];
#pragma unroll
  for (int nd = 0; nd < 16; ++nd) oacc[nd][0] = oacc[nd][1] = oacc[nd][2] = oacc[nd][3] = 0.0f;
  int i = 0;
  for (; i < ntile && ok; ++i) {
    const int s = i % kDecStages;
    ok = __all_sync(0xffffffffu, mbar_wait(&sm.full[s], (i / kDecStages) & 1, abort, a.err,
                                           kSiteDFull));
    if (!ok) break;
    DecStage& st = sm.st[s];
    const long long key0 = c0 + static_cast<long long>(i) * kTile;  // key of slot 0
    // Slots past the context (after position p) may hold stale values, which
    // must not reach P V even with P = 0: this warp zeroes its own V rows there.
    {
      const long long kk = key0 + 32 * lw + lane;
      if (kk > p) {
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int cc = 0; cc < 16; ++cc)
          *reinterpret_cast<uint4*>(&st.v[0][0] + ring_off(32 * lw + lane, cc)) = z;
        fence_proxy_async_smem();  // before a later TMA copy into this stage
      }
      __syncwarp();
    }
    // S = q' K^T over this warp's 32 keys
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
    const uint32_t kbase = smem_u32(st.k[0]);
#pragma unroll
    for (int kp2 = 0; kp2 < 4; ++kp2) {
      uint32_t qa0[2], qa2[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int kk = 2 * kp2 + e;
        qa0[e] = row_ok ? sm.qa[grp][8 * kk + tig] : 0u;
        qa2[e] = row_ok ? sm.qa[grp][8 * kk + 4 + tig] : 0u;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t b[4];
        const int slot = 32 * lw + 8 * j + (lane & 7);
        ldsm_x4(kbase + ring_off(slot, 4 * kp2 + (lane >> 3)), b);
        mma_16816(acc[j], qa0[0], 0u, qa2[0], 0u, b[0], b[1]);
        mma_16816(acc[j], qa0[1], 0u, qa2[1], 0u, b[2], b[3]);
      }
    }
    // running maximum and rescale (log2 units)
    float tm = -INFINITY;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const long long key = key0 + 32 * lw + 8 * j + 2 * tig + e;
        acc[j][e] = key <= p ? acc[j][e] * a.scale_log2 : -INFINITY;
        tm = fmaxf(tm, acc[j][e]);
      }
    }
    tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 1));
    tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 2));
    const float mn = fmaxf(m, tm);
    const float mu = mn == -INFINITY ? 0.0f : mn;
    const float corr = m == -INFINITY ? 0.0f : ex2_approx(m - mu);
    m = mn;
    l *= corr;
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) {
      oacc[nd][0] *= corr;
      oacc[nd][1] *= corr;
    }
    uint32_t pa[4];
    float ls = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float p0 = ex2_approx(acc[j][0] - mu), p1 = ex2_approx(acc[j][1] - mu);
      ls += p0 + p1;
      pa[j] = pack_bf16x2(p0, p1);
    }
    ls += __shfl_xor_sync(0xffffffffu, ls, 1);
    ls += __shfl_xor_sync(0xffffffffu, ls, 2);
    l += ls;
    if (!row_ok) pa[0] = pa[1] = pa[2] = pa[3] = 0u;
    const uint32_t vbase = smem_u32(st.v[0]);
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) {
      uint32_t b[4];
      ldsm_x4_trans(vbase + ring_off(32 * lw + lane, nd), b);
      mma_16816(oacc[nd], pa[0], 0u, pa[1], 0u, b[0], b[1]);
      mma_16816(oacc[nd], pa[2], 0u, pa[3], 0u, b[2], b[3]);
    }
    __syncwarp();
    // every warp's reads of this stage are done before the producer refills it
    consumers_sync();
    if (lw == 0 && lane == 0) mbar_arrive(&sm.empty[i % kDecStages]);
  }
  ok = __all_sync(0xffffffffu, ok);
  // ---- merge the four warps' partials into the chunk's (m, l, O)
  const int last_stage = (i + kDecStages - 1) % kDecStages;  // its reads are done: reuse it
  float* part = reinterpret_cast<float*>(&sm.st[last_stage]);
  if (tig == 0 && row_ok) {
    sm.mw[lw][grp] = m;
    sm.lw[lw][grp] = l;
  }
  if (row_ok) {
#pragma unroll
    for (int nd = 0; nd < 16; ++nd)
      *reinterpret_cast<float2*>(part + (lw * kGlobalMaxGroup + grp) * kOStride + 8 * nd + 2 * tig) =
          make_float2(oacc[nd][0], oacc[nd][1]);
  }
  consumers_sync();
  if (!ok) return;
  for (int h = lw; h < a.G; h += 4) {
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) mx = fmaxf(mx, sm.mw[w][h]);
    const float mu = mx == -INFINITY ? 0.0f : mx;
    float f[4], lsum = 0.0f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      f[w] = sm.mw[w][h] == -INFINITY ? 0.0f : ex2_approx(sm.mw[w][h] - mu);
      lsum += f[w] * sm.lw[w][h];
    }
    float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float4 v4 =
          *reinterpret_cast<const float4*>(part + (w * kGlobalMaxGroup + h) * kOStride + 4 * lane);
      y[0] += f[w] * v4.x;
      y[1] += f[w] * v4.y;
      y[2] += f[w] * v4.z;
      y[3] += f[w] * v4.w;
    }
    const long long slot = ((static_cast<long long>(n) * a.Hkv + kvh) * a.chunks + c) * a.G + h;
    *reinterpret_cast<float4*>(a.part_o + slot * kHeadDim + 4 * lane) =
        make_float4(y[0], y[1], y[2], y[3]);
    if (lane == 0) *reinterpret_cast<float2*>(a.part_ml + slot * 2) = make_float2(mx, lsum);
  }
}

// One warp per (sequence, query head): o = sum_c 2^(m_c - m) O_c / sum_c 2^(m_c - m) l_c.
__global__ void __launch_bounds__(256) global_combine_kernel(const GlobalDecArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long r = static_cast<long long>(blockIdx.x) * 8 + warp;
  if (r >= static_cast<long long>(a.N) * a.Hq) return;
  const int n = static_cast<int>(r / a.Hq), hq = static_cast<int>(r % a.Hq);
  const int kvh = hq / a.G, h = hq - kvh * a.G;
  const long long p = a.pos[n];
  if (p < 0 || p >= a.cap) return;
  const int nc = static_cast<int>(p / kGlobalChunk) + 1;
  const long long base = (static_cast<long long>(n) * a.Hkv + kvh) * a.chunks;
  float mx = -INFINITY;
  for (int c = 0; c < nc; ++c) mx = fmaxf(mx, a.part_ml[((base + c) * a.G + h) * 2]);
  float y[4] = {0.f, 0.f, 0.f, 0.f}, lsum = 0.0f;
  for (int c = 0; c < nc; ++c) {
    const long long slot = (base + c) * a.G + h;
    const float2 ml = *reinterpret_cast<const float2*>(a.part_ml + slot * 2);
    const float f = ml.x == -INFINITY ? 0.0f : ex2_approx(ml.x - mx);
    lsum += f * ml.y;
    const float4 v4 = *reinterpret_cast<const float4*>(a.part_o + slot * kHeadDim + 4 * lane);
    y[0] += f * v4.x;
    y[1] += f * v4.y;
    y[2] += f * v4.z;
    y[3] += f * v4.w;
  }
  const float il = 1.0f / lsum;
  *reinterpret_cast<uint2*>(a.o + r * kHeadDim + 4 * lane) =
      make_uint2(pack_bf16x2(y[0] * il, y[1] * il), pack_bf16x2(y[2] * il, y[3] * il));
}

template <int kPairs>
int launch_fwd_impl(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                    const CUtensorMap& to, const GlobalFwdArgs& a, int num_sms,
                    cudaStream_t stream) {
  const size_t smem = sizeof(Smem);
  static int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaFuncAttributes attr;
    cudaError_t e = cudaFuncGetAttributes(&attr, global_fwd_kernel<kPairs>);
    if (e != cudaSuccess) return map_cuda_error(e);
    if (attr.numRegs != kRegsLaunch) return SWA_ERR_UNSUPPORTED;
    e = cudaFuncSetAttribute(global_fwd_kernel<kPairs>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return map_cuda_error(e);
    configured_device = dev;
  }
  const long long grid = a.units < num_sms ? a.units : num_sms;
  return launch_dependent(global_fwd_kernel<kPairs>, static_cast<unsigned>(grid), kThreads, smem,
                          stream, tq, tk, tv, to, a);
}

}  // namespace glb

int launch_global_kv(const GlobalKvArgs& a, long long rows, cudaStream_t stream) {
  const long long grid = (rows + 7) / 8;
  if (grid > 0x7fffffffLL) return SWA_ERR_UNSUPPORTED;
  if (grid == 0) return SWA_OK;
  return launch_dependent(glb::global_kv_kernel, static_cast<unsigned>(grid), 256, 0, stream, a,
                          rows);
}

int launch_global_fwd(int rot_dim, const CUtensorMap& tq, const CUtensorMap& tk,
                      const CUtensorMap& tv, const CUtensorMap& to, const GlobalFwdArgs& a,
                      cudaStream_t stream) {
  DeviceInfo di;
  int rc = current_device_info(&di);
  if (rc != SWA_OK) return rc;
  switch (rot_dim) {
    case 0: return glb::launch_fwd_impl<0>(tq, tk, tv, to, a, di.num_sms, stream);
    case 32: return glb::launch_fwd_impl<16>(tq, tk, tv, to, a, di.num_sms, stream);
    case 42: return glb::launch_fwd_impl<21>(tq, tk, tv, to, a, di.num_sms, stream);
    case 48: return glb::launch_fwd_impl<24>(tq, tk, tv, to, a, di.num_sms, stream);
    default: return SWA_ERR_UNSUPPORTED;
  }
}

int launch_global_decode(const CUtensorMap& tk, const CUtensorMap& tv, const GlobalDecArgs& a,
                         cudaStream_t stream) {
  DeviceInfo di;
  int rc = current_device_info(&di);
  if (rc != SWA_OK) return rc;
  const size_t smem = sizeof(glb::DecSmem) + 1024;
  static int configured_device = -1;
  if (configured_device != di.device) {
    cudaError_t e = cudaFuncSetAttribute(glb::global_decode_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return map_cuda_error(e);
    configured_device = di.device;
  }
  const long long items = static_cast<long long>(a.N) * a.Hkv * a.chunks;
  if (items > 0x7fffffffLL) return SWA_ERR_UNSUPPORTED;
  rc = launch_dependent(glb::global_decode_kernel, static_cast<unsigned>(items), glb::kDecThreads,
                        smem, stream, tk, tv, a);
  if (rc != SWA_OK) return rc;
  const long long rows = static_cast<long long>(a.N) * a.Hq;
  return launch_dependent(glb::global_combine_kernel, static_cast<unsigned>((rows + 7) / 8), 256, 0,
                          stream, a);
}

}  // namespace swa
