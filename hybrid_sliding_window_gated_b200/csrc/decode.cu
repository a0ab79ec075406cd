// decode.cu -- one decode step of the gated sliding-window attention core
// against per-sequence 128-slot K/V rings, for sm_100a.
//
// For each sequence n with new token at position p (ZGCM-1 pages: onedev.kr
// summary, "어떻게 동작하나" -- decoding is memory-bandwidth bound; jaehun.me
// review, "Why the KV Cache Shrinks by 6.4x" -- a window layer keeps only its
// last W tokens):
//   k' = RoPE_p(RMSNorm(k_new)) is written to ring slot p mod W, v_new too;
//   q' = RoPE_p(RMSNorm(q)) attends over the W slots, slot s holding position
//   p - ((p - s) mod W) (ignored when negative);  o = A * sigmoid(g).
//
// One CTA per (sequence, KV head): the 32 KiB K ring and 32 KiB V ring arrive
// by TMA (128-byte swizzle) while the warps normalise and rotate q and k_new.
// Warp w takes slots 32w .. 32w+31: S = q' K^T and the partial P V run on the
// tensor cores with mma.sync (the G <= 8 query heads of the group are the M
// rows, zero-padded to 16), with a per-warp maximum; the four partial results
// are combined in shared memory (split-K softmax), scaled by 1/l and gated.
// The warp owning slot p mod W patches that row, in shared memory and in the
// ring, with k' (rounded to bf16) and v_new before reading it.
#include "decode_internal.h"
#include "ptx.cuh"
#include "warp_mma.cuh"

namespace swa {
namespace dec {

constexpr int kThreads = 128;
constexpr int kHalfBytes = kWindow * 64 * 2;  // 128 slots x 64 dims of bf16 (one TMA box)
constexpr int kQStride = 68;                  // words per packed q' row (bank-conflict padding)
constexpr int kOStride = 136;                 // floats per partial-O row (padding)

struct alignas(1024) Smem {
  uint8_t k[2][kHalfBytes];  // K ring, dims 0..63 and 64..127, 128B-swizzled
  uint8_t v[2][kHalfBytes];  // V ring
  uint32_t qa[kDecMaxGroup][kQStride];  // q' as packed bf16 pairs
  float scratch[4][kHeadDim];           // per-warp norm / RoPE staging
  float mw[4][kDecMaxGroup];            // per-warp row maxima (log2 units)
  float lw[4][kDecMaxGroup];            // per-warp row sums
  uint64_t kfull, vfull;
  int abort;
};
// The partial outputs [4 warps][G heads][kOStride] reuse the K ring once the
// scores are done.
static_assert(4 * kDecMaxGroup * kOStride * 4 <= 2 * kHalfBytes, "partial O does not fit");
static_assert(sizeof(Smem) + 1024 <= 113 * 1024, "decode smem should allow two CTAs per SM");

enum Site { kSiteKFull = 0x40, kSiteVFull };

// Byte offset of 16-byte chunk c (0..15) of slot row s in a [half][slot][64]
// 128B-swizzled ring tile.
__device__ __forceinline__ uint32_t ring_off(int s, int c) {
  return static_cast<uint32_t>((c >> 3) * kHalfBytes + s * 128 + (((c & 7) ^ (s & 7)) << 4));
}

// x (4 dims 4*lane .. 4*lane+3 of one head) -> RoPE_p(x / rms(x) * w) in
// place, using the warp's scratch row; cs/sn hold this lane's pair rotation.
__device__ __forceinline__ void norm_rope_row(float (&x)[4], const float* w, float eps,
                                              float* scratch, int lane, int half_rot, float cs,
                                              float sn) {
  float ss = x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float rinv = rsqrtf(ss * (1.0f / kHeadDim) + eps);
  const float4 wv = *reinterpret_cast<const float4*>(w + 4 * lane);
  x[0] *= rinv * wv.x;
  x[1] *= rinv * wv.y;
  x[2] *= rinv * wv.z;
  x[3] *= rinv * wv.w;
  if (half_rot > 0) {
    *reinterpret_cast<float4*>(scratch + 4 * lane) = make_float4(x[0], x[1], x[2], x[3]);
    __syncwarp();
    if (lane < half_rot) {
      const float a = scratch[lane], b = scratch[lane + half_rot];
      scratch[lane] = a * cs - b * sn;             // x_j cos - x_{j+P} sin
      scratch[lane + half_rot] = b * cs + a * sn;  // x_{j+P} cos + x_j sin
    }
    __syncwarp();
    const float4 y = *reinterpret_cast<const float4*>(scratch + 4 * lane);
    x[0] = y.x;
    x[1] = y.y;
    x[2] = y.z;
    x[3] = y.w;
    __syncwarp();  // the scratch row is reused by the next head
  }
}

__device__ __forceinline__ void load4(const uint16_t* p, float (&x)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  x[0] = bf16_lo(u.x);
  x[1] = bf16_hi(u.x);
  x[2] = bf16_lo(u.y);
  x[3] = bf16_hi(u.y);
}

__global__ void __launch_bounds__(kThreads)
    swa_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const DecArgs a) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x / a.Hkv, kvh = blockIdx.x - n * a.Hkv;
  const long long p = a.pos[n];
  if (p < 0) {
    if (tid == 0) atomicCAS(a.err, 0, kDevErrBadPosition);
    return;
  }
  const int s0 = static_cast<int>(p & (kWindow - 1));  // slot of the new token
  const int owner = s0 >> 5;                           // warp whose slots hold it

  if (tid == 0) {
    mbar_init(&sm.kfull, 1);
    mbar_init(&sm.vfull, 1);
    sm.abort = 0;
    fence_barrier_init();
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    mbar_arrive_expect_tx(&sm.kfull, 2 * kHalfBytes);
    tma_load_4d(sm.k[0], &tm_k, &sm.kfull, 0, 0, kvh, n);
    tma_load_4d(sm.k[1], &tm_k, &sm.kfull, 64, 0, kvh, n);
    mbar_arrive_expect_tx(&sm.vfull, 2 * kHalfBytes);
    tma_load_4d(sm.v[0], &tm_v, &sm.vfull, 0, 0, kvh, n);
    tma_load_4d(sm.v[1], &tm_v, &sm.vfull, 64, 0, kvh, n);
  }

  // ---- while the rings load: q' for heads warp, warp+4; k' and v_new on the
  // owner warp; the gate values this thread will apply.
  float cs = 1.0f, sn = 0.0f;
  if (lane < a.half_rot) rope_cos_sin(static_cast<double>(p), a.inv_freq[lane], &cs, &sn);
  for (int h = warp; h < a.G; h += 4) {
    float x[4];
    load4(a.q + ((static_cast<long long>(n) * a.Hq + kvh * a.G + h) * kHeadDim + 4 * lane), x);
    norm_rope_row(x, a.wq, a.eps, sm.scratch[warp], lane, a.half_rot, cs, sn);
    sm.qa[h][2 * lane] = pack_bf16x2(x[0], x[1]);
    sm.qa[h][2 * lane + 1] = pack_bf16x2(x[2], x[3]);
  }
  uint2 kp = make_uint2(0u, 0u), vp = make_uint2(0u, 0u);
  const long long kv_row = (static_cast<long long>(n) * a.Hkv + kvh) * kHeadDim;
  if (warp == owner) {
    float x[4];
    load4(a.k_new + kv_row + 4 * lane, x);
    norm_rope_row(x, a.wk, a.eps, sm.scratch[warp], lane, a.half_rot, cs, sn);
    kp = make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]));
    vp = *reinterpret_cast<const uint2*>(a.v_new + kv_row + 4 * lane);
  }
  uint2 gv[kDecMaxGroup / 4];
#pragma unroll
  for (int i = 0; i < kDecMaxGroup / 4; ++i) {
    const int h = warp + 4 * i;
    if (h < a.G)
      gv[i] = *reinterpret_cast<const uint2*>(
          a.g + (static_cast<long long>(n) * a.Hq + kvh * a.G + h) * kHeadDim + 4 * lane);
  }
  __syncthreads();  // barrier init and q' visible

  // Ring row offset of this sequence's slot s0 and the chunk this lane patches.
  const long long ring_row = ((static_cast<long long>(n) * a.Hkv + kvh) * kWindow + s0) * kHeadDim;
  const uint32_t patch_off = ring_off(s0, lane >> 1) + (lane & 1) * 8;

  mbar_wait(&sm.kfull, 0, &sm.abort, a.err, kSiteKFull);
  __syncthreads();
  if (sm.abort) {
    if (tid == 0) {
      mbar_wait_drain(&sm.kfull, 0);
      mbar_wait_drain(&sm.vfull, 0);
    }
    return;
  }
  if (warp == owner) {
    *reinterpret_cast<uint2*>(&sm.k[0][0] + patch_off) = kp;
    *reinterpret_cast<uint2*>(a.k_cache + ring_row + 4 * lane) = kp;
    __syncwarp();
  }

  // ---- S = q' K^T over this warp's 32 slots (4 n-tiles of 8 slots).
  const int grp = lane >> 2, tig = lane & 3;
  const bool row_ok = grp < a.G;
  float acc[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
  const uint32_t kbase = smem_u32(sm.k[0]);
#pragma unroll
  for (int kp2 = 0; kp2 < 4; ++kp2) {  // pairs of 16-dim k-steps
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
      const int slot = 32 * warp + 8 * j + (lane & 7);
      ldsm_x4(kbase + ring_off(slot, 4 * kp2 + (lane >> 3)), b);
      mma_16816(acc[j], qa0[0], 0u, qa2[0], 0u, b[0], b[1]);
      mma_16816(acc[j], qa0[1], 0u, qa2[1], 0u, b[2], b[3]);
    }
  }

  // ---- softmax pieces over this warp's slots, in log2 units.
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int s = 32 * warp + 8 * j + 2 * tig + e;
      const bool valid = p - ((p - s) & (kWindow - 1)) >= 0;
      acc[j][e] = valid ? acc[j][e] * a.scale_log2 : -INFINITY;
      m = fmaxf(m, acc[j][e]);
    }
  }
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
  const float mu = m == -INFINITY ? 0.0f : m;
  float l = 0.0f;
  uint32_t pa[4];  // P as packed bf16: slots 2tig.. of n-tiles 0..3
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float p0 = ex2_approx(acc[j][0] - mu), p1 = ex2_approx(acc[j][1] - mu);
    l += p0 + p1;
    pa[j] = pack_bf16x2(p0, p1);
  }
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  if (!row_ok) pa[0] = pa[1] = pa[2] = pa[3] = 0u;

  mbar_wait(&sm.vfull, 0, &sm.abort, a.err, kSiteVFull);
  __syncthreads();
  if (sm.abort) {
    if (tid == 0) mbar_wait_drain(&sm.vfull, 0);
    return;
  }
  if (warp == owner) {
    *reinterpret_cast<uint2*>(&sm.v[0][0] + patch_off) = vp;
    *reinterpret_cast<uint2*>(a.v_cache + ring_row + 4 * lane) = vp;
    __syncwarp();
  }

  // ---- partial O = P V over this warp's slots: 16 n-tiles of 8 dims, two
  // 16-slot k-steps each.
  float oacc[16][4];
  const uint32_t vbase = smem_u32(sm.v[0]);
#pragma unroll
  for (int nd = 0; nd < 16; ++nd) {
    oacc[nd][0] = oacc[nd][1] = oacc[nd][2] = oacc[nd][3] = 0.0f;
    uint32_t b[4];
    const int slot = 32 * warp + lane;  // matrix lane/8 = slots 8(lane/8) .. +7
    ldsm_x4_trans(vbase + ring_off(slot, nd), b);
    mma_16816(oacc[nd], pa[0], 0u, pa[1], 0u, b[0], b[1]);
    mma_16816(oacc[nd], pa[2], 0u, pa[3], 0u, b[2], b[3]);
  }

  __syncthreads();  // every warp is done with the K ring: reuse it for partials
  float* part = reinterpret_cast<float*>(sm.k[0]);  // [4][G][kOStride]
  if (row_ok) {
    float* dst = part + (warp * kDecMaxGroup + grp) * kOStride + 2 * tig;
#pragma unroll
    for (int nd = 0; nd < 16; ++nd)
      *reinterpret_cast<float2*>(dst + 8 * nd) = make_float2(oacc[nd][0], oacc[nd][1]);
    if (tig == 0) {
      sm.mw[warp][grp] = m;
      sm.lw[warp][grp] = l;
    }
  }
  __syncthreads();

  // ---- combine: o = (sum_w O_w 2^(m_w - m)) / (sum_w l_w 2^(m_w - m)) * sigmoid(g)
#pragma unroll
  for (int i = 0; i < kDecMaxGroup / 4; ++i) {
    const int h = warp + 4 * i;
    if (h >= a.G) break;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) mx = fmaxf(mx, sm.mw[w][h]);
    float f[4], lsum = 0.0f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      f[w] = sm.mw[w][h] == -INFINITY ? 0.0f : ex2_approx(sm.mw[w][h] - mx);
      lsum += f[w] * sm.lw[w][h];
    }
    float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float4 v4 =
          *reinterpret_cast<const float4*>(part + (w * kDecMaxGroup + h) * kOStride + 4 * lane);
      y[0] += f[w] * v4.x;
      y[1] += f[w] * v4.y;
      y[2] += f[w] * v4.z;
      y[3] += f[w] * v4.w;
    }
    const float inv_l = 1.0f / lsum;
    const float gx[4] = {bf16_lo(gv[i].x), bf16_hi(gv[i].x), bf16_lo(gv[i].y), bf16_hi(gv[i].y)};
    float ov[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) ov[e] = y[e] * inv_l / (1.0f + __expf(-gx[e]));
    *reinterpret_cast<uint2*>(a.o + (static_cast<long long>(n) * a.Hq + kvh * a.G + h) * kHeadDim +
                              4 * lane) =
        make_uint2(pack_bf16x2(ov[0], ov[1]), pack_bf16x2(ov[2], ov[3]));
  }
}

}  // namespace dec

int launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecArgs& a,
                  cudaStream_t stream) {
  const size_t smem = sizeof(dec::Smem) + 1024;
  static int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(dec::swa_decode_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return map_cuda_error(e);
    configured_device = dev;
  }
  const long long grid = static_cast<long long>(a.N) * a.Hkv;
  dec::swa_decode_kernel<<<static_cast<unsigned>(grid), dec::kThreads, smem, stream>>>(tk, tv, a);
  return map_cuda_error(cudaGetLastError());
}

}  // namespace swa
