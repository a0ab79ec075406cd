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
// A unit is one (sequence, KV head): 64 KiB of ring plus 2.5 KiB of new-token
// rows.  The kernel is persistent (one CTA per SM, a contiguous range of units
// each) and streams: a producer warp keeps a 3-stage ring of units in flight
// (the K and V rings by TMA with 128-byte swizzle, q, g, k_new, v_new by bulk
// copies, the position by a plain load), while two consumer groups of four
// warps take alternate units.  In a group, warp w takes slots 32w .. 32w+31:
// S = q' K^T and the partial P V run on the tensor cores with mma.sync (the
// G <= 8 query heads of the group are the M rows, zero-padded to 16), with a
// per-warp maximum; the four partials are combined in shared memory (split-K
// softmax), scaled by 1/l and gated.  The warp owning slot p mod W patches that
// row, in shared memory and in the ring, with k' (rounded to bf16) and v_new
// before reading it.
#include "decode_internal.h"
#include "launch.cuh"
#include "ptx.cuh"
#include "rowops.cuh"
#include "warp_mma.cuh"

namespace swa {
namespace dec {

constexpr int kGroups = 2;                       // consumer groups of 4 warps
constexpr int kThreads = 32 * (1 + 4 * kGroups);  // producer warp + consumers
constexpr int kStages = 3;
constexpr int kHalfBytes = kWindow * 64 * 2;  // 128 slots x 64 dims of bf16 (one TMA box)
constexpr int kQStride = 68;                  // words per packed q' row (bank-conflict padding)
constexpr int kOStride = 136;                 // floats per partial-O row (padding)

struct alignas(1024) Stage {
  uint8_t k[2][kHalfBytes];  // K ring, dims 0..63 and 64..127, 128B-swizzled
  uint8_t v[2][kHalfBytes];  // V ring
  uint16_t q[kDecMaxGroup][kHeadDim];  // the group's query rows
  uint16_t g[kDecMaxGroup][kHeadDim];  // gate logits
  uint16_t kn[kHeadDim], vn[kHeadDim];  // new token's k and v
  float2 rot[kMaxPairs];                // rot(pos w_p): the position's rotation, per pair
  long long pos;
};

struct Group {
  uint32_t qa[kDecMaxGroup][kQStride];  // q' as packed bf16 pairs
  float scratch[4][kHeadDim];           // per-warp norm / RoPE staging
  float mw[4][kDecMaxGroup];            // per-warp row maxima (log2 units)
  float lw[4][kDecMaxGroup];            // per-warp row sums
};

struct alignas(1024) Smem {
  Stage st[kStages];
  Group grp[kGroups];
  uint64_t full[kStages], empty[kStages];
  uint64_t never;  // completed by nothing: SWA_FLAG_FORCE_TIMEOUT waits on it
  int abort;
};
// The partial outputs [4 warps][G heads][kOStride] reuse a stage's K ring once
// the scores are done.
static_assert(4 * kDecMaxGroup * kOStride * 4 <= 2 * kHalfBytes, "partial O does not fit");
static_assert(sizeof(Smem) + 1024 <= 232448, "decode shared memory");

enum Site { kSiteFull = 0x40, kSiteEmpty, kSiteGroup, kSiteForced };

// Byte offset of 16-byte chunk c (0..15) of slot row s in a [half][slot][64]
// 128B-swizzled ring tile.
__device__ __forceinline__ uint32_t ring_off(int s, int c) {
  return static_cast<uint32_t>((c >> 3) * kHalfBytes + s * 128 + (((c & 7) ^ (s & 7)) << 4));
}

// 1-D bulk copy global -> shared, completing on `bar` (16-byte aligned, size a
// multiple of 16).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Barrier over the 128 threads of consumer group `id` that also ANDs `v`
// across them: every decision taken after it is the same on the whole group.
__device__ __forceinline__ bool group_and(bool v, int id) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id)
      : "memory");
  return r != 0;
}

// One (sequence n, KV head kvh) unit, by the 128 threads of consumer group
// `gi` (local warp lw).  The stage holds the unit's rings and new-token rows.
__device__ __forceinline__ void process_unit(Stage& st, Group& gp, const DecArgs& a, int n,
                                             int kvh, int gi, int lw, int lane) {
  const int bar_id = 1 + gi;
  const long long p = st.pos;
  if (p < 0) {  // the same value for the whole group
    if (lw == 0 && lane == 0) atomicCAS(a.err, 0, kDevErrBadPosition);
    return;
  }
  const int s0 = static_cast<int>(p & (kWindow - 1));  // slot of the new token
  const int owner = s0 >> 5;                           // warp whose slots hold it

  // ---- q' for heads lw, lw+4; k' and v_new on the owner warp
  float cs = 1.0f, sn = 0.0f;
  if (lane < a.half_rot) {  // from the producer, once per sequence
    const float2 r = st.rot[lane];
    cs = r.x;
    sn = r.y;
  }
  for (int h = lw; h < a.G; h += 4) {
    float x[4];
    load4(st.q[h] + 4 * lane, x);
    norm_rope_row(x, a.wq, a.eps, gp.scratch[lw], lane, a.half_rot, cs, sn);
    gp.qa[h][2 * lane] = pack_bf16x2(x[0], x[1]);
    gp.qa[h][2 * lane + 1] = pack_bf16x2(x[2], x[3]);
  }
  if (lw == owner) {
    float x[4];
    load4(st.kn + 4 * lane, x);
    norm_rope_row(x, a.wk, a.eps, gp.scratch[lw], lane, a.half_rot, cs, sn);
    const uint2 kp = make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]));
    const uint2 vp = *reinterpret_cast<const uint2*>(st.vn + 4 * lane);
    // Slot s0 of the rings: this lane's 4 dims, in shared memory and in HBM
    // (the ring copy in shared memory has landed, so the global row is free).
    const uint32_t off = ring_off(s0, lane >> 1) + (lane & 1) * 8;
    *reinterpret_cast<uint2*>(&st.k[0][0] + off) = kp;
    *reinterpret_cast<uint2*>(&st.v[0][0] + off) = vp;
    const long long ring_row =
        ((static_cast<long long>(n) * a.Hkv + kvh) * kWindow + s0) * kHeadDim;
    *reinterpret_cast<uint2*>(a.k_cache + ring_row + 4 * lane) = kp;
    *reinterpret_cast<uint2*>(a.v_cache + ring_row + 4 * lane) = vp;
  }
  group_and(true, bar_id);  // q' and the patched rows visible to the group

  // ---- S = q' K^T over this warp's 32 slots (4 n-tiles of 8 slots).
  const int grp = lane >> 2, tig = lane & 3;
  const bool row_ok = grp < a.G;
  float acc[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
  const uint32_t kbase = smem_u32(st.k[0]);
#pragma unroll
  for (int kp2 = 0; kp2 < 4; ++kp2) {  // pairs of 16-dim k-steps
    uint32_t qa0[2], qa2[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int kk = 2 * kp2 + e;
      qa0[e] = row_ok ? gp.qa[grp][8 * kk + tig] : 0u;
      qa2[e] = row_ok ? gp.qa[grp][8 * kk + 4 + tig] : 0u;
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

  // ---- softmax pieces over this warp's slots, in log2 units.
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int s = 32 * lw + 8 * j + 2 * tig + e;
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

  // ---- partial O = P V over this warp's slots: 16 n-tiles of 8 dims, two
  // 16-slot k-steps each.
  float oacc[16][4];
  const uint32_t vbase = smem_u32(st.v[0]);
#pragma unroll
  for (int nd = 0; nd < 16; ++nd) {
    oacc[nd][0] = oacc[nd][1] = oacc[nd][2] = oacc[nd][3] = 0.0f;
    uint32_t b[4];
    const int slot = 32 * lw + lane;  // matrix lane/8 = slots 8(lane/8) .. +7
    ldsm_x4_trans(vbase + ring_off(slot, nd), b);
    mma_16816(oacc[nd], pa[0], 0u, pa[1], 0u, b[0], b[1]);
    mma_16816(oacc[nd], pa[2], 0u, pa[3], 0u, b[2], b[3]);
  }

  group_and(true, bar_id);  // every warp is done with the K ring: reuse it
  float* part = reinterpret_cast<float*>(st.k[0]);  // [4][kDecMaxGroup][kOStride]
  if (row_ok) {
    float* dst = part + (lw * kDecMaxGroup + grp) * kOStride + 2 * tig;
#pragma unroll
    for (int nd = 0; nd < 16; ++nd)
      *reinterpret_cast<float2*>(dst + 8 * nd) = make_float2(oacc[nd][0], oacc[nd][1]);
    if (tig == 0) {
      gp.mw[lw][grp] = m;
      gp.lw[lw][grp] = l;
    }
  }
  group_and(true, bar_id);

  // ---- combine: o = (sum_w O_w 2^(m_w - m)) / (sum_w l_w 2^(m_w - m)) * sigmoid(g)
  for (int h = lw; h < a.G; h += 4) {
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) mx = fmaxf(mx, gp.mw[w][h]);
    float f[4], lsum = 0.0f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      f[w] = gp.mw[w][h] == -INFINITY ? 0.0f : ex2_approx(gp.mw[w][h] - mx);
      lsum += f[w] * gp.lw[w][h];
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
    float gx[4];
    load4(st.g[h] + 4 * lane, gx);
    float ov[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) ov[e] = y[e] * inv_l / (1.0f + __expf(-gx[e]));
    *reinterpret_cast<uint2*>(a.o + (static_cast<long long>(n) * a.Hq + kvh * a.G + h) * kHeadDim +
                              4 * lane) =
        make_uint2(pack_bf16x2(ov[0], ov[1]), pack_bf16x2(ov[2], ov[3]));
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    swa_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const DecArgs a) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long units = static_cast<long long>(a.N) * a.Hkv;
  const long long u0 = units * blockIdx.x / gridDim.x;
  const int n_units = static_cast<int>(units * (blockIdx.x + 1) / gridDim.x - u0);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 2);  // the copies' expect_tx arrive + the position
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.never, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort = &sm.abort;
  // Launched as a programmatic dependent of the previous kernel on the stream:
  // the set-up above overlapped its tail; every read and write of global
  // memory below waits for it to complete.  The next launch may start its own
  // set-up as soon as SMs free up.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Lane 0 issues the copies; the whole warp then writes the position and
    // its rotation (computed once per sequence: a sequence's KV-head units
    // are consecutive) into the stage before the position's arrive.
    if (lane == 0) {
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
    }
    const uint32_t row_bytes = kHeadDim * 2;
    const uint32_t bytes = 4 * kHalfBytes + 2 * a.G * row_bytes + 2 * row_bytes;
    int issued[kStages] = {0};
    bool ok = true;
    long long seq = -1, p = 0;  // the last sequence seen, its position
    float2 rot = make_float2(1.0f, 0.0f);
    for (int i = 0; i < n_units; ++i) {
      const int s = i % kStages;
      bool w = true;
      if (lane == 0 && i >= kStages)
        w = mbar_wait(&sm.empty[s], ((i / kStages) - 1) & 1, abort, a.err, kSiteEmpty);
      if (!__shfl_sync(0xffffffffu, w ? 1 : 0, 0)) {
        ok = false;
        break;
      }
      const long long u = u0 + i;
      const int n = static_cast<int>(u / a.Hkv), kvh = static_cast<int>(u - u / a.Hkv * a.Hkv);
      Stage& st = sm.st[s];
      if (lane == 0) {
        mbar_arrive_expect_tx(&sm.full[s], bytes);
        tma_load_4d(st.k[0], &tm_k, &sm.full[s], 0, 0, kvh, n);
        tma_load_4d(st.k[1], &tm_k, &sm.full[s], 64, 0, kvh, n);
        tma_load_4d(st.v[0], &tm_v, &sm.full[s], 0, 0, kvh, n);
        tma_load_4d(st.v[1], &tm_v, &sm.full[s], 64, 0, kvh, n);
        const long long qrow = (static_cast<long long>(n) * a.Hq + kvh * a.G) * kHeadDim;
        const long long kvrow = (static_cast<long long>(n) * a.Hkv + kvh) * kHeadDim;
        bulk_load(st.q, a.q + qrow, a.G * row_bytes, &sm.full[s]);
        bulk_load(st.g, a.g + qrow, a.G * row_bytes, &sm.full[s]);
        bulk_load(st.kn, a.k_new + kvrow, row_bytes, &sm.full[s]);
        bulk_load(st.vn, a.v_new + kvrow, row_bytes, &sm.full[s]);
        ++issued[s];
      }
      if (n != seq) {  // read while the copies fly
        seq = n;
        p = a.pos[n];
        if (lane < a.half_rot)
          rope_cos_sin(static_cast<double>(p), a.inv_freq[lane], &rot.x, &rot.y);
      }
      if (lane == 0) st.pos = p;
      if (lane < a.half_rot) st.rot[lane] = rot;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.full[s]);  // releases the position and rotation
    }
    if (!ok && lane == 0) {
      // Every copy issued lands before the CTA releases its shared memory.
      for (int s = 0; s < kStages; ++s)
        if (issued[s] > 0) mbar_wait_drain(&sm.full[s], (issued[s] - 1) & 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------- consumer group
    const int gi = (warp - 1) >> 2, lw = (warp - 1) & 3;
    bool live = true;
    if (a.flags & SWA_FLAG_FORCE_TIMEOUT)  // a wait that runs out, for the tests
      live = group_and(mbar_wait(&sm.never, 0, abort, a.err, kSiteForced), 1 + gi);
    for (int i = gi; live && i < n_units; i += kGroups) {
      const int s = i % kStages;
      const bool got = mbar_wait(&sm.full[s], (i / kStages) & 1, abort, a.err, kSiteFull);
      if (!group_and(got, 1 + gi)) break;  // the same decision on the whole group
      const long long u = u0 + i;
      const int n = static_cast<int>(u / a.Hkv), kvh = static_cast<int>(u - u / a.Hkv * a.Hkv);
      process_unit(sm.st[s], sm.grp[gi], a, n, kvh, gi, lw, lane);
      group_and(true, 1 + gi);  // the group is done with the stage
      if (lw == 0 && lane == 0) mbar_arrive(&sm.empty[s]);
    }
  }
  __syncthreads();
}

// Prefill -> ring handoff.  Slot s of ring (b, kv head h) takes the latest
// position p of the sequence's tokens with p = s (mod W): k' = RoPE_p(RMSNorm
// (k_p)) rounded to bf16, exactly as a decode step writes its new token, and
// v_p as it is.  Slots that no position reaches keep their contents.  One warp
// per (sequence, slot): the slot's rotation is computed once for all KV heads,
// whose rows lie next to each other; 4 dims per lane, so each 256-byte row is
// one coalesced access.  Dense form: tokens 0 .. T-1 of row b at positions
// 0 .. T-1.  Varlen form: lens[b] tokens from row starts[b] at positions
// pos0[b] ..; a sequence whose numbers do not fit the rows (or are negative)
// is reported and skipped.
__global__ void __launch_bounds__(128) swa_prefill_ring_kernel(const RingArgs a) {
  __shared__ __align__(16) float scratch[4][kHeadDim];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long gw = static_cast<long long>(blockIdx.x) * 4 + warp;
  const int b = static_cast<int>(gw / kWindow), s = static_cast<int>(gw % kWindow);
  if (b >= a.B) return;  // warp-uniform
  long long first = 0, len = a.T, p0 = 0;  // row of token 0, tokens, position of token 0
  if (a.lens != nullptr) {
    first = a.starts[b];
    len = a.lens[b];
    p0 = a.pos0 != nullptr ? a.pos0[b] : 0;
    if (first < 0 || len < 0 || p0 < 0 || len > a.T || first > a.T - len) {
      if (s == 0 && lane == 0) atomicCAS(a.err, 0, kDevErrBadPosition);
      return;
    }
  } else {
    first = static_cast<long long>(b) * a.T;
  }
  if (len == 0) return;
  // the latest position p in [p0, p0 + len) with p = s (mod W)
  const long long last = p0 + len - 1;
  const long long p = last - (((last - s) % kWindow) + kWindow) % kWindow;
  if (p < p0) return;  // no position of this sequence reaches slot s
  const long long row_tok = first + (p - p0);
  float cs = 1.0f, sn = 0.0f;
  if (lane < a.half_rot) rope_cos_sin(static_cast<double>(p), a.inv_freq[lane], &cs, &sn);
  for (int h = 0; h < a.Hkv; ++h) {
    const long long row = (row_tok * a.Hkv + h) * kHeadDim;
    float x[4];
    load4(a.k + row + 4 * lane, x);
    const uint2 vv = *reinterpret_cast<const uint2*>(a.v + row + 4 * lane);
    norm_rope_row(x, a.wk, a.eps, scratch[warp], lane, a.half_rot, cs, sn);
    const long long ring_row = ((static_cast<long long>(b) * a.Hkv + h) * kWindow + s) * kHeadDim;
    *reinterpret_cast<uint2*>(a.k_cache + ring_row + 4 * lane) =
        make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]));
    *reinterpret_cast<uint2*>(a.v_cache + ring_row + 4 * lane) = vv;
  }
}

}  // namespace dec

int launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecArgs& a,
                  cudaStream_t stream) {
  DeviceInfo di;
  int rc = current_device_info(&di);
  if (rc != SWA_OK) return rc;
  const size_t smem = sizeof(dec::Smem) + 1024;
  static int configured_device = -1;
  if (configured_device != di.device) {
    cudaError_t e = cudaFuncSetAttribute(dec::swa_decode_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return map_cuda_error(e);
    configured_device = di.device;
  }
  const long long units = static_cast<long long>(a.N) * a.Hkv;
  const long long grid = units < di.num_sms ? units : di.num_sms;
  return launch_dependent(dec::swa_decode_kernel, static_cast<unsigned>(grid), dec::kThreads, smem,
                          stream, tk, tv, a);
}

int launch_prefill_ring(const RingArgs& a, cudaStream_t stream) {
  const long long grid = static_cast<long long>(a.B) * (kWindow / 4);  // 4 warps per block
  if (grid > 0x7fffffffLL) return SWA_ERR_UNSUPPORTED;
  return launch_dependent(dec::swa_prefill_ring_kernel, static_cast<unsigned>(grid), 128, 0, stream,
                          a);
}

}  // namespace swa
