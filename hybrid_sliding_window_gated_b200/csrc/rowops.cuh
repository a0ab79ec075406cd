// rowops.cuh -- one warp per 128-dim row, 4 dims per lane: the decode-side
// RMSNorm + partial RoPE of a single token's q or k row, and bf16 loads.
#pragma once
#include "ptx.cuh"
#include "swa_internal.h"

namespace swa {

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

}  // namespace swa
