// decode_internal.h -- arguments of the decode-step kernel (host and device).
#pragma once
#include "swa_internal.h"

namespace swa {

constexpr int kDecMaxGroup = 8;  // query heads per KV head the decode kernel takes

struct DecArgs {
  int N, Hq, Hkv, G;
  int half_rot;      // rot_dim / 2 rotated pairs
  int flags;         // SWA_FLAG_* debug bits (0 in normal use)
  float scale_log2;  // softmax scale * log2(e)
  float eps;
  const int64_t* pos;
  const uint16_t* q;      // [N, Hq, D]
  const uint16_t* k_new;  // [N, Hkv, D]
  const uint16_t* v_new;  // [N, Hkv, D]
  const uint16_t* g;      // [N, Hq, D]
  const float* wq;
  const float* wk;
  uint16_t* k_cache;  // [N, Hkv, W, D]
  uint16_t* v_cache;
  uint16_t* o;        // [N, Hq, D]
  int* err;
  double inv_freq[kMaxPairs];
};

// Device error codes beyond the wait timeouts: a decode position below 0.
constexpr int kDevErrBadPosition = 0x200;

int launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecArgs& a,
                  cudaStream_t stream);

// Prefill -> ring handoff (see swa_prefill_to_ring and its varlen form).
struct RingArgs {
  int B, T, Hkv;
  int half_rot;
  float eps;
  const uint16_t* k;  // [B, T, Hkv, D], or [T, Hkv, D] rows for the varlen form
  const uint16_t* v;
  const float* wk;
  uint16_t* k_cache;  // [B, Hkv, W, D]
  uint16_t* v_cache;
  // Varlen form (null for the dense one): sequence b's token i is row
  // starts[b] + i of k and v, at position pos0[b] + i (pos0 may be null: 0),
  // for i < lens[b].
  const int64_t* starts;
  const int64_t* lens;
  const int64_t* pos0;
  int* err;
  double inv_freq[kMaxPairs];
};

int launch_prefill_ring(const RingArgs& a, cudaStream_t stream);

}  // namespace swa
