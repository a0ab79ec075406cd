// global_internal.h -- arguments of the global causal GQA layer's kernels
// (host and device): the full-length KV-cache writer, the causal prefill
// attention and the decode step over the cache.
#pragma once
#include "swa_internal.h"

namespace swa {

// Write k' = RoPE_p(RMSNorm(k)) (rounded to bf16) and v into slot p of the
// full-length caches.  Prefill: rows (b, t) of k, v [B, T, Hkv, D] at p = t.
// Decode: rows n of k, v [N, Hkv, D] at p = pos[n].
struct GlobalKvArgs {
  int B, T, Hkv;
  int half_rot;
  float eps;
  long long cap;          // cache slots per (sequence, KV head)
  const int64_t* pos;     // decode: [N] positions; prefill: null
  const uint16_t* k;
  const uint16_t* v;
  const float* wk;
  uint16_t* k_cache;      // [B, Hkv, cap, D]
  uint16_t* v_cache;
  int* err;
  double inv_freq[kMaxPairs];
};

struct GlobalFwdArgs {
  int B, T, Hq, Hkv, G;
  int tiles;            // query (and key) tiles per sequence
  int pairs;            // head pairs per KV head: ceil(G / 2)
  long long units;      // tiles * B * Hkv * pairs
  float scale_log2;
  float eps;
  int flags;
  const float* wq;
  const float* wk;
  float* lse;           // [B, Hq, T] or null
  int* err;
  double inv_freq[kMaxPairs];
};

// Decode: each work item is (sequence, KV head, chunk of kGlobalChunk keys);
// its partial result goes to the workspace and a second kernel combines them.
constexpr int kGlobalChunk = 2048;
constexpr int kGlobalMaxGroup = 8;

struct GlobalDecArgs {
  int N, Hq, Hkv, G;
  int half_rot;
  int chunks;           // chunk slots per (sequence, KV head) in the workspace
  int flags;
  float scale_log2;
  float eps;
  long long cap;
  const int64_t* pos;
  const uint16_t* q;    // [N, Hq, D]
  const float* wq;
  float* part_o;        // [N, Hkv, chunks, G, D] fp32
  float* part_ml;       // [N, Hkv, chunks, G, 2] fp32: row maximum (log2 units), row sum
  uint16_t* o;          // [N, Hq, D]
  int* err;
  double inv_freq[kMaxPairs];
};

inline size_t global_decode_ws_bytes(long long N, int Hkv, int G, long long cap) {
  const long long chunks = (cap + kGlobalChunk - 1) / kGlobalChunk;
  const size_t po = static_cast<size_t>(N) * Hkv * chunks * G * kHeadDim * 4;
  const size_t pm = static_cast<size_t>(N) * Hkv * chunks * G * 2 * 4;
  return ((po + 255) & ~static_cast<size_t>(255)) + ((pm + 255) & ~static_cast<size_t>(255));
}

int launch_global_kv(const GlobalKvArgs& a, long long rows, cudaStream_t stream);
int launch_global_fwd(int rot_dim, const CUtensorMap& tq, const CUtensorMap& tk,
                      const CUtensorMap& tv, const CUtensorMap& to, const GlobalFwdArgs& a,
                      cudaStream_t stream);
int launch_global_decode(const CUtensorMap& tk, const CUtensorMap& tv, const GlobalDecArgs& a,
                         cudaStream_t stream);

}  // namespace swa
