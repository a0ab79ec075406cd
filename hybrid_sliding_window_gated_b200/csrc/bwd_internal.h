// bwd_internal.h -- arguments of the backward kernels (host and device).
#pragma once
#include "swa_internal.h"

namespace swa {

struct BwdArgs {
  int B, T, Hq, Hkv, G;
  int tiles_per_chain;
  long long total_tiles;
  float scale;       // softmax scale
  float scale_log2;  // scale * log2(e)
  float eps;
  int flags;  // SWA_FLAG_* debug bits (0 in normal use)
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* g;
  const uint16_t* dO;
  const float* lse;  // [B, Hq, T] natural-log normaliser from the forward
  const float* wq;
  const float* wk;
  uint16_t* dq;
  uint16_t* dk;
  uint16_t* dv;
  uint16_t* dg;
  float* dwq;
  float* dwk;
  // Workspace.  Row i of dA is staged as dA_i 2^e_i, with e_i chosen from
  // max|dO_i| so the row's largest value lies in [1, 2) (fp16 keeps its full
  // precision there whatever the scale of the upstream gradient).
  uint16_t* ws_da;  // dA_i 2^e_i, fp16 tiles [B, Hq, tiles] of 128 x 128 (operand layout)
  float* ws_d;      // D_i 2^e_i = (dA_i 2^e_i) . A_i, [B, Hq, T] fp32
  float* ws_lse;    // log2 of the renormalised softmax normaliser, plus e_i, [B, Hq, T] fp32
  int* ws_ee;       // min of e_i over each query tile's rows, [B, Hq, tiles]
  int* ws_ek;       // dS scale exponent of each query tile (from max|v|), [B, Hkv, tiles]
  // Optional fp32 copies of dk and dv for the first n_lo and the last n_hi
  // key rows of every sequence, [B, n, Hkv, 2, D] (dk, then dv); 0 and null
  // when unused.
  int n_lo, n_hi;
  float* edge_lo;
  float* edge_hi;
  // A chunk with the previous chunk's halo: its W-1 keys precede row 0 (key
  // tile -1 of each chain, the key-major pass's extra tile), and this chunk's
  // share of their dk, dv goes to dkv_halo [B, W-1, Hkv, 2, D] fp32.
  int halo;
  long long pos0;            // position of row 0
  int kv_tiles;              // key tiles per chain in the key-major pass: tiles + halo
  long long kv_total_tiles;
  const uint16_t* k_halo;    // [B, W-1, Hkv, D]
  float* dkv_halo;
  int* err;
  double inv_freq[kMaxPairs];
};

// Device error code: a norm weight too large for the fp16 operands (|w| > 4096).
constexpr int kDevErrBadWeights = 0x201;
// Device error code: a value the fp16 staging cannot carry: |v| > 65504, or
// a finite |dO| >= 2^63 (beyond the per-row scaling's range).
constexpr int kDevErrRange = 0x202;

// Workspace layout, each part 256-byte aligned: dA tiles, D, the renormalised
// lse (D and lse share the size bwd_ws_d_bytes), then the two exponent records.
inline size_t bwd_round256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }
inline size_t bwd_ws_da_bytes(long long B, long long T, int Hq) {  // whole 128 x 128 tiles
  return bwd_round256(static_cast<size_t>(B) * ((T + kTile - 1) / kTile) * Hq * kTile * kHeadDim * 2);
}
inline size_t bwd_ws_d_bytes(long long B, long long T, int Hq) {
  return bwd_round256(static_cast<size_t>(B) * T * Hq * 4);
}
inline size_t bwd_ws_ee_bytes(long long B, long long T, int Hq) {
  return bwd_round256(static_cast<size_t>(B) * ((T + kTile - 1) / kTile) * Hq * 4);
}
inline size_t bwd_ws_ek_bytes(long long B, long long T, int Hkv) {
  return bwd_round256(static_cast<size_t>(B) * ((T + kTile - 1) / kTile) * Hkv * 4);
}
inline size_t bwd_ws_total_bytes(long long B, long long T, int Hq, int Hkv) {
  return bwd_ws_da_bytes(B, T, Hq) + 2 * bwd_ws_d_bytes(B, T, Hq) + bwd_ws_ee_bytes(B, T, Hq) +
         bwd_ws_ek_bytes(B, T, Hkv);
}

// tkh, tvh: the halo K and V (any valid map when a.halo is 0).
int launch_bwd(const swa_params_t* p, const CUtensorMap& tq, const CUtensorMap& tk,
               const CUtensorMap& tv, const CUtensorMap& tkh, const CUtensorMap& tvh,
               const BwdArgs& a, cudaStream_t stream);

}  // namespace swa
