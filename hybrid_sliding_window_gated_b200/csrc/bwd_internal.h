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
  uint16_t* ws_da;  // workspace: dA = dO * sigmoid(g), [B, T, Hq, D] fp16
  float* ws_d;      // workspace: D_i = dA_i . A_i, [B, Hq, T] fp32
  float* ws_lse;    // workspace: lse renormalised to the backward's scores, [B, Hq, T] fp32
  int* err;
  double inv_freq[kMaxPairs];
};

// Device error code: a norm weight too large for the fp16 operands (|w| > 4096).
constexpr int kDevErrBadWeights = 0x201;
// Device error code: a value of v or dO beyond the fp16 range (|x| > 65504).
constexpr int kDevErrRange = 0x202;

// Workspace layout: dA rows, then D, then the renormalised lse, each 256-byte
// aligned (D and lse share the size bwd_ws_d_bytes).
inline size_t bwd_ws_da_bytes(long long B, long long T, int Hq) {
  return ((static_cast<size_t>(B) * T * Hq * kHeadDim * 2) + 255) & ~static_cast<size_t>(255);
}
inline size_t bwd_ws_d_bytes(long long B, long long T, int Hq) {
  return ((static_cast<size_t>(B) * T * Hq * 4) + 255) & ~static_cast<size_t>(255);
}

int launch_bwd(const swa_params_t* p, const CUtensorMap& tq, const CUtensorMap& tk,
               const CUtensorMap& tv, const CUtensorMap& tda, const BwdArgs& a,
               cudaStream_t stream);

}  // namespace swa
