// swa_internal.h -- host-side declarations shared by the library's .cu files.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/swa.h"

namespace swa {

constexpr int kHeadDim = 128;  // the tensor-core path is built for head_dim 128
constexpr int kWindow = 128;   // and a 128-token window (one key tile per query tile)
constexpr int kTile = 128;     // query / key tile rows
constexpr int kMaxPairs = 24;  // rot_dim <= 48

struct FwdArgs {
  int B, T, Hq, Hkv, G;
  int tiles_per_chain;
  long long total_tiles;
  float scale_log2;  // softmax scale * log2(e)
  float eps;
  int flags;         // SWA_FLAG_* debug bits (0 in normal use)
  int halo;          // 1: the previous chunk's last W-1 tokens precede row 0 (key tile -1)
  long long pos0;    // position of row 0
  const float* wq;
  const float* wk;
  const float* qkv_scale;  // FP8 (E4M3) q, k, v: their dequantisation factors; null for bf16
  const uint16_t* g;
  uint16_t* o;
  float* lse;
  int* err;  // sticky device error word
  double inv_freq[kMaxPairs];  // base^(-2j/rot_dim)
};

struct DeviceInfo {
  int device;
  int num_sms;
};

// Current device and its SM count (cached per device).
int current_device_info(DeviceInfo* info);

// cuTensorMapEncodeTiled through the runtime's driver entry point: bf16
// elements, or single bytes when `bytes` is set.
int encode_tmap_4d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                   uint64_t d3, uint32_t box0, uint32_t box1, uint32_t box2, uint32_t box3,
                   CUtensorMapSwizzle swizzle, bool bytes = false);

// tkh, tvh: tensor maps of the halo K and V [B, W-1, Hkv, D] (used only when
// a.halo is set; any valid map otherwise).
int launch_fwd(const swa_params_t* p, const CUtensorMap& tq, const CUtensorMap& tk,
               const CUtensorMap& tv, const CUtensorMap& tg, const CUtensorMap& to,
               const CUtensorMap& tkh, const CUtensorMap& tvh, const FwdArgs& a,
               cudaStream_t stream);

int map_cuda_error(cudaError_t e);

// Shape checks shared by every entry point (SWA_OK, INVALID_ARG or UNSUPPORTED).
int check_params(const swa_params_t* p, bool decode);

// Address of the device error word on the current device.
int device_error_word(int** ptr);

}  // namespace swa
