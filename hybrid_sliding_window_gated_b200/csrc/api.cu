// api.cu -- the C ABI declared in include/swa.h: argument validation, TMA
// tensor-map construction, kernel launch and error mapping.  No entry point
// allocates device memory or synchronises (except swa_get_last_device_error).
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "bwd_internal.h"
#include "decode_internal.h"
#include "global_internal.h"
#include "swa_internal.h"

namespace swa {

// Sticky per-device error word written by bounded waits that ran out.
__device__ int g_device_error = 0;

// Device scratch of swa_bwd_noalloc: a fixed file-scope array, so that entry
// point needs no allocation at all.  Calls that use it must not overlap on
// one device.
constexpr size_t kStaticScratchBytes = 64ull << 20;
static __device__ __align__(256) unsigned char g_bwd_scratch[kStaticScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int g_num_sms[kMaxDevices] = {0};
int* g_err_ptr[kMaxDevices] = {nullptr};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

}  // namespace

int map_cuda_error(cudaError_t e) { return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA; }

int current_device_info(DeviceInfo* info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SWA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_num_sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      return SWA_ERR_CUDA;
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0) return SWA_ERR_UNSUPPORTED;  // built for sm_100a only
    g_num_sms[dev] = n;
  }
  info->device = dev;
  info->num_sms = g_num_sms[dev];
  return SWA_OK;
}

// Address of the static backward scratch on the current device (cached).
static int static_scratch(void** ptr) {
  static void* addr[kMaxDevices] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SWA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (addr[dev] == nullptr && cudaGetSymbolAddress(&addr[dev], g_bwd_scratch) != cudaSuccess)
    return SWA_ERR_CUDA;
  *ptr = addr[dev];
  return SWA_OK;
}

int device_error_word(int** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SWA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_err_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return SWA_ERR_CUDA;
    g_err_ptr[dev] = static_cast<int*>(p);
  }
  *ptr = g_err_ptr[dev];
  return SWA_OK;
}

int encode_tmap_4d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                   uint64_t d3, uint32_t box0, uint32_t box1, uint32_t box2, uint32_t box3,
                   CUtensorMapSwizzle swizzle, bool bytes) {
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return SWA_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  const cuuint64_t dims[4] = {d0, d1, d2, d3};
  const cuuint64_t eb = bytes ? 1 : 2;
  const cuuint64_t strides[3] = {d0 * eb, d0 * d1 * eb, d0 * d1 * d2 * eb};  // bytes, dims 1..3
  const cuuint32_t box[4] = {box0, box1, box2, box3};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(map, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        4, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SWA_OK : SWA_ERR_CUDA;
}

// Shape checks shared by every entry point.  Returns SWA_OK, INVALID_ARG or
// UNSUPPORTED (a valid shape the tensor-core path is not built for).
int check_params(const swa_params_t* p, bool decode) {
  if (p == nullptr) return SWA_ERR_INVALID_ARG;
  if (p->B < 0 || (!decode && p->T < 0) || p->Hq <= 0 || p->Hkv <= 0 || p->head_dim <= 0 ||
      p->window <= 0 || p->rot_dim < 0 || (p->rot_dim & 1) || p->rot_dim > p->head_dim ||
      !(p->eps >= 0.0f) || !(p->scale >= 0.0f) || (p->Hq % p->Hkv) != 0 ||
      (p->rot_dim > 0 && !(p->rope_base > 0.0)))
    return SWA_ERR_INVALID_ARG;
  if (p->head_dim != kHeadDim || p->window != kWindow) return SWA_ERR_UNSUPPORTED;
  if (!(p->rot_dim == 0 || p->rot_dim == 32 || p->rot_dim == 42 || p->rot_dim == 48))
    return SWA_ERR_UNSUPPORTED;
  if (p->B > (1ll << 30) || (!decode && p->T > (1ll << 30)) || p->Hq > 4096)
    return SWA_ERR_UNSUPPORTED;
  // B x T tokens at most 2^40, so that every element count and byte offset
  // below (B T Hq 128 x 2 bytes < 2^60) and every tile count fits in int64.
  if (!decode && p->B * p->T > (1ll << 40)) return SWA_ERR_UNSUPPORTED;
  return SWA_OK;
}

// The global layers have no window: their parameter blocks carry window = 0.
static int check_params_global(const swa_params_t* p, bool decode) {
  if (p == nullptr || p->window != 0) return SWA_ERR_INVALID_ARG;
  swa_params_t c = *p;
  c.window = kWindow;
  return check_params(&c, decode);
}

static float score_scale(const swa_params_t* p) {
  return p->scale > 0.0f ? p->scale : static_cast<float>(1.0 / std::sqrt((double)p->head_dim));
}

static void fill_inv_freq(const swa_params_t* p, double* out) {
  for (int j = 0; j < kMaxPairs; ++j)
    out[j] = (2 * j < p->rot_dim) ? std::pow(p->rope_base, -2.0 * j / p->rot_dim) : 0.0;
}

}  // namespace swa

namespace swa {

// swa_fwd, swa_fwd_fp8 when qkv_scale is set (q, k, v then point at E4M3
// bytes), and swa_fwd_halo when k_halo / v_halo are set.
static int fwd_impl(const swa_params_t* p, const void* q, const void* k, const void* v,
                    const float* qkv_scale, const swa_bf16_t* g, const float* wq, const float* wk,
                    swa_bf16_t* o, float* lse, const swa_bf16_t* k_halo,
                    const swa_bf16_t* v_halo, int64_t pos0, void* stream) {
  int rc = check_params(p, false);
  if (rc != SWA_OK) return rc;
  const bool halo = k_halo != nullptr || v_halo != nullptr;
  if (pos0 < 0 || (halo && (!k_halo || !v_halo || pos0 < kWindow - 1)) ||
      pos0 > (1ll << 40))
    return SWA_ERR_INVALID_ARG;
  if (p->B == 0 || p->T == 0) return SWA_OK;
  if (!q || !k || !v || !g || !wq || !wk || !o) return SWA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(o) ||
      !aligned16(wq) || !aligned16(wk) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (halo && (!aligned16(k_halo) || !aligned16(v_halo))))
    return SWA_ERR_INVALID_ARG;

  FwdArgs a{};
  a.B = static_cast<int>(p->B);
  a.T = static_cast<int>(p->T);
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.G = p->Hq / p->Hkv;
  a.tiles_per_chain = static_cast<int>((p->T + kTile - 1) / kTile);
  a.total_tiles = static_cast<long long>(a.tiles_per_chain) * p->B * p->Hkv;
  a.scale_log2 = score_scale(p) * 1.4426950408889634f;
  a.eps = p->eps;
  a.flags = p->flags;
  a.wq = wq;
  a.wk = wk;
  a.qkv_scale = qkv_scale;
  a.halo = halo ? 1 : 0;
  a.pos0 = pos0;
  a.g = g;
  a.o = o;
  a.lse = lse;
  rc = device_error_word(&a.err);
  if (rc != SWA_OK) return rc;
  fill_inv_freq(p, a.inv_freq);

  // Every bf16 tensor moves in boxes of 128 rows x 64 dims (128-byte rows,
  // 128B swizzle): the MMA operand layout for q, k, v, and the same layout for
  // the gate and output tiles that pass through a Q slot.  FP8 q, k, v move
  // in boxes of 128 rows x 128 one-byte dims, expanded in shared memory.
  CUtensorMap tq, tk, tv, tg, to;
  const uint64_t D = kHeadDim, T = p->T, B = p->B;
  const bool f8 = qkv_scale != nullptr;
  const uint32_t bx = f8 ? 128 : 64;
  if ((rc = encode_tmap_4d(&tq, q, D, p->Hq, T, B, bx, 1, kTile, 1, CU_TENSOR_MAP_SWIZZLE_128B, f8)) ||
      (rc = encode_tmap_4d(&tk, k, D, p->Hkv, T, B, bx, 1, kTile, 1, CU_TENSOR_MAP_SWIZZLE_128B, f8)) ||
      (rc = encode_tmap_4d(&tv, v, D, p->Hkv, T, B, bx, 1, kTile, 1, CU_TENSOR_MAP_SWIZZLE_128B, f8)) ||
      (rc = encode_tmap_4d(&tg, g, D, p->Hq, T, B, 64, 1, kTile, 1, CU_TENSOR_MAP_SWIZZLE_128B)) ||
      (rc = encode_tmap_4d(&to, o, D, p->Hq, T, B, 64, 1, kTile, 1, CU_TENSOR_MAP_SWIZZLE_128B)))
    return rc;
  // The halo's W-1 rows per (sequence, KV head), loaded as key tile -1 from row -1.
  CUtensorMap tkh = tk, tvh = tv;
  if (halo &&
      ((rc = encode_tmap_4d(&tkh, k_halo, D, p->Hkv, kWindow - 1, B, 64, 1, kTile, 1,
                            CU_TENSOR_MAP_SWIZZLE_128B)) ||
       (rc = encode_tmap_4d(&tvh, v_halo, D, p->Hkv, kWindow - 1, B, 64, 1, kTile, 1,
                            CU_TENSOR_MAP_SWIZZLE_128B))))
    return rc;
  return launch_fwd(p, tq, tk, tv, tg, to, tkh, tvh, a, static_cast<cudaStream_t>(stream));
}

}  // namespace swa

using namespace swa;

extern "C" {

const char* swa_version(void) { return "swa-b200 0.1 (sm_100a)"; }

const char* swa_error_string(int code) {
  switch (code) {
    case SWA_OK: return "ok";
    case SWA_ERR_INVALID_ARG: return "invalid argument (null/misaligned pointer or bad shape)";
    case SWA_ERR_UNSUPPORTED: return "unsupported shape for the sm_100a tensor-core path";
    case SWA_ERR_CUDA: return "a CUDA runtime call failed";
    case SWA_ERR_DEVICE_TIMEOUT: return "a kernel wait timed out on the device";
    default: return "unknown error";
  }
}

int swa_get_last_device_error(void* stream, int* site) {
  int* word = nullptr;
  int rc = device_error_word(&word);
  if (rc != SWA_OK) return rc;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SWA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SWA_ERR_CUDA;
  if (site) *site = v;
  if (v == 0) return SWA_OK;
  const int zero = 0;
  if (cudaMemcpy(word, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return SWA_ERR_CUDA;
  // 0x100 + site: a wait ran out; 0x200 and up: an argument the kernel checked
  return v >= kDevErrBadPosition ? SWA_ERR_INVALID_ARG : SWA_ERR_DEVICE_TIMEOUT;
}

int swa_fwd(const swa_params_t* p, const swa_bf16_t* q, const swa_bf16_t* k, const swa_bf16_t* v,
            const swa_bf16_t* g, const float* wq, const float* wk, swa_bf16_t* o, float* lse,
            void* stream) {
  return fwd_impl(p, q, k, v, nullptr, g, wq, wk, o, lse, nullptr, nullptr, 0, stream);
}

int swa_fwd_halo(const swa_params_t* p, const swa_bf16_t* q, const swa_bf16_t* k,
                 const swa_bf16_t* v, const swa_bf16_t* g, const float* wq, const float* wk,
                 const swa_bf16_t* k_halo, const swa_bf16_t* v_halo, int64_t pos0, swa_bf16_t* o,
                 float* lse, void* stream) {
  return fwd_impl(p, q, k, v, nullptr, g, wq, wk, o, lse, k_halo, v_halo, pos0, stream);
}

int swa_fwd_fp8(const swa_params_t* p, const uint8_t* q, const uint8_t* k, const uint8_t* v,
                const float* qkv_scale, const swa_bf16_t* g, const float* wq, const float* wk,
                swa_bf16_t* o, float* lse, void* stream) {
  if (p != nullptr && p->B > 0 && p->T > 0 &&
      (qkv_scale == nullptr || (reinterpret_cast<uintptr_t>(qkv_scale) & 3u)))
    return SWA_ERR_INVALID_ARG;
  return fwd_impl(p, q, k, v, qkv_scale, g, wq, wk, o, lse, nullptr, nullptr, 0, stream);
}

}  // extern "C"

extern "C" {

}  // extern "C"

namespace swa {

// swa_bwd and swa_bwd_edges: the edge rows' fp32 copies are optional
// (n_lo = n_hi = 0 and null buffers for swa_bwd).
static int bwd_impl(const swa_params_t* p, const swa_bf16_t* q, const swa_bf16_t* k,
                    const swa_bf16_t* v, const swa_bf16_t* g, const float* wq, const float* wk,
                    const float* lse, const swa_bf16_t* dO, swa_bf16_t* dq, swa_bf16_t* dk,
                    swa_bf16_t* dv, swa_bf16_t* dg, float* dwq, float* dwk, int64_t n_lo,
                    float* edge_lo, int64_t n_hi, float* edge_hi, const swa_bf16_t* k_halo,
                    const swa_bf16_t* v_halo, int64_t pos0, float* dkv_halo, void* workspace,
                    size_t workspace_bytes, void* stream) {
  int rc = check_params(p, false);
  if (rc != SWA_OK) return rc;
  const bool halo = k_halo != nullptr || v_halo != nullptr || dkv_halo != nullptr;
  if (pos0 < 0 || pos0 > (1ll << 40) ||
      (halo && (!k_halo || !v_halo || !dkv_halo || pos0 < kWindow - 1 || !aligned32(k_halo) ||
                !aligned16(v_halo) || (reinterpret_cast<uintptr_t>(dkv_halo) & 7u))))
    return SWA_ERR_INVALID_ARG;
  if (n_lo < 0 || n_hi < 0 || n_lo > p->T || n_hi > p->T || (n_lo > 0 && edge_lo == nullptr) ||
      (n_hi > 0 && edge_hi == nullptr) || (reinterpret_cast<uintptr_t>(edge_lo) & 7u) ||
      (reinterpret_cast<uintptr_t>(edge_hi) & 7u))
    return SWA_ERR_INVALID_ARG;
  if (p->B == 0 || p->T == 0) return SWA_OK;
  if (!q || !k || !v || !g || !wq || !wk || !lse || !dO || !dq || !dk || !dv || !dg || !dwq ||
      !dwk || !workspace)
    return SWA_ERR_INVALID_ARG;
  // Rows of q, k, g, dO and of the gradients move in 32-byte accesses, one
  // row per thread.
  if (!aligned32(q) || !aligned32(k) || !aligned16(v) || !aligned32(g) || !aligned16(wq) ||
      !aligned16(wk) || !aligned32(dO) || !aligned32(dq) || !aligned32(dk) || !aligned32(dv) ||
      !aligned32(dg) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(dwq) & 3u) || (reinterpret_cast<uintptr_t>(dwk) & 3u) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SWA_ERR_INVALID_ARG;
  const size_t da_bytes = bwd_ws_da_bytes(p->B, p->T, p->Hq);
  const size_t d_bytes = bwd_ws_d_bytes(p->B, p->T, p->Hq);
  const size_t ee_bytes = bwd_ws_ee_bytes(p->B, p->T, p->Hq);
  if (workspace_bytes < bwd_ws_total_bytes(p->B, p->T, p->Hq, p->Hkv)) return SWA_ERR_INVALID_ARG;

  BwdArgs a{};
  a.B = static_cast<int>(p->B);
  a.T = static_cast<int>(p->T);
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.G = p->Hq / p->Hkv;
  a.tiles_per_chain = static_cast<int>((p->T + kTile - 1) / kTile);
  a.total_tiles = static_cast<long long>(a.tiles_per_chain) * p->B * p->Hkv;
  a.scale = score_scale(p);
  a.scale_log2 = a.scale * 1.4426950408889634f;
  a.flags = p->flags;
  a.eps = p->eps;
  a.q = q;
  a.k = k;
  a.g = g;
  a.dO = dO;
  a.lse = lse;
  a.wq = wq;
  a.wk = wk;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.dg = dg;
  a.dwq = dwq;
  a.dwk = dwk;
  a.ws_da = static_cast<uint16_t*>(workspace);
  a.ws_d = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + da_bytes);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.ws_lse = reinterpret_cast<float*>(ws + da_bytes + d_bytes);
  a.ws_ee = reinterpret_cast<int*>(ws + da_bytes + 2 * d_bytes);
  a.ws_ek = reinterpret_cast<int*>(ws + da_bytes + 2 * d_bytes + ee_bytes);
  a.n_lo = static_cast<int>(n_lo);
  a.n_hi = static_cast<int>(n_hi);
  a.halo = halo ? 1 : 0;
  a.pos0 = pos0;
  a.kv_tiles = a.tiles_per_chain + a.halo;
  a.kv_total_tiles = static_cast<long long>(a.kv_tiles) * p->B * p->Hkv;
  a.k_halo = k_halo;
  a.dkv_halo = dkv_halo;
  a.edge_lo = n_lo > 0 ? edge_lo : nullptr;
  a.edge_hi = n_hi > 0 ? edge_hi : nullptr;
  rc = device_error_word(&a.err);
  if (rc != SWA_OK) return rc;
  fill_inv_freq(p, a.inv_freq);
  if (a.total_tiles > (1ll << 30)) return SWA_ERR_UNSUPPORTED;

  CUtensorMap tq, tk, tv;
  const uint64_t D = kHeadDim, T = p->T, B = p->B;
  if ((rc = encode_tmap_4d(&tq, q, D, p->Hq, T, B, 64, 1, kTile, 1, CU_TENSOR_MAP_SWIZZLE_128B)) ||
      (rc = encode_tmap_4d(&tk, k, D, p->Hkv, T, B, 64, 1, kTile, 1, CU_TENSOR_MAP_SWIZZLE_128B)) ||
      (rc = encode_tmap_4d(&tv, v, D, p->Hkv, T, B, 64, 1, kTile, 1, CU_TENSOR_MAP_SWIZZLE_128B)))
    return rc;
  CUtensorMap tkh = tk, tvh = tv;
  if (halo &&
      ((rc = encode_tmap_4d(&tkh, k_halo, D, p->Hkv, kWindow - 1, B, 64, 1, kTile, 1,
                            CU_TENSOR_MAP_SWIZZLE_128B)) ||
       (rc = encode_tmap_4d(&tvh, v_halo, D, p->Hkv, kWindow - 1, B, 64, 1, kTile, 1,
                            CU_TENSOR_MAP_SWIZZLE_128B))))
    return rc;
  return launch_bwd(p, tq, tk, tv, tkh, tvh, a, static_cast<cudaStream_t>(stream));
}

}  // namespace swa

extern "C" {

int swa_bwd(const swa_params_t* p, const swa_bf16_t* q, const swa_bf16_t* k, const swa_bf16_t* v,
            const swa_bf16_t* g, const float* wq, const float* wk, const float* lse,
            const swa_bf16_t* dO, swa_bf16_t* dq, swa_bf16_t* dk, swa_bf16_t* dv, swa_bf16_t* dg,
            float* dwq, float* dwk, void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_impl(p, q, k, v, g, wq, wk, lse, dO, dq, dk, dv, dg, dwq, dwk, 0, nullptr, 0, nullptr,
                  nullptr, nullptr, 0, nullptr, workspace, workspace_bytes, stream);
}

int swa_bwd_edges(const swa_params_t* p, const swa_bf16_t* q, const swa_bf16_t* k,
                  const swa_bf16_t* v, const swa_bf16_t* g, const float* wq, const float* wk,
                  const float* lse, const swa_bf16_t* dO, swa_bf16_t* dq, swa_bf16_t* dk,
                  swa_bf16_t* dv, swa_bf16_t* dg, float* dwq, float* dwk, int64_t n_lo,
                  float* dkv_lo, int64_t n_hi, float* dkv_hi, void* workspace,
                  size_t workspace_bytes, void* stream) {
  return bwd_impl(p, q, k, v, g, wq, wk, lse, dO, dq, dk, dv, dg, dwq, dwk, n_lo, dkv_lo, n_hi,
                  dkv_hi, nullptr, nullptr, 0, nullptr, workspace, workspace_bytes, stream);
}

int swa_bwd_halo(const swa_params_t* p, const swa_bf16_t* q, const swa_bf16_t* k,
                 const swa_bf16_t* v, const swa_bf16_t* g, const float* wq, const float* wk,
                 const float* lse, const swa_bf16_t* dO, swa_bf16_t* dq, swa_bf16_t* dk,
                 swa_bf16_t* dv, swa_bf16_t* dg, float* dwq, float* dwk,
                 const swa_bf16_t* k_halo, const swa_bf16_t* v_halo, int64_t pos0,
                 float* dkv_halo, int64_t n_hi, float* dkv_hi, void* workspace,
                 size_t workspace_bytes, void* stream) {
  return bwd_impl(p, q, k, v, g, wq, wk, lse, dO, dq, dk, dv, dg, dwq, dwk, 0, nullptr, n_hi,
                  dkv_hi, k_halo, v_halo, pos0, dkv_halo, workspace, workspace_bytes, stream);
}

int swa_bwd_noalloc(const swa_params_t* p, const swa_bf16_t* q, const swa_bf16_t* k,
                    const swa_bf16_t* v, const swa_bf16_t* g, const float* wq, const float* wk,
                    const float* lse, const swa_bf16_t* dO, swa_bf16_t* dq, swa_bf16_t* dk,
                    swa_bf16_t* dv, swa_bf16_t* dg, float* dwq, float* dwk, void* stream) {
  int rc = check_params(p, false);
  if (rc != SWA_OK) return rc;
  if (p->B == 0 || p->T == 0) return SWA_OK;
  const size_t need = bwd_ws_total_bytes(p->B, p->T, p->Hq, p->Hkv);
  if (need > kStaticScratchBytes) return SWA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if ((rc = static_scratch(&scratch)) != SWA_OK) return rc;
  return swa_bwd(p, q, k, v, g, wq, wk, lse, dO, dq, dk, dv, dg, dwq, dwk, scratch,
                 kStaticScratchBytes, stream);
}

size_t swa_bwd_workspace_size(const swa_params_t* p) {
  if (check_params(p, false) != SWA_OK) return 0;
  return bwd_ws_total_bytes(p->B, p->T, p->Hq, p->Hkv);
}

int swa_prefill_to_ring(const swa_params_t* p, const swa_bf16_t* k, const swa_bf16_t* v,
                        const float* wk, swa_bf16_t* k_cache, swa_bf16_t* v_cache, void* stream) {
  int rc = check_params(p, false);
  if (rc != SWA_OK) return rc;
  if (p->B == 0 || p->T == 0) return SWA_OK;
  if (!k || !v || !wk || !k_cache || !v_cache) return SWA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(wk) || !aligned16(k_cache) ||
      !aligned16(v_cache))
    return SWA_ERR_INVALID_ARG;
  RingArgs a{};
  a.B = static_cast<int>(p->B);
  a.T = static_cast<int>(p->T);
  a.Hkv = p->Hkv;
  a.half_rot = p->rot_dim / 2;
  a.eps = p->eps;
  a.k = k;
  a.v = v;
  a.wk = wk;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  fill_inv_freq(p, a.inv_freq);
  return launch_prefill_ring(a, static_cast<cudaStream_t>(stream));
}

int swa_prefill_to_ring_varlen(const swa_params_t* p, const int64_t* starts, const int64_t* lens,
                               const int64_t* pos0, const swa_bf16_t* k, const swa_bf16_t* v,
                               const float* wk, swa_bf16_t* k_cache, swa_bf16_t* v_cache,
                               void* stream) {
  int rc = check_params(p, false);
  if (rc != SWA_OK) return rc;
  if (p->B == 0) return SWA_OK;
  if (!starts || !lens || !wk || !k_cache || !v_cache || (p->T > 0 && (!k || !v)))
    return SWA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(starts) & 7u) || (reinterpret_cast<uintptr_t>(lens) & 7u) ||
      (reinterpret_cast<uintptr_t>(pos0) & 7u) || !aligned16(k) || !aligned16(v) ||
      !aligned16(wk) || !aligned16(k_cache) || !aligned16(v_cache))
    return SWA_ERR_INVALID_ARG;
  RingArgs a{};
  a.B = static_cast<int>(p->B);
  a.T = static_cast<int>(p->T);
  a.Hkv = p->Hkv;
  a.half_rot = p->rot_dim / 2;
  a.eps = p->eps;
  a.k = k;
  a.v = v;
  a.wk = wk;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.starts = starts;
  a.lens = lens;
  a.pos0 = pos0;
  if ((rc = device_error_word(&a.err)) != SWA_OK) return rc;
  fill_inv_freq(p, a.inv_freq);
  return launch_prefill_ring(a, static_cast<cudaStream_t>(stream));
}

int swa_decode_step(const swa_params_t* p, const int64_t* pos, const swa_bf16_t* q,
                    const swa_bf16_t* k_new, const swa_bf16_t* v_new, const swa_bf16_t* g,
                    const float* wq, const float* wk, swa_bf16_t* k_cache, swa_bf16_t* v_cache,
                    swa_bf16_t* o, void* stream) {
  int rc = check_params(p, true);
  if (rc != SWA_OK) return rc;
  if (p->Hq / p->Hkv > kDecMaxGroup) return SWA_ERR_UNSUPPORTED;
  if (p->B == 0) return SWA_OK;
  if (!pos || !q || !k_new || !v_new || !g || !wq || !wk || !k_cache || !v_cache || !o)
    return SWA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(pos) & 7u) || !aligned16(q) || !aligned16(k_new) ||
      !aligned16(v_new) || !aligned16(g) || !aligned16(wq) || !aligned16(wk) ||
      !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o))
    return SWA_ERR_INVALID_ARG;

  DecArgs a{};
  a.N = static_cast<int>(p->B);
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.G = p->Hq / p->Hkv;
  a.half_rot = p->rot_dim / 2;
  a.flags = p->flags;
  a.scale_log2 = score_scale(p) * 1.4426950408889634f;
  a.eps = p->eps;
  a.pos = pos;
  a.q = q;
  a.k_new = k_new;
  a.v_new = v_new;
  a.g = g;
  a.wq = wq;
  a.wk = wk;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.o = o;
  rc = device_error_word(&a.err);
  if (rc != SWA_OK) return rc;
  fill_inv_freq(p, a.inv_freq);

  // Each (sequence, KV head) ring [W, D] arrives as two 128-slot x 64-dim
  // boxes with 128B swizzle.
  CUtensorMap tk, tv;
  const uint64_t D = kHeadDim, W = kWindow, N = p->B;
  if ((rc = encode_tmap_4d(&tk, k_cache, D, W, p->Hkv, N, 64, kWindow, 1, 1,
                           CU_TENSOR_MAP_SWIZZLE_128B)) ||
      (rc = encode_tmap_4d(&tv, v_cache, D, W, p->Hkv, N, 64, kWindow, 1, 1,
                           CU_TENSOR_MAP_SWIZZLE_128B)))
    return rc;
  return launch_decode(tk, tv, a, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

extern "C" {

int swa_global_fwd(const swa_params_t* p, const swa_bf16_t* q, const swa_bf16_t* k,
                   const swa_bf16_t* v, const float* wq, const float* wk, swa_bf16_t* o,
                   float* lse, swa_bf16_t* k_cache, swa_bf16_t* v_cache, int64_t cache_cap,
                   void* stream) {
  int rc = check_params_global(p, false);
  if (rc != SWA_OK) return rc;
  if (cache_cap < p->T) return SWA_ERR_INVALID_ARG;
  if (p->B == 0 || p->T == 0) return SWA_OK;
  if (cache_cap > (1ll << 30) || p->B * cache_cap > (1ll << 40)) return SWA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !wq || !wk || !o || !k_cache || !v_cache) return SWA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(wq) ||
      !aligned16(wk) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return SWA_ERR_INVALID_ARG;
  int* err = nullptr;
  if ((rc = device_error_word(&err)) != SWA_OK) return rc;

  GlobalKvArgs kv{};
  kv.B = static_cast<int>(p->B);
  kv.T = static_cast<int>(p->T);
  kv.Hkv = p->Hkv;
  kv.half_rot = p->rot_dim / 2;
  kv.eps = p->eps;
  kv.cap = cache_cap;
  kv.pos = nullptr;
  kv.k = k;
  kv.v = v;
  kv.wk = wk;
  kv.k_cache = k_cache;
  kv.v_cache = v_cache;
  kv.err = err;
  fill_inv_freq(p, kv.inv_freq);

  GlobalFwdArgs a{};
  a.B = static_cast<int>(p->B);
  a.T = static_cast<int>(p->T);
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.G = p->Hq / p->Hkv;
  a.tiles = static_cast<int>((p->T + kTile - 1) / kTile);
  a.pairs = (a.G + 1) / 2;
  a.units = static_cast<long long>(a.tiles) * p->B * p->Hkv * a.pairs;
  if (a.units > (1ll << 30)) return SWA_ERR_UNSUPPORTED;
  a.scale_log2 = score_scale(p) * 1.4426950408889634f;
  a.eps = p->eps;
  a.flags = p->flags;
  a.wq = wq;
  a.wk = wk;
  a.lse = lse;
  a.err = err;
  fill_inv_freq(p, a.inv_freq);

  // q and o in boxes of 128 tokens x 64 dims, as in swa_fwd; the caches
  // [B, Hkv, cap, D] in boxes of 128 slots x 64 dims.
  CUtensorMap tq, tk, tv, to;
  const uint64_t D = kHeadDim, T = p->T, B = p->B, cap = cache_cap;
  if ((rc = encode_tmap_4d(&tq, q, D, p->Hq, T, B, 64, 1, kTile, 1, CU_TENSOR_MAP_SWIZZLE_128B)) ||
      (rc = encode_tmap_4d(&to, o, D, p->Hq, T, B, 64, 1, kTile, 1, CU_TENSOR_MAP_SWIZZLE_128B)) ||
      (rc = encode_tmap_4d(&tk, k_cache, D, cap, p->Hkv, B, 64, kTile, 1, 1,
                           CU_TENSOR_MAP_SWIZZLE_128B)) ||
      (rc = encode_tmap_4d(&tv, v_cache, D, cap, p->Hkv, B, 64, kTile, 1, 1,
                           CU_TENSOR_MAP_SWIZZLE_128B)))
    return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long rows = p->B * (static_cast<long long>(a.tiles) * kTile);
  if ((rc = launch_global_kv(kv, rows, st)) != SWA_OK) return rc;
  return launch_global_fwd(p->rot_dim, tq, tk, tv, to, a, st);
}

size_t swa_global_decode_workspace_size(const swa_params_t* p, int64_t cache_cap) {
  if (check_params_global(p, true) != SWA_OK || cache_cap <= 0) return 0;
  return global_decode_ws_bytes(p->B, p->Hkv, p->Hq / p->Hkv, cache_cap);
}

int swa_global_decode_step(const swa_params_t* p, const int64_t* pos, const swa_bf16_t* q,
                           const swa_bf16_t* k_new, const swa_bf16_t* v_new, const float* wq,
                           const float* wk, swa_bf16_t* k_cache, swa_bf16_t* v_cache,
                           int64_t cache_cap, swa_bf16_t* o, void* workspace,
                           size_t workspace_bytes, void* stream) {
  int rc = check_params_global(p, true);
  if (rc != SWA_OK) return rc;
  if (cache_cap <= 0) return SWA_ERR_INVALID_ARG;
  if (p->Hq / p->Hkv > kGlobalMaxGroup) return SWA_ERR_UNSUPPORTED;
  if (cache_cap > (1ll << 30)) return SWA_ERR_UNSUPPORTED;
  if (p->B == 0) return SWA_OK;
  if (!pos || !q || !k_new || !v_new || !wq || !wk || !k_cache || !v_cache || !o || !workspace)
    return SWA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(pos) & 7u) || !aligned16(q) || !aligned16(k_new) ||
      !aligned16(v_new) || !aligned16(wq) || !aligned16(wk) || !aligned16(k_cache) ||
      !aligned16(v_cache) || !aligned16(o) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SWA_ERR_INVALID_ARG;
  const int G = p->Hq / p->Hkv;
  if (workspace_bytes < global_decode_ws_bytes(p->B, p->Hkv, G, cache_cap))
    return SWA_ERR_INVALID_ARG;
  int* err = nullptr;
  if ((rc = device_error_word(&err)) != SWA_OK) return rc;

  GlobalKvArgs kv{};
  kv.B = static_cast<int>(p->B);
  kv.T = 1;
  kv.Hkv = p->Hkv;
  kv.half_rot = p->rot_dim / 2;
  kv.eps = p->eps;
  kv.cap = cache_cap;
  kv.pos = pos;
  kv.k = k_new;
  kv.v = v_new;
  kv.wk = wk;
  kv.k_cache = k_cache;
  kv.v_cache = v_cache;
  kv.err = err;
  fill_inv_freq(p, kv.inv_freq);

  GlobalDecArgs a{};
  a.N = static_cast<int>(p->B);
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.G = G;
  a.half_rot = p->rot_dim / 2;
  a.chunks = static_cast<int>((cache_cap + kGlobalChunk - 1) / kGlobalChunk);
  a.flags = p->flags;
  a.scale_log2 = score_scale(p) * 1.4426950408889634f;
  a.eps = p->eps;
  a.cap = cache_cap;
  a.pos = pos;
  a.q = q;
  a.wq = wq;
  const size_t po = global_decode_ws_bytes(p->B, p->Hkv, G, cache_cap) -
                    (((static_cast<size_t>(p->B) * p->Hkv * a.chunks * G * 2 * 4) + 255) &
                     ~static_cast<size_t>(255));
  a.part_o = static_cast<float*>(workspace);
  a.part_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + po);
  a.o = o;
  a.err = err;
  fill_inv_freq(p, a.inv_freq);

  CUtensorMap tk, tv;
  const uint64_t D = kHeadDim, cap = cache_cap, N = p->B;
  if ((rc = encode_tmap_4d(&tk, k_cache, D, cap, p->Hkv, N, 64, kTile, 1, 1,
                           CU_TENSOR_MAP_SWIZZLE_128B)) ||
      (rc = encode_tmap_4d(&tv, v_cache, D, cap, p->Hkv, N, 64, kTile, 1, 1,
                           CU_TENSOR_MAP_SWIZZLE_128B)))
    return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = launch_global_kv(kv, p->B, st)) != SWA_OK) return rc;
  return launch_global_decode(tk, tv, a, st);
}

}  // extern "C"
