/*
 * swa.h -- C ABI of the gated sliding-window attention core for NVIDIA B200
 * (sm_100a).
 *
 * The operation is the GatedSWA module of ZGCM-1 without its projections:
 *
 *   O = A_SWA(q', k', v) (*) sigma(g),   q' = RoPE(RMSNorm(q)),  k' = RoPE(RMSNorm(k))
 *
 * Sources: "7.39B 오픈 모델로 256K 문맥의 수학 추론과 에이전트 검색을 겨냥한 ZGCM-1"
 * (onedev.kr), section "어떻게 동작하나": GatedSWA(h) = o_proj(A_SWA(q,k,v) (*)
 * sigma(g_proj(h))), 32 query heads and 8 KV heads of dim 128, a 128-token
 * window, RMSNorm as the QK normalisation and partial RoPE with rotary
 * fraction 0.33; and "ZGCM-1: A Fully Open and Extremely Efficient Foundation
 * Model for Math and Agentic Search" (jaehun.me), section "How Gated SWA
 * Behaves": norm and partial RoPE on q and k, GQA attention inside the window
 * (a token sees the window including itself), element-wise sigmoid gate.
 * Section "Why the KV Cache Shrinks by 6.4x" of the same page fixes that a
 * window layer keeps only its last W tokens, which is the decode ring below.
 *
 * Readings taken where the pages are silent:
 *   - RMSNorm per head over head_dim: y = x / sqrt(mean(x^2) + eps) * w, one
 *     fp32 weight vector [head_dim] for q and one for k, shared by all heads;
 *   - RoPE after the norm on the first rot_dim dims, rotate-half pairs
 *     (j, j + rot_dim/2) turned by pos * rope_base^(-2j/rot_dim); the other
 *     dims pass through; prefill positions are 0 .. T-1;
 *   - scores scaled by `scale` (0 selects 1/sqrt(head_dim)); query i attends
 *     keys max(0, i-window+1) .. i; q head h reads KV head h / (Hq/Hkv);
 *   - sigma(g) = 1/(1+exp(-g)) per output element; g are gate logits.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, contiguous
 *     row-major, 16-byte aligned.  Prefill tensors are [B, T, H, head_dim]
 *     (H = Hq for q, g, o, dq, dg; H = Hkv for k, v, dk, dv).  bf16 data is
 *     passed as swa_bf16_t (raw bits).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  The library never synchronises and allocates no
 *     device memory; it keeps only small per-device caches (SM count, kernel
 *     attributes).
 *   - The tensor-core path needs head_dim == 128, window == 128, Hq a
 *     multiple of Hkv and rot_dim even in {0, 32, 42, 48}.  Other shapes return
 *     SWA_ERR_UNSUPPORTED; nothing silently falls back to a slow path.  Size
 *     limits (also SWA_ERR_UNSUPPORTED beyond them): B and T at most 2^30 each,
 *     B x T at most 2^40 tokens, Hq at most 4096.
 *   - Errors: SWA_OK on success; SWA_ERR_INVALID_ARG (null or misaligned
 *     pointer, negative size, Hq % Hkv != 0, ...); SWA_ERR_UNSUPPORTED;
 *     SWA_ERR_CUDA (a CUDA runtime call failed, e.g. the launch); the kernels
 *     bound every internal wait and, when one runs out, record the site in a
 *     sticky device word that swa_get_last_device_error() returns as
 *     SWA_ERR_DEVICE_TIMEOUT.  Arguments that live in device memory (decode
 *     positions) are checked by the kernel, which records a bad one in the same
 *     word, returned as SWA_ERR_INVALID_ARG.
 */
#ifndef SWA_H_
#define SWA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t swa_bf16_t; /* bf16 bit pattern */

enum {
  SWA_OK = 0,
  SWA_ERR_INVALID_ARG = 1,
  SWA_ERR_UNSUPPORTED = 2,
  SWA_ERR_CUDA = 3,
  SWA_ERR_DEVICE_TIMEOUT = 4
};

/* Debug bits for swa_params_t.flags (0 in normal use).  FORCE_TIMEOUT makes
 * the kernels of swa_fwd, swa_bwd and swa_decode_step wait on a barrier that
 * nothing completes, so tests can check that the bounded wait ends the kernel
 * (its copies drained, TMEM freed) and reports SWA_ERR_DEVICE_TIMEOUT. */
enum { SWA_FLAG_FORCE_TIMEOUT = 1 };

typedef struct swa_params {
  int64_t B;        /* batch rows (prefill) or number of sequences (decode) */
  int64_t T;        /* tokens per row (prefill); ignored by decode */
  int32_t Hq;       /* query heads (32 in ZGCM-1) */
  int32_t Hkv;      /* KV heads (8) */
  int32_t head_dim; /* 128 */
  int32_t window;   /* W: keys i-W+1 .. i (128) */
  int32_t rot_dim;  /* rotated dims (42 = 0.33 * 128, even) */
  int32_t flags;    /* SWA_FLAG_* debug bits, 0 normally */
  double rope_base; /* 1e4; 1e7 at the 256K stage */
  float eps;        /* RMSNorm epsilon (1e-6) */
  float scale;      /* score scale; 0 selects 1/sqrt(head_dim) */
} swa_params_t;

/*
 * Forward.  q, g: [B,T,Hq,D]; k, v: [B,T,Hkv,D] (bf16); wq, wk: [D] fp32.
 * Writes o [B,T,Hq,D] bf16 and, when lse != NULL, lse [B,Hq,T] fp32, the
 * natural-log softmax normaliser of each row's scaled scores (what swa_bwd
 * reads).  o and lse must not overlap the inputs.
 */
int swa_fwd(const swa_params_t* p, const swa_bf16_t* q, const swa_bf16_t* k,
            const swa_bf16_t* v, const swa_bf16_t* g, const float* wq, const float* wk,
            swa_bf16_t* o, float* lse, void* stream);

/*
 * swa_fwd for one chunk of longer sequences: row 0 of q, k, v, g is at
 * position pos0, and the W - 1 = 127 tokens before it -- the previous
 * chunk's last ones, positions pos0 - 127 .. pos0 - 1 -- are given as k_halo,
 * v_halo [B, 127, Hkv, D] bf16 (raw k and v, as the previous chunk received
 * them), so every query row sees its whole window.  pos0 >= 127 (with a
 * halo, every halo row is a real token); k_halo and v_halo both set or both
 * NULL (then pos0 only shifts the positions: a chunk without history).
 * Other arguments and results as swa_fwd: o, lse [B, Hq, T] for the chunk's
 * own rows.  For sequence sharding (a rank holds a contiguous slice of every
 * sequence) and continued prefills: the halo crosses the chunk boundary
 * because a token sees the W - 1 before it (jaehun.me review, "How Gated SWA
 * Behaves").
 */
int swa_fwd_halo(const swa_params_t* p, const swa_bf16_t* q, const swa_bf16_t* k,
                 const swa_bf16_t* v, const swa_bf16_t* g, const float* wq, const float* wk,
                 const swa_bf16_t* k_halo, const swa_bf16_t* v_halo, int64_t pos0, swa_bf16_t* o,
                 float* lse, void* stream);

/*
 * swa_fwd with q, k and v in FP8 E4M3 (one byte per element, the OCP E4M3
 * encoding: bias 7, no infinities), each with one fp32 dequantisation factor:
 * the values are q = q8 * qkv_scale[0], k = k8 * qkv_scale[1], v = v8 *
 * qkv_scale[2].  qkv_scale is a [3] fp32 DEVICE array (4-byte aligned), so a
 * caller that keeps delayed-scaling factors on the device passes them as
 * they are.  q, k, v: [B,T,H,D] bytes, 16-byte aligned; g, wq, wk, o, lse as
 * in swa_fwd.  Every E4M3 value is exact in bf16, and the factors fold into
 * per-row factors, so the result has the accuracy of swa_fwd on the
 * dequantised inputs; q, k, v move at half the bytes.  Source: the training
 * recipe's FP8 forward (onedev.kr summary, "무엇과 다른가": Transformer Engine
 * hybrid FP8, E4M3 forward); one factor per tensor is what delayed scaling
 * keeps.
 */
int swa_fwd_fp8(const swa_params_t* p, const uint8_t* q, const uint8_t* k, const uint8_t* v,
                const float* qkv_scale, const swa_bf16_t* g, const float* wq, const float* wk,
                swa_bf16_t* o, float* lse, void* stream);

/*
 * Backward of swa_fwd given the upstream gradient dO [B,T,Hq,D] and the lse
 * that swa_fwd wrote.  Writes dq, dg [B,T,Hq,D] and dk, dv [B,T,Hkv,D]
 * (bf16) and ADDS the weight gradients into dwq, dwk [D] (fp32; the caller
 * zeroes them).  `workspace` is caller-owned device scratch of at least
 * swa_bwd_workspace_size(p) bytes, 256-byte aligned; its contents on entry
 * do not matter.  q, k, g, dO, dq, dk, dv and dg must be 32-byte aligned
 * (their rows move in 32-byte accesses); v 16-byte, as everywhere else; a
 * misaligned pointer returns SWA_ERR_INVALID_ARG before any launch.  The
 * chain rule covers the gate, the softmax, RoPE and the
 * RMSNorm (the weights included).  The contractions run on fp16 operands
 * (three more mantissa bits than bf16).  dA = dO sigma(g) and dS are staged
 * with power-of-two scales -- per query row from max|dO| of the row, per
 * 128-query tile from max|v| of its keys -- so a row whose largest |dO| lies
 * in [2^-62, 2^63) keeps fp16's relative precision, however small the
 * gradient; a finite |dO| >= 2^63, |v| > 65504 or |wq|, |wk| > 4096 is reported by
 * swa_get_last_device_error() as SWA_ERR_INVALID_ARG.  v is staged in fp16
 * as is: exact for |v| >= 2^-14, absolute error at most 2^-25 below that.
 */
int swa_bwd(const swa_params_t* p, const swa_bf16_t* q, const swa_bf16_t* k,
            const swa_bf16_t* v, const swa_bf16_t* g, const float* wq, const float* wk,
            const float* lse, const swa_bf16_t* dO, swa_bf16_t* dq, swa_bf16_t* dk,
            swa_bf16_t* dv, swa_bf16_t* dg, float* dwq, float* dwk, void* workspace,
            size_t workspace_bytes, void* stream);

/*
 * swa_bwd that also writes, in fp32, dk and dv of the first n_lo and the last
 * n_hi tokens of every sequence (0 <= n_lo, n_hi <= T): dkv_lo [B, n_lo, Hkv,
 * 2, D] and dkv_hi [B, n_hi, Hkv, 2, D] (index 0 of the fourth axis is dk, 1
 * is dv), 8-byte aligned, caller-owned device memory; a buffer may be NULL when
 * its count is 0.  The bf16 dk and dv are written as by swa_bwd.  For callers
 * that add the partial gradients of the same keys from two calls -- sequence
 * sharding, where a chunk's first W - 1 keys are the previous chunk's last
 * W - 1 -- and want the sum rounded to bf16 once.  The partial sums are
 * linear in the incoming gradient (the RMSNorm Jacobian depends on k only),
 * so they add exactly.  No counterpart in the pages beyond the window itself
 * (a token sees the W - 1 before it: jaehun.me review, "How Gated SWA
 * Behaves"), whose halo crosses a chunk boundary.
 */
int swa_bwd_edges(const swa_params_t* p, const swa_bf16_t* q, const swa_bf16_t* k,
                  const swa_bf16_t* v, const swa_bf16_t* g, const float* wq, const float* wk,
                  const float* lse, const swa_bf16_t* dO, swa_bf16_t* dq, swa_bf16_t* dk,
                  swa_bf16_t* dv, swa_bf16_t* dg, float* dwq, float* dwk, int64_t n_lo,
                  float* dkv_lo, int64_t n_hi, float* dkv_hi, void* workspace,
                  size_t workspace_bytes, void* stream);

/*
 * The backward of swa_fwd_halo: the chunk's own rows as in swa_bwd, with the
 * halo k_halo, v_halo [B, 127, Hkv, D] and pos0 as given to the forward
 * (both halos set, pos0 >= 127; k_halo 32-byte aligned, its rows move in
 * 32-byte accesses).  Writes, in fp32, this chunk's share of the gradient
 * of the halo keys to dkv_halo [B, 127, Hkv, 2, D] (dk, then dv; 8-byte
 * aligned): the previous chunk adds it to its own share of its last 127 rows
 * (the n_hi rows it asked for here in dkv_hi, as swa_bwd_edges does) and
 * rounds the sum once.  dwq and dwk take this chunk's share, the halo keys'
 * included (the weight gradients are linear in the incoming dk' and dq', so
 * the chunks' shares sum).  Other arguments and results as swa_bwd_edges.
 */
int swa_bwd_halo(const swa_params_t* p, const swa_bf16_t* q, const swa_bf16_t* k,
                 const swa_bf16_t* v, const swa_bf16_t* g, const float* wq, const float* wk,
                 const float* lse, const swa_bf16_t* dO, swa_bf16_t* dq, swa_bf16_t* dk,
                 swa_bf16_t* dv, swa_bf16_t* dg, float* dwq, float* dwk,
                 const swa_bf16_t* k_halo, const swa_bf16_t* v_halo, int64_t pos0,
                 float* dkv_halo, int64_t n_hi, float* dkv_hi, void* workspace,
                 size_t workspace_bytes, void* stream);

/* Bytes of scratch swa_bwd needs for these parameters (0 if unsupported). */
size_t swa_bwd_workspace_size(const swa_params_t* p);

/*
 * swa_bwd without a caller workspace (no paper counterpart: a library
 * convenience).  The scratch is a fixed 64 MiB array inside the library's
 * device image, so the call allocates nothing; problems whose
 * swa_bwd_workspace_size exceeds 64 MiB return SWA_ERR_UNSUPPORTED.  Calls
 * share that array: two of them must not run concurrently on one device
 * (calls on one stream are fine).  Arguments and results are those of swa_bwd.
 */
int swa_bwd_noalloc(const swa_params_t* p, const swa_bf16_t* q, const swa_bf16_t* k,
                    const swa_bf16_t* v, const swa_bf16_t* g, const float* wq, const float* wk,
                    const float* lse, const swa_bf16_t* dO, swa_bf16_t* dq, swa_bf16_t* dk,
                    swa_bf16_t* dv, swa_bf16_t* dg, float* dwq, float* dwk, void* stream);

/*
 * One decode step for p->B sequences against their window caches.
 * pos: [B] int64 device array (8-byte aligned), the position of each
 * sequence's new token, >= 0 (a negative one leaves that sequence's o and ring
 * untouched and is reported by swa_get_last_device_error as
 * SWA_ERR_INVALID_ARG).  q, g: [B,Hq,D]; k_new, v_new: [B,Hkv,D] (bf16).
 * k_cache, v_cache: [B,Hkv,W,D] bf16 rings, updated in place: slot
 * pos mod W receives RoPE(RMSNorm(k_new)) (rounded to bf16) and v_new
 * (bit-exact copy); slot s holds the key of position pos - ((pos - s) mod W),
 * ignored when that position is negative.  Writes o [B,Hq,D] bf16.
 * Distinct sequences must not share ring memory.  Hq / Hkv <= 8 (else
 * SWA_ERR_UNSUPPORTED).  Source: the window layers keep only their last W
 * tokens (jaehun.me review, "Why the KV Cache Shrinks by 6.4x"); decoding is
 * memory-bandwidth bound (onedev.kr summary, "어떻게 동작하나").
 */
int swa_decode_step(const swa_params_t* p, const int64_t* pos, const swa_bf16_t* q,
                    const swa_bf16_t* k_new, const swa_bf16_t* v_new, const swa_bf16_t* g,
                    const float* wq, const float* wk, swa_bf16_t* k_cache,
                    swa_bf16_t* v_cache, swa_bf16_t* o, void* stream);

/*
 * Prefill -> ring handoff: after a prefill of p->T tokens, fill the decode
 * rings so that swa_decode_step can continue at position T.  k, v:
 * [B,T,Hkv,D] bf16 (the prefill's raw k and v); wk [D] fp32.  k_cache,
 * v_cache: [B,Hkv,W,D] bf16 rings, updated in place: slot s receives the
 * latest position p <= T-1 with p = s (mod W) -- k' = RoPE(RMSNorm(k_p)),
 * rounded to bf16 exactly as swa_decode_step writes its new token, and v_p
 * (bit-exact copy).  Slots that no position reaches (s > T-1, when T < W)
 * keep their contents, which the decode ignores.  Pointers 16-byte aligned;
 * returns SWA_ERR_INVALID_ARG / UNSUPPORTED like swa_fwd.  No counterpart in
 * the pages beyond the serving view (the window layers' KV cache holds the
 * last W tokens: jaehun.me review, "Why the KV Cache Shrinks by 6.4x").
 */
int swa_prefill_to_ring(const swa_params_t* p, const swa_bf16_t* k, const swa_bf16_t* v,
                        const float* wk, swa_bf16_t* k_cache, swa_bf16_t* v_cache, void* stream);

/*
 * The prefill -> ring handoff for ragged batches and continued prefills.  p->B
 * sequences; sequence b's lens[b] tokens are rows starts[b] .. starts[b] +
 * lens[b] - 1 of k, v [p->T, Hkv, D] (a packed batch: starts = cumulative
 * lengths; or a padded [B, Tmax] batch: starts[b] = b Tmax, p->T = B Tmax),
 * at positions pos0[b] .. pos0[b] + lens[b] - 1 (pos0 NULL: 0).  Slot s of
 * ring b receives the latest of those positions p with p = s (mod W), as
 * swa_prefill_to_ring writes it; other slots keep their contents (so a
 * continued prefill, pos0 > 0, keeps the earlier chunk's slots it does not
 * reach).  starts, lens, pos0: [B] int64 DEVICE arrays, 8-byte aligned; a
 * sequence with a negative value or rows past p->T is skipped and reported
 * by swa_get_last_device_error as SWA_ERR_INVALID_ARG.  A padded batch's
 * prefill runs through swa_fwd unchanged: causal attention makes each valid
 * row independent of the padding after it.  Source: the serving view of the
 * window layers, which keep only their last W tokens (jaehun.me review,
 * "Why the KV Cache Shrinks by 6.4x").
 */
int swa_prefill_to_ring_varlen(const swa_params_t* p, const int64_t* starts, const int64_t* lens,
                               const int64_t* pos0, const swa_bf16_t* k, const swa_bf16_t* v,
                               const float* wk, swa_bf16_t* k_cache, swa_bf16_t* v_cache,
                               void* stream);

/*
 * Global causal GQA layers (no counterpart of the window: 5 of ZGCM-1's 32
 * layers, at 6, 12, 18, 24 and 30, attend over the whole causal context with
 * the same QK-RMSNorm, partial RoPE and GQA, and without the output gate --
 * onedev.kr summary, "어떻게 동작하나"; jaehun.me review, "How Gated SWA
 * Behaves"; they keep every token's K and V -- "Why the KV Cache Shrinks by
 * 6.4x").  For these calls p->window must be 0 (no window).
 *
 * Prefill: o_i = softmax_j(scale q'_i . k'_j, j <= i) V for positions
 * 0 .. T-1.  q [B,T,Hq,D], k, v [B,T,Hkv,D] bf16; wq, wk [D] fp32.  Writes o
 * [B,T,Hq,D] bf16, lse [B,Hq,T] fp32 when lse != NULL, and the layer's
 * full-length caches k_cache, v_cache [B, Hkv, cache_cap, D] bf16 (cache_cap
 * >= T): slot t of (b, kv head) receives k' = RoPE_t(RMSNorm(k_t)) rounded to
 * bf16 and v_t; the slots from T up to the end of T's 128-slot tile are
 * zeroed, the rest are not touched.  The attention reads K' and V back from
 * those caches.  Pointers 16-byte aligned.  Errors as swa_fwd.
 */
int swa_global_fwd(const swa_params_t* p, const swa_bf16_t* q, const swa_bf16_t* k,
                   const swa_bf16_t* v, const float* wq, const float* wk, swa_bf16_t* o,
                   float* lse, swa_bf16_t* k_cache, swa_bf16_t* v_cache, int64_t cache_cap,
                   void* stream);

/* Bytes of scratch swa_global_decode_step needs (0 if unsupported). */
size_t swa_global_decode_workspace_size(const swa_params_t* p, int64_t cache_cap);

/*
 * One decode step of a global layer for p->B sequences over their
 * full-length caches [B, Hkv, cache_cap, D] (as swa_global_fwd writes them):
 * slot pos[n] receives RoPE_pos(RMSNorm(k_new)) (bf16) and v_new, then q'
 * attends over slots 0 .. pos[n].  pos: [B] int64 device array (8-byte
 * aligned), 0 <= pos < cache_cap (else that sequence is skipped and
 * swa_get_last_device_error returns SWA_ERR_INVALID_ARG); q [B,Hq,D], k_new,
 * v_new [B,Hkv,D] bf16; writes o [B,Hq,D] bf16.  Slots past pos[n] may hold
 * anything.  `workspace`: caller-owned device scratch of
 * swa_global_decode_workspace_size bytes, 256-byte aligned.  Hq / Hkv <= 8
 * (else SWA_ERR_UNSUPPORTED).  The step reads about 4 KiB of cache per key
 * position at 8 KV heads: it is memory-bandwidth bound.
 */
int swa_global_decode_step(const swa_params_t* p, const int64_t* pos, const swa_bf16_t* q,
                           const swa_bf16_t* k_new, const swa_bf16_t* v_new, const float* wq,
                           const float* wk, swa_bf16_t* k_cache, swa_bf16_t* v_cache,
                           int64_t cache_cap, swa_bf16_t* o, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Static description of an error code. */
const char* swa_error_string(int code);

/*
 * Waits for `stream`, then returns SWA_ERR_DEVICE_TIMEOUT if any kernel of
 * this library on the current device recorded a timed-out wait since the
 * last call (the raw site code goes to *site when site != NULL), else SWA_OK.
 * Clears the record.  Returns SWA_ERR_CUDA if the stream itself failed.
 */
int swa_get_last_device_error(void* stream, int* site);

/* Library version string. */
const char* swa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SWA_H_ */
