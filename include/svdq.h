/*
 * svdq.h — C ABI of the B200 (sm_100a) SVDQuant W4A4 / AWQ W4A16 linear library.
 *
 * The method (pages: "Bringing Nunchaku 4-bit Diffusion Inference to
 * Diffusers" and its re-tellings; blog.margrop.com "技术细节 §1", the
 * four-step SVDQuant list; ainews.surl.tw paragraph 2): activation outliers
 * are moved into the weight by a smoothing vector s, the hardest part of
 * the smoothed weight is a 16-bit rank-r branch L1·L2, the residual R is
 * 4-bit, and so are the activations (W4A4).  The low-rank down-projection is
 * fused with the activation quantization and the up-projection with the
 * 4-bit GEMM, so the 16-bit branch costs almost no memory traffic:
 *
 *     x̂ = x·diag(1/s)
 *     y  = Q4(x̂)·Q4(R)ᵀ + (x̂·L1)·L2 + b            (nn.Linear layout, y = x·Wᵀ)
 *
 * On Blackwell the 4-bit format is NVFP4 (same pages, "技术细节 §3" hardware
 * table: svdq_w4a4 nvfp4 for RTX 50 / RTX PRO 6000 / B200): E2M1 element
 * codes, one E4M3 scale per 16 elements along K, and an fp32 tensor scale gs
 * such that value = e2m1 · dec(E4M3) / gs.  Modulation layers use AWQ W4A16
 * (int4 weights, 16-bit activations; ainews.surl.tw paragraph 2).
 *
 * Conventions for every call
 *  - Every pointer argument is a DEVICE pointer owned by the caller, except
 *    where a comment says otherwise.  The library allocates no device memory
 *    per call and keeps no per-call state.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *    asynchronous: they validate, enqueue kernels on `stream` and return.
 *    They never synchronize and read no device scalar on the host.
 *  - Validation happens before anything is enqueued; on any error nothing is
 *    written to any output and a status other than SVDQ_OK is returned; the
 *    thread-local svdq_last_error_detail() says why.
 *  - Device check: the kernels are built for sm_100a only (compute capability
 *    10.0, e.g. B200).  On any other device the calls return
 *    SVDQ_ERR_UNSUPPORTED_DEVICE and never launch: an unsupported GPU gets a
 *    clear error, never a wrong result (the pages' loader check, blog.margrop.com
 *    "技术细节 §3"; app.hamidun.com "Какое железо и модели поддержаны").
 *  - Tensors are row-major.  bf16 / fp16 are IEEE-style 16-bit types passed as
 *    `void*`.  Bulk operands must start on a 16-byte boundary
 *    (SVDQ_ERR_MISALIGNED otherwise).
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum svdq_status {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,        /* bad size, rank, null pointer, stride   */
  SVDQ_ERR_MISALIGNED = 2,         /* a bulk operand is not 16-byte aligned   */
  SVDQ_ERR_UNSUPPORTED_DEVICE = 3, /* current device is not compute 10.0     */
  SVDQ_ERR_CUDA = 4,               /* a CUDA runtime/driver call failed       */
  SVDQ_ERR_DEVICE_TIMEOUT = 5,     /* a bounded in-kernel wait gave up        */
  SVDQ_ERR_NOT_IMPLEMENTED = 6
} svdq_status;

/* Library version (major*10000 + minor*100 + patch). */
int svdq_version(void);

/* Static text for a status code.  Never NULL. */
const char* svdq_status_string(int status);

/* Thread-local detail of the last failing call on this host thread ("" when
 * the last call succeeded).  Valid until the next call on the same thread. */
const char* svdq_last_error_detail(void);

/* Bytes of an NVFP4 scale buffer for a [rows, K] operand in the 128x4 block
 * ("swizzled") layout: ceil(rows/128)*128 * ceil(K/64)*4.  Host-only. */
size_t svdq_nvfp4_scale_bytes(int64_t rows, int64_t K);

/*
 * svdq_quantize_act — smoothing + NVFP4 activation quantization + low-rank
 * down-projection, in one pass over x (the quantize kernel of the pages'
 * fusion: the pages put the low-rank down-projection inside the kernel
 * that quantizes the activations; blog.margrop.com "技术细节 §1" step 4).
 *
 *   x_bf16      [M, K] bf16, row stride ldx elements (ldx >= K, ldx % 8 == 0).
 *   M, K        1 <= M <= 2^30; K >= 64, K % 64 == 0, and K within the
 *               quantize kernel's shared memory (227 KB): K <= 47360 at
 *               r = 0, 46336 at 16, 45312 at 32, 43264 at 64, 39168 at 128.
 *   smooth_s    [K] fp32 smoothing vector s (> 0), 4-byte aligned.  The
 *               kernel multiplies x by RN_fp32(1/s_k).  NULL = no smoothing.
 *   L1t_bf16    L1ᵀ, [r, K] bf16 row-major (K contiguous).  Ignored if r == 0.
 *   r           low-rank rank: 0 (no branch), 16, 32, 64 or 128.
 *   act_gscale  fp32 device scalar gs_a (static tensor scale), 4-byte
 *               aligned (as is act_gscale_out).  NULL =
 *               dynamic: gs_a = 2688 / max|x̂| (1 if that max is 0), computed
 *               on the device by an extra pass over x.
 *   act_gscale_out  fp32 device scalar that receives the gs_a used; may alias
 *               act_gscale; required when act_gscale is NULL, else may be NULL.
 *   q_out       [M, K/2] bytes: E2M1 codes, element k in byte k/2, even k in
 *               the low nibble.  Quantization, per 16-element group g of a
 *               row, each step one IEEE fp32 operation:
 *                 x̂ = x·inv_s; a = max|x̂|; sf = E4M3_rn_sat((a/6)·gs_a);
 *                 d = dec(sf); codes = d == 0 ? ±0 : E2M1_rn_sat(x̂·(gs_a/d)).
 *   sf_out      svdq_nvfp4_scale_bytes(M, K) bytes: the E4M3 group scales in
 *               the 128x4 block layout the tcgen05 block-scaled MMA reads:
 *               byte ((m/128)*(K/64) + g/4)*512 + (m%32)*16 + ((m%128)/32)*4
 *               + g%4.  Rows M..ceil(M/128)*128-1 are written as zeros.
 *   lora_out    [M, r] fp32: x̂·L1 with bf16(x̂) and fp32 accumulation.
 *               NULL allowed iff r == 0.
 *   Errors: INVALID_ARG, MISALIGNED, UNSUPPORTED_DEVICE, CUDA.
 */
svdq_status svdq_quantize_act(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                              const float* smooth_s, const void* L1t_bf16, int r,
                              const float* act_gscale, float* act_gscale_out,
                              uint8_t* q_out, uint8_t* sf_out, float* lora_out,
                              void* stream);

/*
 * svdq_quantize_act_dynamic — svdq_quantize_act with the dynamic tensor scale
 * gs_a = 2688 / max|x̂| (1 if that max is 0) computed inside the same kernel
 * (one launch instead of a max pass, the quantize kernel and a finalize
 * step).  Every CTA first reads its share of x for the max, the CTAs then
 * meet at a grid-wide barrier, and the quantization reads x again (from L2
 * at these sizes).  Outputs are bit-identical to svdq_quantize_act with
 * act_gscale = NULL.
 *
 *   act_gscale_out  fp32 device scalar, receives gs_a.  Required.
 *   workspace   SVDQ_QUANTIZE_WORKSPACE_BYTES of device memory, 16-byte
 *               aligned, owned by the caller; the call clears it before its
 *               kernel runs and leaves unspecified contents.  Calls that may
 *               overlap on the GPU must use distinct workspaces.
 *   Other arguments as svdq_quantize_act.
 *   The kernel is a cooperative launch (all CTAs resident at once: at most
 *   one per SM); its grid barrier waits at most the library's wait bound
 *   (svdq_set_wait_timeout_ns), after which svdq_check_device_errors
 *   reports SVDQ_ERR_DEVICE_TIMEOUT (bit 16) and the outputs are undefined.
 *   Errors: INVALID_ARG, MISALIGNED, UNSUPPORTED_DEVICE, CUDA.
 */
#define SVDQ_QUANTIZE_WORKSPACE_BYTES 16
svdq_status svdq_quantize_act_dynamic(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                                      const float* smooth_s, const void* L1t_bf16, int r,
                                      float* act_gscale_out, void* workspace, uint8_t* q_out,
                                      uint8_t* sf_out, float* lora_out, void* stream);

/*
 * svdq_quantize_act_dynamic_noalloc — svdq_quantize_act_dynamic for callers
 * that cannot allocate device memory when they call it: an inference-engine
 * plugin whose enqueue step must not allocate, a runtime that plans all of
 * its device memory ahead of time, or a latency-bound path that must not
 * pay for an allocation.  Such a caller has no workspace to pass, so this
 * entry point keeps the kernel's scratch (the grid-barrier counter and the
 * max word, 16 bytes) in a static 256-byte device array inside the library
 * instead, and allocates nothing (no cudaMalloc, no allocating library call).
 * The pages have no counterpart; this is an interface convenience.
 *
 *   Arguments, outputs and errors as svdq_quantize_act_dynamic, without the
 *   workspace.  The outputs are those of svdq_quantize_act_dynamic.
 *   The scratch needed does not depend on M, K or r, so no problem size is
 *   rejected for it (the array's limit is 256 bytes).
 *   - The array exists once per device in every process that loads the
 *     library and is held until the process exits.
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current); make that first call before
 *     any stream capture.
 *   - Every call shares the array and clears it before its kernel runs;
 *     calls that overlap on the GPU (other streams, other threads) race on
 *     it and give undefined results.  Serialize them, or use
 *     svdq_quantize_act_dynamic with a workspace per stream.
 */
svdq_status svdq_quantize_act_dynamic_noalloc(const void* x_bf16, int64_t M, int64_t K,
                                              int64_t ldx, const float* smooth_s,
                                              const void* L1t_bf16, int r,
                                              float* act_gscale_out, uint8_t* q_out,
                                              uint8_t* sf_out, float* lora_out, void* stream);

/*
 * svdq_w4a4_linear — the 4-bit GEMM with the low-rank up-projection done
 * inside the same kernel, so the 16-bit branch adds no pass over memory
 * (blog.margrop.com "技术细节 §1", SVDQuant step 4):
 *
 *   y = bf16( dec(A)·dec(W)ᵀ + lora_act·L2 + bias )
 *
 * computed as acc = Σ e2m1_a·sfa·e2m1_w·sfw (tcgen05 block-scaled FP4 MMA,
 * fp32 in TMEM) + (hi + lo)·L2 (bf16 MMAs into the same accumulator, where
 * hi = bf16(lora_act·gs_a·gs_w) and lo = bf16(lora_act·gs_a·gs_w − hi)),
 * y = bf16(acc/(gs_a·gs_w) + bias).
 *
 *   q_act, sf_act, act_gscale   activation operand exactly as
 *               svdq_quantize_act writes it ([M, K/2] codes, scale buffer,
 *               fp32 scalar).
 *   lora_act    [M, r] fp32 (svdq_quantize_act's lora_out).  Ignored if r == 0.
 *   q_w         [N, K/2] E2M1 codes of the residual R (same packing).
 *   sf_w        svdq_nvfp4_scale_bytes(N, K) bytes, same layout.
 *   w_gscale    fp32 device scalar gs_w (4-byte aligned, as is act_gscale).
 *   L2t_bf16    L2ᵀ, [N, r] bf16 row-major (r contiguous).  Ignored if r == 0.
 *   r           0, 16, 32, 64 or 128.
 *   bias_bf16   [N] bf16 (2-byte aligned) or NULL.
 *   M, N, K     1 <= M <= 2^30; 16 <= N <= 2^30, N % 16 == 0;
 *               64 <= K <= 2^20, K % 64 == 0.
 *   y_bf16      [M, N] bf16, row stride ldy elements (ldy >= N, ldy % 8 == 0).
 *   Errors: INVALID_ARG, MISALIGNED, UNSUPPORTED_DEVICE, CUDA.
 */
svdq_status svdq_w4a4_linear(const uint8_t* q_act, const uint8_t* sf_act,
                             const float* act_gscale, const float* lora_act,
                             const uint8_t* q_w, const uint8_t* sf_w, const float* w_gscale,
                             const void* L2t_bf16, int r, const void* bias_bf16,
                             int64_t M, int64_t N, int64_t K,
                             void* y_bf16, int64_t ldy, void* stream);

/*
 * svdq_w4a4_linear_act — svdq_w4a4_linear with an activation applied in
 * the epilogue before the bf16 rounding (the fused GELU of the MLP
 * up-projection; blog.margrop.com "技术细节 §2", GELU/MLP fusion):
 *
 *   y = bf16( act( dec(A)·dec(W)ᵀ + lora_act·L2 + bias ) )
 *
 *   activation  SVDQ_ACT_NONE (0): identity, the same as svdq_w4a4_linear;
 *               SVDQ_ACT_GELU_TANH (1): 0.5·v·(1 + tanh(√(2/π)(v + 0.044715·v³)))
 *               evaluated in fp32 with the hardware tanh approximation
 *               (relative error about 2^-11, below the bf16 output rounding).
 *   Other arguments and errors as svdq_w4a4_linear; an unknown activation
 *   is INVALID_ARG.
 */
enum { SVDQ_ACT_NONE = 0, SVDQ_ACT_GELU_TANH = 1 };
svdq_status svdq_w4a4_linear_act(const uint8_t* q_act, const uint8_t* sf_act,
                                 const float* act_gscale, const float* lora_act,
                                 const uint8_t* q_w, const uint8_t* sf_w, const float* w_gscale,
                                 const void* L2t_bf16, int r, const void* bias_bf16,
                                 int64_t M, int64_t N, int64_t K,
                                 void* y_bf16, int64_t ldy, int activation, void* stream);

/*
 * svdq_w4a4_linear_split — the fused projection with its output stored in
 * `parts` separate buffers: the fused QKV projection (blog.margrop.com
 * "技术细节 §2": the original engine fuses the Q, K and V projections),
 * one quantized activation, one GEMM over the concatenated weight
 * [W_q; W_k; W_v], and Q, K and V written straight to their own tensors.
 *
 *   y = bf16( act( dec(A)·dec(W)ᵀ + lora_act·L2 + bias ) )        [M, N]
 *   columns [i·N/parts, (i+1)·N/parts) of y  ->  y_parts[i], [M, N/parts]
 *
 *   parts     1, 2 or 3.  N/parts must be a multiple of 128 when parts > 1
 *             (an output tile never straddles two parts).
 *   y_parts   HOST array of `parts` device pointers, each 16-byte aligned
 *             and row-major with leading dimension ldy; the array is read
 *             during the call only.
 *   ldy       >= N/parts, a multiple of 8.
 *   Other arguments and errors as svdq_w4a4_linear_act; parts == 1 is that
 *   call.
 */
svdq_status svdq_w4a4_linear_split(const uint8_t* q_act, const uint8_t* sf_act,
                                   const float* act_gscale, const float* lora_act,
                                   const uint8_t* q_w, const uint8_t* sf_w, const float* w_gscale,
                                   const void* L2t_bf16, int r, const void* bias_bf16,
                                   int64_t M, int64_t N, int64_t K, int parts,
                                   void* const* y_parts, int64_t ldy, int activation,
                                   void* stream);

/*
 * awq_w4a16_linear — int4-weight × bf16-activation linear for the
 * bandwidth-bound modulation layers (ainews.surl.tw paragraph 2;
 * app.hamidun.com "Что такое Nunchaku и SVDQuant"):
 *
 *   y[m,n] = bf16( Σ_k (x[m,k]·act_scale_inv[k]) · (q[n,k] − z[n,k/g])·sc[n,k/g] + b[n] )
 *
 *   x_bf16        [M, K] bf16, contiguous, 16-byte aligned.  1 <= M <= 8.
 *   K             K >= 64, K % 64 == 0; K <= 14400 for M <= 4 and K <= 7104
 *                 for M > 4 (the per-CTA activation fragment table lives in
 *                 shared memory: 16 or 32 bytes per k).
 *   act_scale_inv [K] fp32 (1/a_k of the AWQ per-channel scale), 16-byte
 *                 aligned, or NULL.
 *   qweight       [N, K/8] uint32, 16-byte aligned: nibble j (bits 4j..4j+3)
 *                 of word w of row n is q[n, 8w + j], an unsigned 0..15.
 *   scales_f16, zeros_f16   [N, K/group] fp16, 2-byte aligned; zeros hold
 *                 integers 0..15.
 *   group         must be 64.
 *   bias_bf16     [N] bf16 (2-byte aligned) or NULL.
 *   N             16 <= N <= 2^30, N % 16 == 0.
 *   y_bf16        [M, N] bf16, contiguous, 2-byte aligned.
 *   Results do not depend on the kernel chosen beyond fp32 summation order:
 *   K % 256 == 0, K <= 3072, scales and zeros 16-byte aligned and at most
 *   16 row strips of 16 per SM go to a weight-streaming kernel (16-row
 *   strips through a shared-memory ring by TMA); every other shape to a
 *   register-streaming kernel, which sets the K limits above.
 *   Errors: INVALID_ARG, MISALIGNED, UNSUPPORTED_DEVICE, CUDA.
 */
svdq_status awq_w4a16_linear(const void* x_bf16, int64_t M, int64_t K,
                             const float* act_scale_inv, const uint32_t* qweight,
                             const void* scales_f16, const void* zeros_f16, int group,
                             const void* bias_bf16, int64_t N, void* y_bf16, void* stream);

/*
 * svdq_check_device_errors — synchronizes `stream` and reports whether any
 * kernel of this library on the current device gave up a bounded in-kernel
 * wait (SVDQ_ERR_DEVICE_TIMEOUT; the device error word is then cleared) or
 * the stream holds a CUDA error (SVDQ_ERR_CUDA).  For tests and debugging:
 * it blocks the host.
 */
svdq_status svdq_check_device_errors(void* stream);

/*
 * svdq_set_wait_timeout_ns — upper bound, in nanoseconds of %globaltimer,
 * on every in-kernel wait of later launches from this process (default
 * 2e9 = 2 s; 0 restores the default).  After the bound a kernel records
 * SVDQ_ERR_DEVICE_TIMEOUT in the device error word, drains its own copies,
 * frees its tensor memory and returns.  Returns the previous value.
 */
uint64_t svdq_set_wait_timeout_ns(uint64_t ns);

/*
 * svdq_set_gemm_pairs — how later svdq_w4a4_linear* launches from this
 * process tile the output.  enable = 0 (the default): 128 x 192 tiles where
 * 192 divides N / parts, else 128 x 128, each on one SM.  enable = 1: where
 * M > 128, 256 x 192 (or 256 x 128) tiles, each computed by a pair of SMs (a
 * 2-CTA cluster) with one tcgen05 MMA over both SMs' shared and tensor
 * memory.  Both give results within the same bound of the exact product (the
 * accumulation order inside a tile may differ).  On B200 the one-SM tiles
 * are the faster of the two for the shapes measured (the pair's block scales
 * are staged into each SM's tensor memory by that SM's warps, and the signal
 * that both SMs' scales are in place crosses SMs every K step).  Returns the
 * previous setting.  Host-only; never fails.
 */
int svdq_set_gemm_pairs(int enable);

/*
 * svdq_set_pdl — whether later launches from this process allow
 * programmatic dependent launch (CUDA's launch attribute
 * programmaticStreamSerialization; default 1).  With it a kernel of this
 * library may be scheduled onto the GPU while the kernel before it on the
 * stream is still finishing; it initialises its barriers, allocates its
 * tensor memory and prefetches its tensor-map descriptors, then waits for
 * that kernel to complete and its writes to be visible (griddepcontrol.wait)
 * before it touches any operand in global memory, so every argument keeps
 * plain stream-order semantics.  Each kernel also signals at its start that
 * the next one may be scheduled.  0 launches in plain stream order.
 * awq_w4a16_linear with M > 4 always launches in plain stream order (it
 * measured slower on B200 with the attribute).  The pages have no
 * counterpart (this is a launch property of the B200 implementation).
 * Returns the previous setting.  Host-only; never fails.
 */
int svdq_set_pdl(int enable);

/*
 * svdq_debug_set_fault — TEST HOOK.  flags = 1 makes the next launches of
 * svdq_w4a4_linear skip one producer arrive so that the consumer's bounded
 * wait runs out; flags = 2 makes the first CTA of the next
 * svdq_quantize_act_dynamic launches skip its arrival at the grid barrier so
 * that the other CTAs' bounded waits run out (host-side fault injection;
 * nothing traps or faults).  0 clears it.  Returns the previous flags.
 */
int svdq_debug_set_fault(int flags);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H_ */
