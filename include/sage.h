/*
 * sage.h -- C ABI of libsage.so: SageAttention-style quantized attention
 * forward for NVIDIA B200 (sm_100a).
 *
 * Method sources (web pages):
 *   [SA1]   "SageAttention: Accurate 8-Bit Attention for Plug-and-Play
 *           Inference Acceleration" (review page): Algorithm 1 (SAGEAttn-B),
 *           Eq. 4-5, Eq. 6 (Smooth K), implementation details 1-2.
 *   [SA2++] "SageAttention2++: A More Efficient Implementation of
 *           SageAttention2" (review page): section "核心公式" (delta_Q,
 *           delta_K, delta_P, delta_V formulas; Eq. (1)-(2)).
 *
 * Conventions shared by every entry point
 *   - Tensors are dense, row-major, in device memory unless the name says
 *     "host".  Q and O are [B, H, N, d]; K and V are [B, H_kv, N, d]
 *     (the (B, H, N, d) shapes of [SA1] Table 7).  d is the innermost axis.
 *   - d must be 64 or 128; H must be a multiple of H_kv (query head h reads
 *     kv head h / (H / H_kv)).  N may be any value >= 0; the last 128-token
 *     block of a ragged sequence is short.  B == 0 or N == 0 is a no-op.
 *   - q, k, v, o, q_hat, k_hat, v_hat must be 16-byte aligned (TMA and
 *     vector access); fp32 arrays 4-byte aligned.  Violations return
 *     SAGE_ERR_MISALIGNED before anything is launched.
 *   - The caller owns all memory.  Calls keep no state between them.
 *   - `stream` is a cudaStream_t passed as an opaque pointer (NULL = the
 *     legacy default stream).  Calls are stream-ordered and asynchronous:
 *     the returned status covers argument checks and launch errors only.
 *     Execution errors surface at the caller's next synchronization, or
 *     through sage_get_device_error().
 *   - Inputs holding NaN or Inf are outside the contract.
 *   - There is no CPU or other-architecture fallback: a current device
 *     that is not compute capability 10.0 gives SAGE_ERR_DEVICE.
 *   - Quantization blocks are 128 tokens of one head (b_q = b_kv = 128),
 *     so the scale arrays have nb = ceil(N / 128) entries per head.
 */
#ifndef SAGE_H_
#define SAGE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SAGE_OK = 0,
  SAGE_ERR_INVALID_ARG = 1,     /* null pointer, negative size, sm_scale <= 0 or not finite */
  SAGE_ERR_UNSUPPORTED = 2,     /* d not in {64,128}, H % H_kv != 0, unknown variant        */
  SAGE_ERR_MISALIGNED = 3,      /* a device pointer not 16-byte aligned                      */
  SAGE_ERR_DEVICE = 4,          /* current device is not compute capability 10.0 (B200)      */
  SAGE_ERR_CUDA = 5,            /* a CUDA runtime / driver call failed                       */
  SAGE_ERR_DEVICE_TIMEOUT = 6,  /* a kernel gave up on a bounded wait (see device error)     */
  SAGE_ERR_NO_MEMORY = 7        /* stream-ordered allocation failed / workspace too small    */
} sage_status_t;

typedef enum {
  /* INT8 Q K^T, P~ and V in fp16 for P~V, fp32 accumulator ([SA1] Algorithm 1). */
  SAGE_VARIANT_B = 0,
  /* INT8 Q K^T, P~ and V in FP8 E4M3 ("8+8" of [SA2++]): static delta_P = 1/448,
   * per-channel delta_V = colmax|V| / 448, fp32 accumulator. */
  SAGE_VARIANT_8P8 = 1,
  /* 8+8 with the narrowed ranges of [SA2++] Eq. (2) and Table 2, P_r = 56 and
   * V_r = 9: P operand = e4m3(56 P~), delta_V = colmax|V| / 9.  The [SA2++]
   * pair is chosen so that an FP16 accumulator cannot overflow; tcgen05 runs
   * E4M3 MMAs with an fp32 accumulator at the same rate, so the accumulator
   * here stays fp32 in tensor memory.  Same operand layout as SAGE_VARIANT_8P8
   * (v_hat must be quantized with v_r = 9 for sage_attn_fwd_quantized). */
  SAGE_VARIANT_8P8_R56 = 2
} sage_variant_t;

/*
 * Pre-pass for Q and K ([SA1] Algorithm 1 steps 1-2, Eq. 6; [SA2++] delta_Q,
 * delta_K formulas).
 *   q      : fp16 [B,H,N,d]        k : fp16 [B,H_kv,N,d]       (inputs)
 *   q_hat  : int8 [B,H,N,d]        = RNE(x_q / delta_q[blk]), x_q = fp32(q) * sm_scale
 *   k_hat  : int8 [B,H_kv,N,d]     = RNE(x_k / delta_k[blk]), x_k = fp32(k) - mean_k[c]
 *   delta_q: fp32 [B,H,nb]         = max|x_q over the block| / 127  (0 for an all-zero block)
 *   delta_k: fp32 [B,H_kv,nb]      = max|x_k over the block| / 127
 *   mean_k : fp32 [B,H_kv,d]       = (1/N) sum_t k[t,c]; the sum is exact (fixed point,
 *                                    units of 2^-24), converted to fp64, divided by N
 *                                    in fp64, rounded once to fp32.
 * Both divisions are IEEE fp32 round-to-nearest; codes lie in [-127, 127].
 * Results are bit-identical whatever the launch configuration.
 * Scratch: takes ceil(N/256)*B*H_kv*d*8 bytes of stream-ordered device memory
 * (cudaMallocAsync on `stream`, freed on `stream`).
 */
sage_status_t sage_smooth_quant_qk(const void* q, const void* k, int B, int H, int H_kv,
                                   int N, int d, float sm_scale, int8_t* q_hat, int8_t* k_hat,
                                   float* delta_q, float* delta_k, float* mean_k, void* stream);

/*
 * sage_smooth_quant_qk without any device allocation.  The paper has no
 * counterpart: this entry point exists for callers that must not allocate
 * device memory while they run, for example a serving runtime that plans all
 * of its device memory up front and treats any allocation after warm-up as an
 * error, or code that runs where the stream-ordered memory pool of the device
 * is owned by someone else.  Arguments, layouts and results are those of
 * sage_smooth_quant_qk, bit for bit.
 *
 * Scratch: the int64 partial column sums of K (B*H_kv*ceil(N/256)*d of them)
 * go to a static array in the library's device memory, 4 MiB per device
 * (524,288 entries: e.g. B*H_kv = 32 heads of N = 32768 tokens at d = 128).
 * Larger sizes are rejected with SAGE_ERR_UNSUPPORTED before anything is
 * launched (sage_last_error_detail() says why); use sage_smooth_quant_qk for
 * them.  No entry of the array has to start at zero: each call writes every
 * partial sum it later reads.
 *
 * Set-up: the first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and keeps it for the life
 * of the process; make that first call before any stream capture begins.
 * cudaDeviceReset() on that device invalidates the kept address (the
 * library's device memory is created anew): a process that resets a device
 * must unload and reload libsage.so before calling this entry point again.
 *
 * Concurrency: there is ONE array per device.  Calls issued in order on one
 * stream are safe; calls that may overlap on the same device (other streams,
 * other host threads) race on it and can produce wrong results, since the
 * array keeps whatever the last writer left.  Order such calls with events.
 */
sage_status_t sage_smooth_quant_qk_noalloc(const void* q, const void* k, int B, int H,
                                           int H_kv, int N, int d, float sm_scale,
                                           int8_t* q_hat, int8_t* k_hat, float* delta_q,
                                           float* delta_k, float* mean_k, void* stream);

/*
 * FP8 E4M3 quantization of V for the 8+8 variant ([SA2++] delta_V formula and
 * Eq. (2) with a general V_r).
 *   v      : fp16 [B,H_kv,N,d]
 *   v_r    : top of the code range (448 for 8+8); must be in (0, 448]
 *   v_hat  : uint8 E4M3 codes, [B,H_kv,N,d] (the layout of v; see sage_v_hat_layout)
 *            = e4m3_rne_satfinite(fp32(v) / delta_v[c])
 *   delta_v: fp32 [B,H_kv,d] = max_t |v[t,c]| / v_r (IEEE fp32 division; 0 -> codes 0)
 * Scratch: ceil(N/256)*B*H_kv*d*4 bytes, stream-ordered as above.
 */
sage_status_t sage_quant_v_fp8(const void* v, int B, int H_kv, int N, int d, float v_r,
                               uint8_t* v_hat, float* delta_v, void* stream);

/*
 * The whole pre-pass in three launches (column statistics of K and V, their
 * finalisation, one quantization launch for Q, K and V): the results of
 * sage_smooth_quant_qk and, when v != NULL, of sage_quant_v_fp8 with the
 * given v_r, bit for bit.  v, v_hat and delta_v are either all NULL
 * (SAGEAttn-B needs no V pre-pass) or all set.
 * Scratch: ceil(N/256)*B*H_kv*d*12 bytes, stream-ordered as above.
 */
sage_status_t sage_smooth_quant_qkv(const void* q, const void* k, const void* v, int B, int H,
                                    int H_kv, int N, int d, float sm_scale, float v_r,
                                    int8_t* q_hat, int8_t* k_hat, uint8_t* v_hat, float* delta_q,
                                    float* delta_k, float* mean_k, float* delta_v, void* stream);

/*
 * sage_smooth_quant_qkv with a rotary position embedding of Q and K fused in
 * front of the quantizers ([SA1] implementation detail 1: Q and K are rotated
 * and quantized in one pass, with no rotated copy written to HBM; the
 * SageAttention summary page's fused RoPE + quantization kernel).
 *   cos_t, sin_t: fp32 [N, d/2] device tables, 16-byte aligned, shared by all
 *                 batches and heads: row t holds cos/sin of token t's angles.
 * Rotate-half pairing: channel i < d/2 pairs with i + d/2; with c = cos_t[t,i],
 * s = sin_t[t,i] (fp32 products, then the sum, each rounded to nearest),
 *   x'[i]       = fp16( x[i] * c - x[i+d/2] * s )
 *   x'[i+d/2]   = fp16( x[i+d/2] * c + x[i] * s )
 * and the results are those of sage_smooth_quant_qkv on the rotated fp16 Q
 * and K, bit for bit (V is not rotated).  Scratch as sage_smooth_quant_qkv.
 */
sage_status_t sage_smooth_quant_qkv_rope(const void* q, const void* k, const void* v,
                                         const float* cos_t, const float* sin_t, int B, int H,
                                         int H_kv, int N, int d, float sm_scale, float v_r,
                                         int8_t* q_hat, int8_t* k_hat, uint8_t* v_hat,
                                         float* delta_q, float* delta_k, float* mean_k,
                                         float* delta_v, void* stream);

/*
 * Attention on pre-quantized operands ([SA1] Algorithm 1 steps 3-9, Eq. 4-5):
 * per 128-row q block and ascending 128-key kv tiles,
 *   S = int32(q_hat k_hat^T) * delta_q[i] * delta_k[j]   (tcgen05 kind::i8)
 *   online softmax (running max m, row sum l, rescale of O)
 *   O += P~ V  (variant B: fp16 P~ and fp16 V; 8+8: e4m3(448 P~) and v_hat)
 *   O = O / l  (8+8: times delta_v[c] / 448), rounded to fp16.
 *   v_or_vhat: fp16 V for SAGE_VARIANT_B, E4M3 codes for SAGE_VARIANT_8P8 / _R56
 *   delta_v  : fp32 [B,H_kv,d] for 8+8, ignored (may be NULL) for B
 *   o        : fp16 [B,H,N,d] output
 *   causal   : 0 or 1; square, top-left aligned mask (key t visible to query r iff t <= r)
 * The kernel runs one CTA per SM, each walking a fixed list of work items
 * (two 128-row q blocks of one head); causal lists hold the longest items
 * first.  No scratch memory.
 */
sage_status_t sage_attn_fwd_quantized(const int8_t* q_hat, const int8_t* k_hat,
                                      const float* delta_q, const float* delta_k,
                                      const void* v_or_vhat, const float* delta_v, void* o,
                                      int B, int H, int H_kv, int N, int d, int causal,
                                      int variant, void* stream);

/* Bytes of workspace sage_attn_fwd_ws needs for these sizes (0 for empty inputs). */
size_t sage_attn_workspace_bytes(int B, int H, int H_kv, int N, int d, int variant);

/*
 * Whole forward pass ([SA1] Algorithm 1 with Smooth K; variant selects B or 8+8):
 * pre-pass kernels then the attention kernel, on `stream`.
 *   q, k, v : fp16 inputs as above; o : fp16 [B,H,N,d] output
 *   sm_scale: softmax scale folded into the quantization of Q (> 0, finite;
 *             1/sqrt(d) is the usual value)
 * Intermediates (q_hat, k_hat, scales, mean_k, v_hat, scratch) come from
 * cudaMallocAsync on `stream` and are freed on `stream` (_ws: from the
 * caller's workspace of at least sage_attn_workspace_bytes() bytes,
 * 256-byte aligned; SAGE_ERR_NO_MEMORY if it is smaller).
 */
sage_status_t sage_attn_fwd(const void* q, const void* k, const void* v, void* o, int B, int H,
                            int H_kv, int N, int d, int causal, float sm_scale, int variant,
                            void* stream);
sage_status_t sage_attn_fwd_ws(const void* q, const void* k, const void* v, void* o, int B,
                               int H, int H_kv, int N, int d, int causal, float sm_scale,
                               int variant, void* workspace, size_t ws_bytes, void* stream);

/*
 * End-to-end call on HOST buffers: copies q, k, v (fp16, host memory; pinned
 * memory gives full PCIe/C2C bandwidth and lets copies overlap the kernels)
 * to the current device, runs the whole pass, copies o back to host memory
 * and synchronizes `stream` before returning.  The (batch, kv head) units are
 * processed in up to 8 chunks: copies in run on an internal stream, the
 * kernels on `stream`, copies out on a second internal stream, so one
 * chunk's transfers overlap another chunk's kernels.  The results equal
 * sage_attn_fwd's.  Device buffers are stream-ordered allocations on
 * `stream`, freed before return.  The two internal streams and their events
 * are created on a device's first call and reused by later calls (a call
 * made while another one holds them on the same device creates and
 * destroys its own); after cudaDeviceReset the library must be reloaded
 * before the next call on that device.
 */
sage_status_t sage_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                                 void* o_host, int B, int H, int H_kv, int N, int d, int causal,
                                 float sm_scale, int variant, void* stream);

/*
 * Variable-length batches: B sequences of different lengths packed along the
 * token axis (the models of [SA1] Table 7 have lengths that are not
 * multiples of the block size, N = 17776 or N = 1105; batching them without
 * padding means packing).  Every sequence is its own attention problem, with
 * its own mean(K), its own 128-token blocks counted from its first token and
 * its own delta_V: the results for sequence b are those of the fixed-length
 * entry points on that sequence alone (B = 1, N = its length).
 *   q, o      : fp16 [H, T, d]      k, v : fp16 [H_kv, T, d]
 *   cu_seqlens: int32 [B+1] in DEVICE memory, non-decreasing, cu_seqlens[0]
 *               = 0 and cu_seqlens[B] = T: sequence b holds tokens
 *               cu_seqlens[b] .. cu_seqlens[b+1]-1 of every head
 *   max_seqlen: host value >= every cu_seqlens[b+1] - cu_seqlens[b]; sizes
 *               the per-sequence arrays below (nbm = ceil(max_seqlen / 128))
 *   T         : total tokens (<= 2^30)
 * Offsets outside [0, T] are clamped and lengths above max_seqlen cut, so
 * malformed offsets give wrong results for the affected sequences but never
 * an access outside the tensors.  Causal masks are per sequence (key t
 * visible to query r of the same sequence iff t <= r).
 */

/* Pre-pass of a packed batch (sage_smooth_quant_qkv per sequence).
 *   q_hat: int8 [H, T, d]; k_hat, v_hat: [H_kv, T, d] (v, v_hat, delta_v: all
 *          NULL for SAGEAttn-B, or all set)
 *   delta_q: fp32 [B, H, nbm]; delta_k: fp32 [B, H_kv, nbm] (entries past a
 *          sequence's last block are not written)
 *   mean_k, delta_v: fp32 [B, H_kv, d]
 * Scratch: B*H_kv*ceil(max_seqlen/256)*d*12 bytes, stream-ordered. */
sage_status_t sage_smooth_quant_qkv_varlen(const void* q, const void* k, const void* v,
                                           const int32_t* cu_seqlens, int B, int max_seqlen, int T,
                                           int H, int H_kv, int d, float sm_scale, float v_r,
                                           int8_t* q_hat, int8_t* k_hat, uint8_t* v_hat,
                                           float* delta_q, float* delta_k, float* mean_k,
                                           float* delta_v, void* stream);

/* Attention of a packed batch on pre-quantized operands (layouts as written
 * by sage_smooth_quant_qkv_varlen; v_or_vhat fp16 [H_kv, T, d] for B, E4M3
 * codes for 8+8).  No scratch memory. */
sage_status_t sage_attn_fwd_varlen_quantized(const int8_t* q_hat, const int8_t* k_hat,
                                             const float* delta_q, const float* delta_k,
                                             const void* v_or_vhat, const float* delta_v, void* o,
                                             const int32_t* cu_seqlens, int B, int max_seqlen, int T,
                                             int H, int H_kv, int d, int causal, int variant,
                                             void* stream);

/* Whole forward pass of a packed batch; intermediates stream-ordered on
 * `stream` as for sage_attn_fwd. */
sage_status_t sage_attn_fwd_varlen(const void* q, const void* k, const void* v, void* o,
                                   const int32_t* cu_seqlens, int B, int max_seqlen, int T, int H,
                                   int H_kv, int d, int causal, float sm_scale, int variant,
                                   void* stream);

/* Layout of v_hat: 0 = [B,H_kv,N,d] (same as v).  Always 0 in this library. */
int sage_v_hat_layout(void);

/*
 * Synchronizes `stream`, then reads and clears the library's device error
 * word on the current device.  Returns SAGE_OK, SAGE_ERR_DEVICE_TIMEOUT if a
 * kernel abandoned a bounded wait (it then skipped the rest of its work,
 * released its tensor memory and exited), or SAGE_ERR_CUDA.
 * If `detail` is not NULL it receives the raw error word (bit 0: timeout;
 * bits 8-15: which wait gave up).
 */
sage_status_t sage_get_device_error(void* stream, uint32_t* detail);

/* Upper bound, in nanoseconds, of every bounded wait inside the kernels
 * (default 2e9).  Applies to launches made after the call; process-wide. */
void sage_set_wait_timeout_ns(uint64_t ns);

/*
 * Failure-detection self-test: launches one CTA that waits on a shared-memory
 * barrier nothing will ever complete, with the bound `timeout_ns`.  The wait
 * gives up, records a timeout in the device error word and the kernel exits
 * normally; sage_get_device_error() then reports SAGE_ERR_DEVICE_TIMEOUT.
 */
sage_status_t sage_selftest_wait_timeout(uint64_t timeout_ns, void* stream);

/* Description of the step that last failed in this thread (for SAGE_ERR_CUDA
 * and friends): the CUDA call, its error string and code.  "none" if no
 * failure was recorded.  The pointer stays valid until the thread's next call. */
const char* sage_last_error_detail(void);

/* Static description of a status code. */
const char* sage_status_string(sage_status_t status);

/* Library version, as "major.minor.patch". */
const char* sage_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_H_ */
