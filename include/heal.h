/*
 * heal.h -- C ABI of libheal.so, the B200 (sm_100a) hot path of HEAL.
 *
 * HEAL ("Demystifying Numerical Instability in LLM Inference: Achieving Reproducible
 * Inference for Mission-Critical Tasks with HEAL", arXiv 2606.21023) keeps FP32-level
 * numerics without an FP32 pipeline:
 *   - GEMMs are synthesised on 16-bit tensor cores by algebraic error compensation
 *     (authors' v2 abstract; gist.science technical summary, section 2.B);
 *   - Q/K/V are stored as INT16 and unpacked into FP16 pairs for the attention
 *     contractions (abstract; technical summary, section 2.A).
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library never
 *     allocates, frees or retains them; scratch comes from caller-provided workspaces.
 *   - Every call is asynchronous and stream-ordered on `stream` (NULL = legacy default
 *     stream).  Arguments are validated on the host before any launch; a rejected call
 *     launches nothing and leaves every output untouched.
 *   - Return codes: HEAL_OK, HEAL_ERR_INVALID_ARGUMENT (null pointer, bad size, stride
 *     or alignment), HEAL_ERR_UNSUPPORTED (valid but outside what the kernels cover),
 *     HEAL_ERR_CUDA (a CUDA runtime error at launch; the CUDA error is cleared).
 *     Device-side failures (a bounded wait that ran out) are reported asynchronously by
 *     heal_get_device_status().
 *   - Matrices are row-major with explicit leading dimensions in elements.  No C++
 *     exception crosses this boundary.
 */
#ifndef HEAL_H_
#define HEAL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* heal_stream_t;

typedef enum {
  HEAL_OK = 0,
  HEAL_ERR_INVALID_ARGUMENT = 1,
  HEAL_ERR_UNSUPPORTED = 2,
  HEAL_ERR_CUDA = 3,
  HEAL_ERR_TIMEOUT = 4
} heal_status_t;

/* 16-bit format of the hi/lo residual split (technical summary, section 2.B: "a primary
 * 16-bit value and a residual error term"; the overflow remark there names FP16).
 *   HEAL_SPLIT_FP16_S11: hi = fp16_rn(x), lo = fp16_rn((x - hi) * 2^11); the products
 *                        that use lo are scaled by 2^-11.  Default; FP32-level accuracy.
 *   HEAL_SPLIT_BF16:     hi = bf16_rn(x), lo = bf16_rn(x - hi).  Wider range, ~16 bits. */
typedef enum { HEAL_SPLIT_FP16_S11 = 0, HEAL_SPLIT_BF16 = 1 } heal_split_fmt_t;

/* Fixed tile configurations of heal_gemm_compensated.  All configurations produce
 * bitwise-identical C (see heal_gemm_compensated).  HEAL_TILE_AUTO picks by shape. */
enum {
  HEAL_TILE_AUTO = -1,
  HEAL_TILE_128x128 = 0,      /* 1 CTA per tile, full K per tile                        */
  HEAL_TILE_256x256_PAIR = 1, /* a cluster of 2 CTAs per 256x256 tile (tcgen05 cta_group::2):
                                 each CTA stages and splits 128 rows of A and 128 columns of
                                 B; the default for M, N >= 256                           */
  HEAL_TILE_SKINNY_SPLITK = 2, /* operands swapped (weights on the MMA M side), K split
                                 over CTAs; needs a workspace (M <= 64)                 */
  HEAL_TILE_SKINNY_FULLK = 3,  /* operands swapped, full K per CTA, no workspace (M <= 64) */
  HEAL_TILE_SKINNY_CHAIN = 4   /* operands swapped, K split over a cluster of 2-8 CTAs per
                                 128-row tile of C^T; each CTA keeps its chunks in TMEM and
                                 the running sum passes from CTA to CTA in ascending chunk
                                 order through distributed shared memory; no workspace.
                                 M <= 32; other shapes (or too few SMs for two CTAs per
                                 tile) run HEAL_TILE_SKINNY_FULLK.  The automatic choice
                                 for M <= 32 when no workspace is given                   */
};

typedef struct {
  int tile_config;          /* HEAL_TILE_* ; -1 = automatic                                  */
  const int8_t* chan_exp;   /* nullable device pointer, int8 [K]: outlier-channel rescale.
                               Column k of A is multiplied by 2^-e_k and row k of B by 2^e_k
                               before the split.  Powers of two, so A.B is unchanged; it
                               keeps FP16 hi parts finite for large channels (technical
                               summary, section 2.B, "Overflow Handling").  |e_k| <= 64.   */
  int b_layout;             /* 0: B is K x N row-major (ldb >= N); 1: B is N x K row-major
                               (ldb >= K), the torch.nn.Linear weight layout                 */
  int b_presplit;           /* 0: B is FP32 and is split by the kernel.
                               1: `B` holds the 16-bit hi part and `b_lo` the lo part, both
                                  written by heal_split in `fmt`, in b_layout; the kernel
                                  splits only A (same bits as 0).
                               2: `B` is a 16-bit matrix in fmt's 16-bit type (FP16 for
                                  HEAL_SPLIT_FP16_S11, BF16 for HEAL_SPLIT_BF16) with no
                                  residual: only A is split and C = Ah.B + s.Al.B, the
                                  two-product form of the technical summary, section 2.B
                                  (16-bit weights, half the weight bytes); b_lo must be null.
                               With 1 or 2 the kernel applies chan_exp to A only: B's rows
                               must already carry the factor 2^e_k.                         */
  const void* b_lo;         /* lo part when b_presplit = 1, else null                        */
  void* workspace;          /* device scratch for HEAL_TILE_SKINNY_SPLITK (nullable; 16-byte
                               aligned): the per-chunk values [K/64][M][N] FP32, added in
                               ascending chunk order by a second kernel.  Its contents need
                               no initialisation.                                          */
  size_t workspace_bytes;
  int b_static;             /* 1: B (and b_lo) are not written by work queued before this call
                               on the stream (weights).  GEMM kernels start with programmatic
                               dependent launch and wait for the preceding kernel before they
                               touch A, chan_exp, C or the workspace; with b_static they may
                               request the first stages of B before that wait.  0: B is
                               waited for like A.                                           */
  int b_split_pass;         /* 1 (b_presplit = 0, chan_exp null, B contiguous: ldb = N or K):
                               B is split once per call by heal_split's kernel into the
                               workspace (its hi and lo parts, 4*K*N bytes after the split-K
                               part) and the product then reads the 16-bit parts, as with
                               b_presplit = 1.  The same bits as 0; for large B the two
                               launches are faster than splitting B inside every tile.
                               heal_gemm_workspace_bytes counts these bytes when the flag
                               is set.                                                       */
  int reserved[2];          /* must be zero                                                  */
} heal_gemm_opts_t;

/* K1. Hi/lo split of n FP32 values (technical summary, section 2.B, "Mechanism").
 *   x  : device, float32 [n]
 *   hi : device, 16-bit [n] (fp16 or bf16 encodings per fmt), written
 *   lo : device, 16-bit [n], written
 * Elementwise, round-to-nearest-even; |x| >= 65520 gives an infinite FP16 hi.
 * n == 0 is a no-op.  Pointers must be 4-byte aligned (16-byte for full speed).      */
heal_status_t heal_split(const float* x, void* hi, void* lo, int64_t n,
                         heal_split_fmt_t fmt, heal_stream_t stream);

/* K2/K3. Error-compensated GEMM  C = A . B  on 16-bit tensor cores (authors' abstract;
 * technical summary, section 2.B).
 *   A : device float32, M x K row-major, leading dimension lda >= K
 *   B : device float32 (or 16-bit hi when opts->b_presplit), layout per opts->b_layout
 *   C : device float32, M x N row-major, ldc >= N; FP32 result, no 16-bit store.
 * Both operands are split into hi/lo in shared memory by the kernel and
 *   C = Ah.Bh + s.(Ah.Bl + Al.Bh),  s = 2^-11 (FP16_S11) or 1 (BF16),
 * with FP32 accumulation.  K is processed in chunks of 64: each chunk's value comes
 * from the tensor cores, and chunk values are added in ascending order in FP32 round-
 * to-nearest.  The result is therefore identical bit for bit across runs and across
 * tile configurations.
 * Alignment: A, B, C (and b_lo) 16-byte aligned; lda, ldb multiples of 4 (8 for a
 * pre-split B).  M, N, K >= 1 and < 2^31.  HEAL_TILE_SKINNY_SPLITK needs
 * opts->workspace of at least heal_gemm_workspace_bytes(); other configs need none.   */
heal_status_t heal_gemm_compensated(int M, int N, int K,
                                    const float* A, int64_t lda,
                                    const void* B, int64_t ldb,
                                    float* C, int64_t ldc,
                                    heal_split_fmt_t fmt,
                                    const heal_gemm_opts_t* opts, /* nullable: defaults */
                                    heal_stream_t stream);

/* Workspace bytes that heal_gemm_compensated needs for this shape and tile config
 * (0 when the config uses none).  Host-only, no CUDA call.                            */
size_t heal_gemm_workspace_bytes(int M, int N, int K, const heal_gemm_opts_t* opts);

/* K4. INT16 quantization of Q/K/V rows into a cache (technical summary, section 2.A).
 *   x : device, bf16 (x_is_bf16 = 1) or float32, logical [B, T, H, D] with element
 *       strides (x_stride_batch, x_stride_tok, x_stride_head, 1)
 *   q_cache     : device int16 [B, H, Tmax, D], rows t_offset .. t_offset+T-1 written
 *   scale_cache : device float32 [B, H, Tmax], same rows written
 * Per (token, head) row: absmax = max|x|, inv = fp32(32767/absmax),
 * q = clamp(rint(fp32(x*inv)), +-32767), s = fp32(absmax/32767); an all-zero row gives
 * q = 0, s = 0.  D must be a power of two in [8, 256]; x, q_cache 16-byte aligned;
 * strides multiples of 8 elements.  t_offset + T <= Tmax.  Rows holding a NaN or an
 * infinity get unspecified codes (the definition above does not cover them).          */
heal_status_t heal_kv_quantize_int16(const void* x, int x_is_bf16,
                                     int B, int T, int H, int D,
                                     int64_t x_stride_batch, int64_t x_stride_tok,
                                     int64_t x_stride_head,
                                     int16_t* q_cache, float* scale_cache,
                                     int Tmax, int t_offset, heal_stream_t stream);

/* K5. Attention on INT16 Q/K/V (technical summary, section 2.A "Mechanism").
 *   q          : device int16 [B, Hq, Tq, D]        q_scale : float32 [B, Hq, Tq]
 *   k_cache    : device int16 [B, Hkv, Tmax, D]     k_scale : float32 [B, Hkv, Tmax]
 *   v_cache    : device int16 [B, Hkv, Tmax, D]     v_scale : float32 [B, Hkv, Tmax]
 *   kv_len     : device int32 [B], 1 <= kv_len[b] <= Tmax (tokens 0..kv_len-1 valid)
 *   out        : device float32 [B, Hq, Tq, D]
 * Query head h reads KV head h / (Hq/Hkv).  Query i sits at position kv_len - Tq + i;
 * with causal = 1 it sees tokens t <= its position.  QK^T is the exact integer dot
 * product (each INT16 value byte-split into a signed high byte and an unsigned low byte,
 * four 8-bit integer tensor-core products, combined in int64); FP32 online softmax; PV
 * with P split into two FP16 parts and V byte-split into two exact FP16 values.
 * Two kernels, chosen by the number of query rows per KV head, R = (Hq/Hkv) * Tq:
 *   R <= 8 (decode): logit * log2(e) = fp32(fp32(fp32(S_int) * s_k) *
 *     fp32(s_q * softmax_scale * log2(e))) in FP32, as in the prefill kernel; the context
 *     is cut into chunks whose partial results are merged in ascending chunk order.
 *   R > 8 (prefill, D = 128 only): 128 query rows per tile on the tcgen05 tensor cores;
 *     logit * log2(e) = fp32(fp32(S_int) * s_k) * fp32(s_q * softmax_scale * log2(e))
 *     in FP32; a conversion pass first writes the byte planes of Q, K and V into the
 *     workspace.
 * Both are deterministic (identical results from run to run).
 * Limits: D in {64, 128} (128 when R > 8); Hq % Hkv == 0; Tmax % 64 == 0;
 * q, the caches, k_scale, v_scale, out and workspace 16-byte aligned.
 * workspace  : device, >= heal_attention_workspace_bytes_gqa(B, Hq, Hkv, Tq, Tmax) bytes
 *              (heal_attention_workspace_bytes(B, Hq, Tq, Tmax) is an upper bound)
 * qk_int_out : nullable test hook, int64 [B, Hq, Tq, Tmax]; when given, the exact
 *              S_int of every visible (query, token) pair is written there.          */
heal_status_t heal_attention_int16(const int16_t* q, const float* q_scale,
                                   const int16_t* k_cache, const float* k_scale,
                                   const int16_t* v_cache, const float* v_scale,
                                   int B, int Hq, int Hkv, int D, int Tq,
                                   const int32_t* kv_len, int Tmax,
                                   float softmax_scale, int causal, float* out,
                                   void* workspace, size_t workspace_bytes,
                                   int64_t* qk_int_out, heal_stream_t stream);

/* Scratch bytes for heal_attention_int16 (host-only, no CUDA call).  The _gqa form is
 * exact for the given Hkv; the short form is an upper bound valid for every Hkv that
 * divides Hq (for Tq = 1: every Hkv with Hq/Hkv <= 8).  0 for invalid sizes.         */
size_t heal_attention_workspace_bytes_gqa(int B, int Hq, int Hkv, int Tq, int Tmax);
size_t heal_attention_workspace_bytes(int B, int Hq, int Tq, int Tmax);

/* Fixed-scratch variant of heal_attention_int16.  The paper has no counterpart to this
 * entry point.  It is for callers that cannot allocate device memory at the time they call
 * attention, and so cannot pass a `workspace`: serving loops that forbid any allocation
 * after start-up to keep a fixed memory budget, and plugin hosts that hand an operator only
 * its input and output tensors and no allocator.
 * Arguments and results are those of heal_attention_int16 without workspace and
 * workspace_bytes; the result is the same, bit for bit, as that call's.  The split-context
 * partial results (and, for prefill shapes, the byte planes) go instead to one array of
 * HEAL_ATTN_STATIC_SCRATCH_BYTES bytes in libheal.so's own device memory, which every GPU
 * that loads the library holds until the process exits.  This call allocates and frees
 * nothing.
 *   - The first call on a device looks up that array's device address (a runtime query),
 *     with that device current, and keeps it for the life of the process.  The kept
 *     address does not survive cudaDeviceReset(): after a reset
 *     of a device, do not call this entry point on that device again in the same process.
 *   - All calls share the one array and it keeps the last call's contents.  Nothing in it
 *     needs to start at zero: every partial result a call reads was written earlier in the
 *     same call.  Calls whose kernels overlap on the GPU (other streams, other host
 *     threads) race on the array and corrupt each other's results: serialise them.
 *   - Size limit: the scratch the workspace variant would need,
 *     heal_attention_workspace_bytes_gqa(B, Hq, Hkv, Tq, Tmax), must fit the array.  For
 *     decode shapes ((Hq/Hkv) * Tq <= 8) that is B * Hq * Tq <= 7939; for prefill shapes
 *     6 * B * Hkv * Tmax * 128 + 2 * B * Hq * Tq * 128 + 4 * B * Hkv * Tmax bytes, plus
 *     4 * B * Hkv rounded up to a multiple of 128, must not exceed 8 MiB (one KV head of an
 *     8192-token cache is already 6 MiB).  Larger problems return HEAL_ERR_UNSUPPORTED and
 *     launch nothing.                                                                       */
#define HEAL_ATTN_STATIC_SCRATCH_BYTES (8u << 20)
heal_status_t heal_attention_int16_noalloc(const int16_t* q, const float* q_scale,
                                           const int16_t* k_cache, const float* k_scale,
                                           const int16_t* v_cache, const float* v_scale,
                                           int B, int Hq, int Hkv, int D, int Tq,
                                           const int32_t* kv_len, int Tmax,
                                           float softmax_scale, int causal, float* out,
                                           int64_t* qk_int_out, heal_stream_t stream);

/* K6. FP32 decoder glue of a Llama-style block (the 8B-class decoder shape the paper's
 * evaluation uses; gist.science technical summary, Results).  The pages describe none of
 * these steps; they stay in FP32 so that no 16-bit store happens at a kernel boundary
 * (technical summary, section 1).  All pointers are device pointers; rows are contiguous.
 *   heal_embedding_gather: out[i, :] = table[ids[i], :], table [vocab, H].  An id outside
 *     [0, vocab) gives a zero row and makes heal_get_device_status report
 *     HEAL_ERR_INVALID_ARGUMENT.
 *   heal_rmsnorm: y[i, :] = x[i, :] / sqrt(mean(x[i, :]^2) + eps) * w (w nullable = 1).
 *   heal_rope: in place on x viewed as [n, heads, D] with row stride `row_stride` floats;
 *     rotate-half pairs (d, d + D/2) by the angle of position pos[i]; cos_t and sin_t are
 *     FP32 tables [max_pos, D/2] made by the caller.
 *   heal_swiglu: out[i, j] = silu(gu[i, j]) * gu[i, F + j], gu [n, 2F], out [n, F].
 *   heal_add: x[e] += y[e] for e < n.
 *   heal_argmax: out[r] = index of the largest x[r, :] (lowest index on ties), x [rows, n].
 *   heal_heads_to_rows: y[b, t, h, :] = x[b, h, t, :] for x [B, H, T, D] (an attention
 *     output) and y [B, T, H, D]; D a multiple of 4 up to 1024, x and y 16-byte aligned
 *     and distinct. */
heal_status_t heal_embedding_gather(const float* table, int vocab, int H, const int32_t* ids,
                                    int n, float* out, heal_stream_t stream);
heal_status_t heal_rmsnorm(const float* x, const float* w, int n, int H, float eps, float* y,
                           heal_stream_t stream);
heal_status_t heal_rope(float* x, int n, int heads, int D, int64_t row_stride,
                        const int32_t* pos, const float* cos_t, const float* sin_t,
                        heal_stream_t stream);
heal_status_t heal_swiglu(const float* gate_up, int n, int F, float* out, heal_stream_t stream);
heal_status_t heal_add(float* x, const float* y, int64_t n, heal_stream_t stream);
heal_status_t heal_argmax(const float* x, int rows, int n, int32_t* out, heal_stream_t stream);
heal_status_t heal_heads_to_rows(const float* x, int B, int H, int T, int D, float* y, heal_stream_t stream);

/* Synchronises `stream`, returns HEAL_ERR_TIMEOUT if any kernel of this library gave up
 * on a bounded wait since the last call, HEAL_ERR_INVALID_ARGUMENT if a kernel met an
 * invalid device-side input (an out-of-range token id), HEAL_ERR_CUDA on a CUDA error,
 * else HEAL_OK.  The flags are cleared by the call.                                     */
heal_status_t heal_get_device_status(heal_stream_t stream);

/* Failure-detection check: launches one warp that waits, with the same bounded wait as
 * every kernel of the library, on an mbarrier that nothing arrives on.  After limit_ms
 * (1 .. 10000) the wait gives up, the device status records a timeout and the kernel
 * returns; heal_get_device_status() then reports HEAL_ERR_TIMEOUT and the CUDA context
 * stays usable.  Nothing faults, traps or hangs.                                        */
heal_status_t heal_probe_wait_timeout(int limit_ms, heal_stream_t stream);

/* Static English description of a status code.                                         */
const char* heal_status_string(heal_status_t status);

/* Library version, e.g. "heal-b200 0.1.0 sm_100a".                                     */
const char* heal_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HEAL_H_ */
