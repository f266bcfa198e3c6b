/*
 * sage.h - C ABI of the quantized attention forward for B200 (sm_100a).
 *
 * The method (SageAttention): K is smoothed by subtracting its per-channel mean,
 * Q and K are quantized to INT8 per block, S = Q K^T runs on INT8 tensor cores
 * with int32 accumulation, is dequantized, scaled and passed through an online
 * softmax; P and V are quantized to FP8 e4m3 (V per channel) and P V is
 * accumulated in two levels (per KV block, then into a running FP32 output).
 * Sources: vibecrowd repo page "thu-ml--sageattention", How it works (INT8 QK^T,
 * FP8 PV, two-level accumulation); glossary page "SageAttention(セージアテンション)",
 * 概要 / 主な特徴・仕組み (K smoothing, INT8/FP8 per tensor); heatdrop review
 * "2–5× attention speedups without the accuracy apology tour", Key highlights
 * (GQA, variable sequence lengths); tutorial page "SageAttention终极指南",
 * 基础使用示例 (sageattn(q, k, v, tensor_layout="HND", is_causal=False),
 * shapes (batch, heads, seq_len, head_dim)).
 *
 * Conventions for every entry point
 * ---------------------------------
 * - Pointers are device memory owned by the caller unless marked "host".  The
 *   library allocates no device memory and keeps no state between calls except
 *   the device watchdog word read by sage_poll_device_status(), the scratch
 *   array of sage_quant_qk_noalloc and the copy streams of sage_attn_host.
 * - Work is enqueued on `stream` (a cudaStream_t); calls return once enqueued.
 *   The library works on the calling thread's current CUDA device: every device
 *   pointer and `stream` must belong to it (make that device current first, e.g.
 *   cudaSetDevice).  A stream of another device is rejected with
 *   SAGE_ERR_INVALID_ARGUMENT; pointers cannot be checked and must not be another
 *   device's memory.
 * - Errors: argument problems return SAGE_ERR_INVALID_ARGUMENT or
 *   SAGE_ERR_UNSUPPORTED before anything is enqueued; a failed launch returns
 *   SAGE_ERR_CUDA.  A kernel whose bounded wait runs out records
 *   SAGE_ERR_DEVICE_TIMEOUT in the device watchdog word and exits early (its
 *   outputs are then undefined).  The word is sticky: until
 *   sage_poll_device_status() reads and clears it, every later kernel of the
 *   library on that device sees it set and returns at once without writing its
 *   outputs, while the entry points that enqueued them still return SAGE_OK.
 *   Poll after work whose results matter.
 * - Input tensors q, k, v hold fp16 or bf16 values with a contiguous last
 *   (head_dim) dimension.  Their other three dimensions are given as element
 *   strides {stride_batch, stride_head, stride_token}: HND (B,H,N,d) and
 *   NHD (B,N,H,d) are both expressed this way.  Varlen problems pack all
 *   sequences along the token dimension (T_total, H, d); stride_batch is then
 *   ignored and token t of sequence b is row cu_seqlens_host[b] + t.
 * - Base pointers and the head/token strides must be 16-byte aligned in bytes.
 *
 * Quantized ("padded token space") buffers written by the quant entry points
 * and read by sage_attn_fwd.  Let n_b be the length of sequence b,
 * P_b = ceil(n_b / 128) * 128, off_b = sum_{b' < b} P_b' and T_pad = sum_b P_b
 * (dense problems: n_b = seqlen for every b).  Padding entries are written as 0.
 *   q8      int8  [Hq ][T_pad][d]       token t of seq b, head h at (h*T_pad + off_b + t)*d
 *   q_scale float [Hq ][T_pad/128]      one scale per 128-token block of a sequence
 *                 ([Hq][T_pad], one per token, with SAGE_GRAN_THREAD)
 *   k8      int8  [Hkv][T_pad][d]       smoothed K codes
 *   k_scale float [Hkv][T_pad/64]       one scale per 64-token block of a sequence
 *                 ([Hkv][T_pad/32], one per 32-token block, with SAGE_GRAN_THREAD)
 *   k_mean  float [B  ][Hkv][d]         per-channel mean of K over the sequence
 *   v8      uint8 [Hkv][d][T_pad]       e4m3 codes, transposed (token-contiguous);
 *                 with SAGE_PV_FP16 two bytes per entry: V's own 16-bit values
 *   v_scale float [B  ][Hkv][d]         per-channel V scale (1.0 with SAGE_PV_FP16)
 * Dequantized values: q = q8 * q_scale, k - k_mean = k8 * k_scale,
 * v = e4m3(v8) * v_scale.
 */
#ifndef SAGE_B200_H
#define SAGE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* sage_stream_t; /* the same handle as cudaStream_t */

typedef enum {
  SAGE_OK = 0,
  SAGE_ERR_INVALID_ARGUMENT = 1, /* null pointer, bad size, misaligned, too small workspace */
  SAGE_ERR_UNSUPPORTED = 2,      /* head_dim not 64/128, unknown dtype, device not sm_100 */
  SAGE_ERR_CUDA = 3,             /* a CUDA runtime call or launch failed */
  SAGE_ERR_DEVICE_TIMEOUT = 4,   /* a kernel's bounded wait ran out (see sage_poll_device_status) */
  SAGE_ERR_TOO_LARGE = 5         /* the problem needs more scratch than sage_quant_qk_noalloc holds */
} sage_status_t;

typedef enum { SAGE_FP16 = 0, SAGE_BF16 = 1, SAGE_FP32 = 2 } sage_dtype_t;

/* Granularity of the INT8 scales of Q and K.
 * SAGE_GRAN_BLOCK (0, the method as stated): one scale per 128-token Q block and per
 *   64-token K block of a sequence.
 * SAGE_GRAN_THREAD (1): finer scales, the reading of the heatdrop review's
 *   "per-thread quantization" (The interesting bit) for this kernel, where one thread
 *   owns one query row and takes keys 32 at a time: one scale per Q token and one per
 *   32-token K block.  Same codes otherwise; the attention kernel folds the scales
 *   into the same per-row, per-32-key factors. */
typedef enum { SAGE_GRAN_BLOCK = 0, SAGE_GRAN_THREAD = 1 } sage_granularity_t;

/* Format of the P V product (vibecrowd page "thu-ml--sageattention", How it works:
 * FP16/FP8 for PV).
 * SAGE_PV_FP8 (0, the method as stated): P and V in FP8 e4m3, V with per-channel scales.
 * SAGE_PV_FP16 (1): the accuracy fallback.  V keeps its 16-bit input values (fp16 or
 *   bf16, no V quantization) and P~ (<= 1) is rounded to that same type; the PV
 *   MMA runs in that type with FP32 accumulation, two levels as with FP8. */
typedef enum { SAGE_PV_FP8 = 0, SAGE_PV_FP16 = 1 } sage_pv_t;

/* Problem description shared by all entry points. */
typedef struct {
  int batch;              /* B: dense batch size, or number of packed sequences (<= 1024) */
  int heads_q;            /* Hq */
  int heads_kv;           /* Hkv; Hq % Hkv == 0, query head h reads KV head h / (Hq/Hkv) */
  int seqlen;             /* dense: tokens per sequence (>= 1); varlen: ignored */
  int head_dim;           /* d: 64 or 128 */
  sage_dtype_t dtype;     /* dtype of q, k, v: SAGE_FP16 or SAGE_BF16 */
  const int32_t* cu_seqlens_host; /* host, NULL for dense; else [batch+1] prefix sums of the
                                     packed sequence lengths, cu[0] = 0, non-decreasing */
  sage_granularity_t granularity; /* INT8 scale granularity of Q and K (zero: per block) */
  sage_pv_t pv;           /* format of the P V product (zero: FP8 e4m3) */
} sage_problem_t;

/* Byte sizes of the quantized buffers and of the quantization workspaces. */
typedef struct {
  size_t q8, q_scale, k8, k_scale, k_mean, v8, v_scale;
  size_t workspace_qk;    /* scratch needed by sage_quant_qk */
  size_t workspace_v;     /* scratch needed by sage_quant_v */
  size_t t_pad;           /* T_pad, the padded token count */
  size_t workspace_qkv;   /* scratch needed by sage_quant_qkv */
} sage_sizes_t;

/* Fill *sizes (host) for problem *p (host).  Pure host computation. */
sage_status_t sage_buffer_sizes(const sage_problem_t* p, sage_sizes_t* sizes);

/*
 * sage_quant_qk - K smoothing and per-block INT8 quantization of Q and K.
 * (glossary page "SageAttention(セージアテンション)", 主な特徴・仕組み: K smoothing;
 *  vibecrowd page, How it works: INT8 quantization for QK^T.)
 *   mu[c]  = fp32(sum_t k[t,c] in fp64 / n_b)              per (sequence, kv head)
 *   k_s    = fp32(k - mu)
 *   per block (Q: 128 tokens x d, K: 64 tokens x d of k_s; with SAGE_GRAN_THREAD
 *   Q: 1 token x d, K: 32 tokens x d):
 *     a = max|x|;  s = fp32(a/127);  x8 = clamp(rint_even(fp32(x * fp32(127/a))), -127, 127)
 *     (a == 0: s = 0, codes 0)
 * Writes q8, q_scale, k8, k_scale, k_mean (layouts above).  `workspace` must
 * hold sizes.workspace_qk bytes (fp64 per-block channel sums); its contents on
 * entry do not matter.  Launches three kernels on `stream`.
 */
sage_status_t sage_quant_qk(const sage_problem_t* p,
                            const void* q, const int64_t q_strides[3],
                            const void* k, const int64_t k_strides[3],
                            int8_t* q8, float* q_scale, int8_t* k8, float* k_scale,
                            float* k_mean, void* workspace, size_t workspace_bytes,
                            sage_stream_t stream);

/*
 * sage_quant_qk_noalloc - sage_quant_qk without a caller workspace.
 * The pages describe no counterpart: this is a deployment convenience.  It is for
 * callers that cannot allocate device memory when they quantize (a framework hook
 * whose allocator is locked, a plugin that may only use the tensors it is given, a
 * pipeline whose buffers are all reserved up front).  Arguments, outputs and
 * results are those of sage_quant_qk; the fp64 column-sum scratch lives instead in
 * a library-owned device array of SAGE_NOALLOC_SCRATCH_BYTES (8 MiB) on every GPU
 * that loads the library, kept until the process exits.
 * - Returns SAGE_ERR_TOO_LARGE, before enqueuing anything, when the problem needs
 *   more scratch than that (sizes.workspace_qk > SAGE_NOALLOC_SCRATCH_BYTES).
 * - The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call before
 *   any stream capture.  It allocates nothing (no cudaMalloc / cudaFree).  The
 *   address is kept for the life of the process: after cudaDeviceReset() on a
 *   device, this entry point must not be called on that device again.
 * - All calls share the array, which keeps the last call's contents (nothing in it
 *   needs clearing); calls that overlap on the GPU, from any stream or thread, race.
 */
#define SAGE_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
sage_status_t sage_quant_qk_noalloc(const sage_problem_t* p,
                                    const void* q, const int64_t q_strides[3],
                                    const void* k, const int64_t k_strides[3],
                                    int8_t* q8, float* q_scale, int8_t* k8, float* k_scale,
                                    float* k_mean, sage_stream_t stream);

/*
 * sage_quant_v - per-channel FP8 e4m3 quantization of V, written transposed.
 * (vibecrowd page, How it works: FP8 for PV; glossary page, 概要: P and V in FP8.)
 *   vmax[c] = max_t |v[t,c]| per (sequence, kv head);  sv = fp32(vmax/448)
 *   v8 = e4m3_rne_satfinite(fp32(v * fp32(448/vmax)))   (vmax == 0: sv = 0, codes 0)
 * Writes v8 and v_scale.  `workspace` must hold sizes.workspace_v bytes.
 * Launches three kernels on `stream`.
 * With p->pv == SAGE_PV_FP16: copies V's 16-bit values into the same transposed
 * layout (two bytes per entry) and sets v_scale to 1; no workspace is needed
 * (sizes.workspace_v is 0 and `workspace` may be NULL).  Two launches.
 */
sage_status_t sage_quant_v(const sage_problem_t* p, const void* v, const int64_t v_strides[3],
                           uint8_t* v8, float* v_scale, void* workspace, size_t workspace_bytes,
                           sage_stream_t stream);

/*
 * sage_quant_qkv - sage_quant_qk and sage_quant_v in one launch.
 * (Same sources and arithmetic as those two entry points; the tutorial page
 * "SageAttention终极指南", 源码结构解析, places quantization in its own module.)
 * Writes q8, q_scale, k8, k_scale, k_mean, v8 and v_scale exactly as the two separate
 * calls would: every code, scale and mean is bit-identical.  One cooperative,
 * persistent launch (one CTA per SM): Q is quantized while the K sums and V maxima
 * are gathered, a grid-wide barrier precedes the means and V scales, another precedes
 * the K and V codes.  Tiles move by TMA, so besides the rules for every entry point
 * the smallest of the three element strides of each input must be at least
 * head_dim (rows do not overlap); SAGE_ERR_INVALID_ARGUMENT otherwise.
 * `workspace` must hold sizes.workspace_qkv bytes; its contents on entry do not
 * matter.  SAGE_ERR_UNSUPPORTED if the device cannot launch cooperative kernels.
 */
sage_status_t sage_quant_qkv(const sage_problem_t* p,
                             const void* q, const int64_t q_strides[3],
                             const void* k, const int64_t k_strides[3],
                             const void* v, const int64_t v_strides[3],
                             int8_t* q8, float* q_scale, int8_t* k8, float* k_scale,
                             float* k_mean, void* v8, float* v_scale, void* workspace,
                             size_t workspace_bytes, sage_stream_t stream);

/*
 * sage_attn_fwd - the attention kernel (tcgen05 INT8 QK^T and FP8 PV, TMEM accumulators).
 * (vibecrowd page, How it works; heatdrop review, The interesting bit and Key highlights.)
 * For each query row i of sequence b, head h (KV head h/(Hq/Hkv)), over KV blocks of
 * 128 keys in order:
 *   x_j  = S_ij * q_scale_i * k_scale_j * sm_scale (S_ij exact int32 from INT8 MMAs; the
 *          scales of row i's Q block and key j's K block at the problem's granularity)
 *   causal: x_j = -inf for j > i
 *   m'   = max(m, max_j x_j);   P~_j = exp(x_j - m');   l = l e^{m-m'} + sum_j P~_j
 *   P8   = e4m3(448 P~);  O = O e^{m-m'} + PV_blk,  PV_blk = P8 V8
 *   out  = O * v_scale / (448 l)           lse = m + ln(l)   (natural log)
 *   (SAGE_PV_FP16: P = P~ rounded to the input's 16-bit type, PV_blk = P V16,
 *    out = O / l.)
 * The logits x and the running max m are fp64.  O is an FP32 accumulator in TMEM:
 * each block it is rescaled by e^{m-m'} in FP32 and the tensor core adds the block's
 * P8 V8 onto it in FP32.  P~ is formed in fp32 with the hardware base-2 exponential
 * from fp64-formed constants; every e4m3 code whose fp32 P~ lies within 32 ulps of a
 * rounding midpoint is decided again in fp64, so the codes are those of the fp64
 * definition.
 * sm_scale <= 0 selects 1/sqrt(head_dim).  is_causal != 0 applies the mask above.
 * out: written in out_dtype (SAGE_FP16, SAGE_BF16 or SAGE_FP32) with element
 * strides out_strides {batch, head, token}, last dimension contiguous, the
 * same packing rules as the inputs.  lse: NULL or float [Hq][T_pad], natural-log
 * sum of exponentials of the smoothed, dequantized logits (padding rows unwritten).
 * One kernel launch on `stream`.
 */
sage_status_t sage_attn_fwd(const sage_problem_t* p,
                            const int8_t* q8, const float* q_scale,
                            const int8_t* k8, const float* k_scale,
                            const uint8_t* v8, const float* v_scale,
                            float sm_scale, int is_causal,
                            void* out, sage_dtype_t out_dtype, const int64_t out_strides[3],
                            float* lse, sage_stream_t stream);

/*
 * sage_debug_qk_int32 - test hook: the exact int32 scores of one (sequence, query head).
 * s_out: int32 [P_b][P_b] row-major, S[i][j] = sum_c q8[i][c] k8[j][c] over the padded
 * rows of sequence `seq`, query head `head_q` and its KV head.  Uses the same
 * TMA + tcgen05.mma kind::i8 + TMEM path as sage_attn_fwd.
 */
sage_status_t sage_debug_qk_int32(const sage_problem_t* p, const int8_t* q8, const int8_t* k8,
                                  int seq, int head_q, int32_t* s_out, sage_stream_t stream);

/*
 * sage_attn_host - the whole path (sage_quant_qk, sage_quant_v, sage_attn_fwd) on
 * HOST buffers, pipelined over chunks of heads.  The pages describe no counterpart:
 * it is the host-side driver of the calls above for inputs that live in host memory.
 * Every head's quantization (mean, blocks, scales) and attention are independent of
 * the other heads, so the outputs are bit-identical to the device path.
 *   Dense problems only (cu_seqlens_host == NULL).  tensor_layout 0: q, k, v and out
 *   are contiguous HND arrays (B, H, N, d); 1: contiguous NHD arrays (B, N, H, d).
 *   q_host, k_host, v_host (dtype p->dtype) and out_host (out_dtype) are host memory;
 *   page-locked memory lets the copies overlap the kernels (pageable memory works
 *   but serializes).  Base pointers must be 16-byte aligned.
 *   The KV heads of each batch entry are taken kv_heads_per_chunk at a time (with
 *   their query heads); <= 0 picks a size giving at least 8 chunks.  For chunk c:
 *   its inputs are copied in on an internal stream, its three kernel calls run on
 *   `stream`, and its output is copied out on a second internal stream, so chunk c's
 *   copy-in overlaps chunk c-1's kernels and chunk c-2's copy-out (two workspace
 *   slots, one cudaMemcpyAsync or cudaMemcpy2DAsync per tensor and chunk).
 *   `workspace` (device) must hold sage_host_workspace_bytes(p, kv_heads_per_chunk,
 *   out_dtype) bytes.  The first copy waits for the work already on `stream`, and
 *   `stream` waits for the last copy-out: synchronize `stream` before reading
 *   out_host.  Calls on one device are serialized while they enqueue; the internal
 *   streams and events are created on first use per device and kept.
 * Errors as for the other entry points; SAGE_ERR_INVALID_ARGUMENT also for varlen
 * problems, a bad layout code or a too-small workspace.
 */
size_t sage_host_workspace_bytes(const sage_problem_t* p, int kv_heads_per_chunk,
                                 sage_dtype_t out_dtype);
sage_status_t sage_attn_host(const sage_problem_t* p, int tensor_layout,
                             const void* q_host, const void* k_host, const void* v_host,
                             void* out_host, sage_dtype_t out_dtype, float sm_scale,
                             int is_causal, int kv_heads_per_chunk, void* workspace,
                             size_t workspace_bytes, sage_stream_t stream);

/*
 * sage_debug_watchdog_selftest - test hook for the failure path of the bounded waits.
 * Launches one 32-thread CTA whose first thread waits on an mbarrier phase that
 * nothing completes, checking the clock as the kernels' waits do, and gives up after
 * limit_us microseconds (1 .. 1000000): it records SAGE_ERR_DEVICE_TIMEOUT in the
 * device watchdog word and returns.  No fault and no hang: the next
 * sage_poll_device_status() reports the timeout and clears the word, and the
 * context stays usable.  SAGE_ERR_INVALID_ARGUMENT for a limit out of range.
 */
sage_status_t sage_debug_watchdog_selftest(unsigned int limit_us, sage_stream_t stream);

/*
 * Synchronize `stream`, then read and clear the device watchdog word of the
 * current device.  Returns SAGE_OK, SAGE_ERR_DEVICE_TIMEOUT or SAGE_ERR_CUDA.
 */
sage_status_t sage_poll_device_status(sage_stream_t stream);

/* Static, human-readable name of a status code. */
const char* sage_status_string(sage_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_B200_H */
