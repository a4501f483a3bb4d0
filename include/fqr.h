/*
 * fqr.h -- C ABI of libfqr.so: the fused pre-attention preparation path for
 * NVIDIA B200 (sm_100a).
 *
 * One call = one kernel launch on the caller's stream.  The library allocates
 * nothing, synchronises nothing, keeps no per-call state, and may be called
 * from several host threads at once.  Every pointer in the parameter structs
 * is a DEVICE pointer owned by the caller (unless stated otherwise); the
 * library only reads the inputs and writes the outputs named below.
 *
 * Types: BF16 tensors are passed as uint16_t (their bit patterns), FP8 E4M3
 * tensors as uint8_t codes.  "elements" means elements of the tensor's own
 * type.  `stream` is a cudaStream_t (NULL = the legacy default stream).
 *
 * Return codes (host side, decided before anything is launched unless noted):
 *   FQR_OK       the kernel was enqueued (or there was nothing to do).
 *   FQR_EINVAL   an argument that the host can check is invalid (a required
 *                pointer is NULL or misaligned, a size is out of range, a
 *                policy value is unknown, upper_max is not finite in (0, 448],
 *                ...).  Nothing was launched.
 *   FQR_ENOTSUP  the arguments are valid but this build does not implement
 *                the combination (for example NeoX RoPE with rot_dim != 128).
 *                Nothing was launched.
 *   FQR_ECUDA    the CUDA runtime refused the launch.
 * Malformed batch METADATA (q_indptr, seq_lens, positions) is not a host
 * error: it is detected on the device, see `flags` below.
 */
#ifndef FQR_H
#define FQR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FQR_OK 0
#define FQR_EINVAL 1
#define FQR_ENOTSUP 2
#define FQR_ECUDA 3

#define FQR_HEAD_DIM 128

/* fqr_append_params.schedule: how rows are spread over the GPU (the results
 * are identical).  AUTO picks LATENCY while every warp task of it (one per
 * 4 heads of a row, plus one per request) has a resident warp of its own --
 * small batches such as decode -- and STREAMING beyond that (large decode
 * batches, prefill); decode-like batches with large last-page tails (48 KiB
 * or more expected per row) keep LATENCY up to 8 passes of tasks. */
#define FQR_SCHEDULE_AUTO 0
#define FQR_SCHEDULE_LATENCY 1
#define FQR_SCHEDULE_STREAMING 2
/* Largest batch (number of requests) one call accepts; per-request metadata
 * is staged in shared memory by every thread block. */
#define FQR_MAX_BATCH 16384

/* fqr_append_params.norm_style: how the bf16 norm weight w scales the
 * normalised value.  RMS: y = x_hat * w.  GEMMA: y = x_hat * (1 + w), with
 * 1 + w formed in fp32 (Gemma-style QK norm, TensorRT-LLM PR #16024). */
#define FQR_NORM_RMS 0
#define FQR_NORM_GEMMA 1

/*
 * fqr_append_paged -- per-head Q/K RMSNorm, RoPE, optional FP8 E4M3
 * quantisation, and the paged K/V append with last-page tail zeroing.
 *
 * Defined by the FlashInfer PR #5956 page (fused QK RMSNorm + NeoX RoPE + FP8
 * E4M3 quantize + NHD paged-KV append), section "Contract"; the norm follows
 * the TensorRT-LLM PR #16024 review excerpt (rsqrt(sum_sq / head_size + eps)),
 * the RoPE the SGLang PR #43425 "Modifications" (fp32 cos/sin cache, NeoX).
 *
 * For every request b, with n_b = q_indptr[b+1] - q_indptr[b] new tokens and
 * L_b = seq_lens[b] the length AFTER the append, packed row r in
 * [q_indptr[b], q_indptr[b+1]) sits at sequence position
 *     p_r = r + L_b - q_indptr[b+1]
 * and goes to slot (page_table[b, p_r / P], p_r % P) of both caches.  RoPE
 * uses positions[r] when `positions` is given, else p_r.  In fp32:
 *     y = x * (1/sqrt(sum(x^2)/128 + eps)) * w         (Q heads with q_norm_w,
 *                                                       K heads with k_norm_w;
 *                                       w -> 1 + w for norm_style GEMMA)
 *            the mean square sum(x^2)/128 is the fp32 rounding of the exact
 *            mean of the squares (no summation order enters); + eps, the
 *            square root and the reciprocal are each correctly rounded
 *     NeoX:  (y_i, y_{i+64})  -> (y_i c_i - y_{i+64} s_i, y_{i+64} c_i + y_i s_i)
 *     GPT-J: (y_2i, y_2i+1)   -> (y_2i c_i - y_2i+1 s_i, y_2i+1 c_i + y_2i s_i)
 *            with c_i = cos_sin[pos, i], s_i = cos_sin[pos, rot_dim/2 + i];
 *            dims >= rot_dim pass through.
 * Outputs by quant_policy:
 *     0: out_q = bf16(q); K = bf16(k); V = the input bits (BF16 caches)
 *     1: s = max(max_i |q_i|, 1e-6) / upper_max for each (row, Q head),
 *        out_q = e4m3(q / s); K = e4m3(k / *k_scale);
 *        V = e4m3(v / *v_scale)                            (FP8 caches)
 *        s is stored in q_scale, by layout:
 *          max_seqlen == 0 (decode):  q_scale[r, h]         fp32 [T, Hq]
 *          max_seqlen  > 0 (prefill): q_scale[b, h, r - q_indptr[b]]
 *                              fp32 [B, Hq, round_up(max_seqlen, 128)];
 *          entries past a request's rows are not written.
 *     2: out_q = e4m3(q * *q_scale_inv); K, V as in policy 1
 * (e4m3 = round to nearest even, saturating at +-448; bf16 = RNE).
 * Then, for every request with L_b > 0, rows [(L_b-1) % P + 1, P) of page
 * page_table[b, (L_b-1) / P] are zeroed in both caches.
 * With out_k / out_v given, the K and V payloads go to row r of those
 * caller-owned buffers instead: the paged caches and the page table are not
 * used (they may be NULL), no slot is written and no tail is zeroed (the
 * FlashInfer PR #5956 review: redirected K/V writes leave the caches alone).
 *
 * flags[b] = 0 after a valid call (requests without new tokens included).
 * flags[b] = -2 (all flags) only if the kernel gave up waiting for its own
 * shared-memory copies (a bounded wait that should never expire).
 * If the metadata is malformed -- q_indptr[0] != 0, q_indptr[B] != T, any
 * q_indptr decrease, L_b < n_b, L_b > max_pages * P (paged caches only), or
 * (derived positions) L_b > cos_sin_rows, or (explicit positions) any
 * position outside [0, cos_sin_rows), or (policy 1 with max_seqlen > 0)
 * n_b > max_seqlen -- then EVERY flag is set to -1 and nothing else is
 * written: no out_q, q_scale, out_k, out_v or cache byte.  The check runs on the device
 * inside the same launch (no host sync), so the call can be captured in a
 * CUDA graph and replayed.  Read the flags after the stream completes.
 *
 * Caller obligations: page ids in the used part of page_table lie in
 * [0, num_pages); a page belongs to one request; no output overlaps an input
 * or another output.
 */
typedef struct fqr_append_params {
  /* packed input rows: bf16 [T, qkv_row_stride]; each row holds Hq Q heads,
   * then Hkv K heads, then Hkv V heads, 128 elements each.  16-byte aligned;
   * qkv_row_stride >= (Hq + 2*Hkv) * 128 and a multiple of 8 (row padding
   * allowed).  Read-only. */
  const uint16_t* qkv;
  int64_t qkv_row_stride;
  int32_t T;             /* packed rows (new tokens), >= 0                    */
  int32_t B;             /* requests, 0 <= B <= FQR_MAX_BATCH                 */
  int32_t Hq, Hkv;       /* Hq % Hkv == 0                                     */
  int32_t head_dim;      /* must be 128                                       */
  /* RMSNorm weights, bf16 [128], 16-byte aligned; NULL = no norm for that
   * tensor.  eps >= 0, finite. */
  const uint16_t* q_norm_w;
  const uint16_t* k_norm_w;
  float eps;
  /* fp32 [cos_sin_rows, rot_dim] = [cos(p f_i) | sin(p f_i)], 16-byte
   * aligned.  rope_style 0 = NeoX (rot_dim must be 128), 1 = GPT-J (any even
   * rot_dim in [2, 128]). */
  const float* cos_sin_cache;
  int32_t cos_sin_rows, rot_dim, rope_style;
  /* int64 [T] RoPE positions, or NULL to derive them from q_indptr/seq_lens */
  const int64_t* positions;
  const int32_t* q_indptr;    /* int32 [B + 1]                                */
  const int32_t* seq_lens;    /* int32 [B], lengths after the append          */
  const int32_t* page_table;  /* int32 [B, max_pages], row-major              */
  int32_t max_pages;
  /* NHD caches [num_pages, page_size, Hkv, 128]: bf16 for policy 0, e4m3 for
   * policies 1/2; 16-byte aligned; pages k_page_stride / v_page_stride
   * elements apart (>= page_size * Hkv * 128, 16-byte multiples). */
  void* k_cache;
  void* v_cache;
  int32_t num_pages, page_size;  /* 2 * B * (page_size - 1) < 2^31              */
  int64_t k_page_stride, v_page_stride;
  int32_t quant_policy;       /* 0, 1 or 2, see above                         */
  const float* q_scale_inv;   /* device fp32 scalar (policy 2)                */
  const float* k_scale;       /* device fp32 scalars (policies 1, 2)          */
  const float* v_scale;
  float upper_max;            /* policy 1: finite, in (0, 448]                */
  /* outputs: out_q [T, Hq, 128] (bf16 for policy 0, e4m3 otherwise),
   * 16-byte aligned; q_scale fp32 [T, Hq] (policy 1 only); flags int32 [B] */
  void* out_q;
  float* q_scale;
  int32_t* flags;
  int32_t schedule;           /* FQR_SCHEDULE_*; 0 = automatic                */
  /* policy 1: 0 = decode q_scale layout [T, Hq]; > 0 = prefill layout
   * [B, Hq, round_up(max_seqlen, 128)] and the n_b <= max_seqlen check.
   * Ignored by policies 0 and 2.  >= 0;
   * B * Hq * round_up(max_seqlen, 128) < 2^31. */
  int32_t max_seqlen;
  int32_t norm_style;         /* FQR_NORM_RMS or FQR_NORM_GEMMA               */
  /* optional caller-owned K / V outputs [T, Hkv, 128] (the cache element
   * type), 16-byte aligned, both or neither; NULL = the paged caches */
  void* out_k;
  void* out_v;
} fqr_append_params;

int fqr_append_paged(const fqr_append_params* p, void* stream);

/*
 * fqr_append_plan_query -- the launch fqr_append_paged would make for *p on
 * the current device, without making it: which schedule, the grid and block
 * shape, and the variants of the latency schedule.  The FlashInfer PR #5956
 * wrapper exposes its launch plan the same way ("launch_plan"); this is its
 * counterpart, for callers that size or log their launches and for tests.
 *
 *   schedule       FQR_SCHEDULE_LATENCY or FQR_SCHEDULE_STREAMING; 0 when the
 *                  call would launch nothing (T = B = 0).
 *   grid           blocks of the launch.
 *   block_threads  threads per block.
 *   tasks          latency: warp tasks (a quad of heads of a row, or a
 *                  request's tail); streaming: units (a packed row, or a
 *                  chunk of one).
 *   warp_check     latency: every warp validates the batch itself (no block
 *                  prologue); streaming: 0.
 *   bulk_tails     latency: tails go out as bulk copies (warps hold several
 *                  tasks).
 *   request_tails  latency: request tasks zero whole tails (small tails, one
 *                  task per warp).
 *
 * Checks *p exactly as fqr_append_paged does and returns the same codes;
 * `plan` must not be NULL (FQR_EINVAL).  Queries the device (SM count,
 * occupancy; cached per device after the first call); launches, allocates
 * and synchronises nothing.
 */
typedef struct fqr_append_plan {
  int32_t schedule;
  int32_t grid;
  int32_t block_threads;
  int32_t tasks;
  int32_t warp_check;
  int32_t bulk_tails;
  int32_t request_tails;
} fqr_append_plan;
int fqr_append_plan_query(const fqr_append_params* p, fqr_append_plan* plan);

/*
 * fqr_pipeline_* -- fqr_append_paged on batches held in pinned host memory,
 * pipelined.  A pipeline has `depth` slots; slot j owns a device input buffer
 * dev_in[j] (in_bytes) and a device result buffer dev_out[j] (out_bytes),
 * allocated by the caller, and a parameter block params[j] whose device
 * pointers point into them (qkv and metadata into dev_in[j]; out_q, flags,
 * q_scale into dev_out[j]) or at resident device data (caches, cos/sin,
 * weights, scales).  Each submit, for the next slot in turn, enqueues on
 * three streams the pipeline owns:
 *   copy-in:  host_in (in_bytes, pinned) -> dev_in[j], once slot j's
 *             previous kernel has run;
 *   compute:  fqr_append_paged(params[j]), after that copy and once slot j's
 *             previous results have been copied out;
 *   copy-out: dev_out[j] -> host_out (out_bytes, pinned).
 * So the copy-in of one batch, the kernel of the one before and the copy-out
 * of the one before that overlap.  One host->device and one device->host copy
 * per batch (cudaMemcpyAsync each); no device memory is allocated.
 *
 * create: checks every params[j] as fqr_append_paged does (T = B = 0 is
 *   rejected), creates three non-blocking streams and 3*depth events on the
 *   current device; *out receives the handle.  FQR_EINVAL / FQR_ENOTSUP /
 *   FQR_ECUDA, with *out = NULL, on failure.
 * submit: asynchronous; host buffers must stay valid until the batch is
 *   done (fqr_pipeline_sync, or a stream that fqr_pipeline_join made wait).
 * fork: the pipeline's streams wait for the work enqueued so far on `stream`.
 * join: `stream` waits for every batch submitted so far.
 * sync: blocks the host until every submitted batch is done.
 * destroy: syncs, then releases the streams and events.
 */
#define FQR_PIPELINE_MAX_DEPTH 8
typedef struct fqr_pipeline fqr_pipeline;
int fqr_pipeline_create(int depth, const fqr_append_params* params, void* const* dev_in,
                        size_t in_bytes, void* const* dev_out, size_t out_bytes,
                        fqr_pipeline** out);
int fqr_pipeline_submit(fqr_pipeline* p, const void* host_in, void* host_out);
int fqr_pipeline_fork(fqr_pipeline* p, void* stream);
int fqr_pipeline_join(fqr_pipeline* p, void* stream);
int fqr_pipeline_sync(fqr_pipeline* p);
int fqr_pipeline_destroy(fqr_pipeline* p);

/*
 * fqr_concat_mla_cache -- MLA variant: rotate the rope part of Q in place and
 * write latent rows [kv_c | rope(k_pe)] into a paged latent cache.
 *
 * Defined by the vLLM issue #24678 page (concat_and_cache_mla fused with
 * RoPE; DeepSeek R1 "RoPE/NoPE interleaved", 64 qk_rope dims) with the slot,
 * position and validation rules of fqr_append_paged.
 *
 * For packed row r of request b at position p_r (as above):
 *   q[r, h, nope_dim : nope_dim + rope_dim] <- bf16(rope(q[...], pos)) for
 *   every head h (in place; dims [0, nope_dim) are not touched);
 *   latent[block_table[b, p_r / block_size], p_r % block_size, :] =
 *     [kv_c[r, 0:rank] | rope(k_pe[r, 0:rope_dim])] encoded as
 *     e4m3(x / *kv_scale) (cache_fp8 = 1) or bf16 (cache_fp8 = 0: kv_c bits
 *     copied, rope part RNE).  k_pe is read-only.  No tail is zeroed.
 * flags as for fqr_append_paged (block_table/max_blocks/block_size play the
 * page table's role); when flagged nothing else is written.
 *
 * Q quantisation (q_quant != 0; vLLM issue #24678: "static per-tensor,
 * dynamic per-token, and dynamic per-group" Q scales): q is then read-only,
 * and with v = [q[r, h, 0:nope] | rope(q[r, h, nope:nope+rope])] in fp32,
 * q_out[r, h, :] (e4m3 [T, Hq, nope + rope], contiguous) receives
 *   FQR_MLA_Q_STATIC:   e4m3(v * *q_scale_inv)
 *   FQR_MLA_Q_TOKEN:    e4m3(v / s), s = max(max |v| over all heads of row r,
 *                       1e-6) / upper_max, q_scale[r] = s         (fp32 [T])
 *   FQR_MLA_Q_HEAD:     the same with the max over head h alone,
 *                       q_scale[r * Hq + h] = s                   (fp32 [T, Hq])
 *   FQR_MLA_Q_GROUP:    the same with the max over each group of q_group
 *                       consecutive values of v of one head (block
 *                       quantisation; the last group of a head is shorter
 *                       when q_group does not divide nope + rope; q_group
 *                       >= nope + rope gives one group per head),
 *                       q_scale[(r * Hq + h) * NG + k] = s of group k,
 *                       NG = ceil((nope + rope) / q_group)  (fp32 [T, Hq, NG])
 *
 * Constraints: rope_dim == 64; nope_dim, q_token_stride, q_head_stride
 * multiples of 4 (of 8, and nope_dim <= 256, with Q quantisation); q_group
 * (FQR_MLA_Q_GROUP) a multiple of 8, at least 8;
 * kv_lora_rank, kv_c_stride
 * multiples of 8; k_pe_stride a multiple of 4; q, kv_c, k_pe, latent_cache,
 * q_out 16-byte aligned.
 */
#define FQR_MLA_Q_NONE 0
#define FQR_MLA_Q_STATIC 1
#define FQR_MLA_Q_TOKEN 2
#define FQR_MLA_Q_HEAD 3
#define FQR_MLA_Q_GROUP 4
typedef struct fqr_mla_params {
  uint16_t* q;                 /* bf16, element (r, h, d) at
                                  r*q_token_stride + h*q_head_stride + d     */
  int32_t T, B, Hq, nope_dim, rope_dim;
  int64_t q_token_stride, q_head_stride;
  const uint16_t* kv_c;        /* bf16 [T, kv_c_stride], first rank used     */
  int32_t kv_lora_rank;
  int64_t kv_c_stride;
  const uint16_t* k_pe;        /* bf16 [T, k_pe_stride], first rope_dim used */
  int64_t k_pe_stride;
  const float* cos_sin_cache;  /* fp32 [cos_sin_rows, rope_dim]              */
  int32_t cos_sin_rows, rope_style;   /* 0 NeoX, 1 GPT-J (interleaved)      */
  const int64_t* positions;    /* int64 [T] or NULL                          */
  const int32_t* q_indptr;     /* int32 [B + 1]                              */
  const int32_t* seq_lens;     /* int32 [B]                                  */
  const int32_t* block_table;  /* int32 [B, max_blocks]                      */
  int32_t max_blocks;
  void* latent_cache;          /* [num_blocks, block_size, rank + rope_dim]  */
  int32_t num_blocks, block_size;
  int32_t cache_fp8;           /* 1 e4m3, 0 bf16                             */
  const float* kv_scale;       /* device fp32 scalar (cache_fp8 = 1)         */
  int32_t* flags;              /* int32 [B]                                  */
  int32_t q_quant;             /* FQR_MLA_Q_*                                */
  const float* q_scale_inv;    /* device fp32 scalar (FQR_MLA_Q_STATIC)      */
  float upper_max;             /* dynamic modes: finite, in (0, 448]         */
  void* q_out;                 /* e4m3 [T, Hq, nope + rope] (q_quant != 0)   */
  float* q_scale;              /* fp32 [T], [T, Hq] or [T, Hq, NG] (dynamic) */
  int32_t q_group;             /* values per group (FQR_MLA_Q_GROUP)         */
} fqr_mla_params;

int fqr_concat_mla_cache(const fqr_mla_params* p, void* stream);

/* Static, NUL-terminated description of a return code. */
const char* fqr_strerror(int code);

#ifdef __cplusplus
}
#endif
#endif /* FQR_H */
