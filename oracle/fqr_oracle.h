/*
 * fqr_oracle.h -- plain CPU oracle of the fused pre-attention preparation path
 * (per-head Q/K RMSNorm, RoPE from a cos/sin cache, optional FP8 E4M3
 * quantisation, paged K/V append with last-page tail zeroing, and the MLA
 * latent concat).
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The
 * product path (the CUDA library) never includes, links or calls it, and this
 * file shares no header, helper or table with it.
 *
 * Precision: fp32 for every arithmetic step, one rounding at each store, as
 * the FlashInfer PR #5956 page states for its own reference ("Contract" and
 * the test list under "What changes": fp32 reference, per-head RMSNorm with
 * eps 1e-6, NeoX RoPE, max(|q|, 1e-6) / upper_max, x / scale payloads).
 * Encoders (BF16, E4M3) are written from the format definitions and compute
 * in exact double arithmetic, which is the definition of round-to-nearest.
 *
 * Storage conventions: BF16 values travel as their uint16_t bit patterns, FP8
 * E4M3 values as uint8_t codes.  head_dim is 128 for the paged append.
 */
#ifndef FQR_ORACLE_H
#define FQR_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FQRO_HEAD_DIM 128

/* ---- format encoders / decoders (from the format definitions) ---------- */
float fqro_bf16_to_f32(uint16_t bits);
uint16_t fqro_f32_to_bf16_rne(float x);
uint8_t fqro_f32_to_e4m3_rn_satfinite(float x);
void fqro_f32_to_e4m3_array(const float* x, uint8_t* out, int64_t n);
void fqro_f32_to_bf16_array(const float* x, uint16_t* out, int64_t n);

/* ---- per-head steps ----------------------------------------------------- */
/* y = x * (1 / sqrt(sum(x^2)/n + eps)) * w   (w == NULL -> w = 1); the mean
 * square is the fp32 rounding of the binary64 mean of the squares */
void fqro_rmsnorm(const float* x, const float* w, int n, float eps, float* y);
/* NeoX rotate-half on y[0, rot): pairs (i, i + rot/2) with cs = [cos | sin] */
void fqro_rope_neox(float* y, const float* cs_row, int rot);
/* GPT-J interleaved on y[0, rot): pairs (2i, 2i + 1) with cs = [cos | sin] */
void fqro_rope_gptj(float* y, const float* cs_row, int rot);

/* ---- metadata validation ------------------------------------------------ */
/* Returns 1 if the batch metadata is malformed (any request), else 0.
 * paged = 0 skips the page-overrun check (no page is addressed);
 * max_seqlen > 0 adds n_b <= max_seqlen. */
int fqro_validate(const int32_t* q_indptr, const int32_t* seq_lens, int32_t B,
                  int32_t T, int32_t max_pages, int32_t page_size,
                  int32_t cos_sin_rows, const int64_t* positions,
                  int32_t max_seqlen, int32_t paged);

/* ---- the paged append --------------------------------------------------- */
typedef struct {
  /* inputs (host memory) */
  const uint16_t* qkv;        /* bf16 [T, row_stride], heads Q | K | V       */
  int64_t row_stride;         /* elements per packed row                     */
  int32_t T, B, Hq, Hkv;
  const uint16_t* q_norm_w;   /* bf16 [128] or NULL (no Q norm)              */
  const uint16_t* k_norm_w;   /* bf16 [128] or NULL (no K norm)              */
  float eps;
  const float* cos_sin;       /* fp32 [cos_sin_rows, rot_dim] = [cos | sin]  */
  int32_t cos_sin_rows, rot_dim;
  int32_t rope_style;         /* 0 NeoX, 1 GPT-J                             */
  const int64_t* positions;   /* [T] or NULL (derived)                       */
  const int32_t* q_indptr;    /* [B + 1]                                     */
  const int32_t* seq_lens;    /* [B], length after the append                */
  const int32_t* page_table;  /* [B, max_pages]                              */
  int32_t max_pages;
  int32_t num_pages, page_size;
  int32_t quant_policy;       /* 0 bf16, 1 dynamic Q, 2 static Q             */
  float q_scale_inv, k_scale, v_scale, upper_max;
  /* outputs (host memory, modified in place) */
  void* k_cache;              /* [num_pages, page_size, Hkv, 128] codes      */
  void* v_cache;
  int64_t k_page_stride, v_page_stride;   /* elements between pages         */
  void* out_q;                /* [T, Hq, 128] bf16 bits or e4m3 codes        */
  float* q_scale;             /* policy 1: [T, Hq] (max_seqlen 0) or
                                 [B, Hq, round_up(max_seqlen, 128)]; else NULL */
  int32_t* flags;             /* [B]                                         */
  int32_t max_seqlen;         /* policy 1: 0 decode layout, > 0 prefill layout
                                 and the n_b <= max_seqlen check              */
  int32_t norm_style;         /* 0: y = x_hat * w, 1 (Gemma): x_hat * (1 + w) */
  void* out_k;                /* [T, Hkv, 128] or NULL (paged caches)        */
  void* out_v;
} fqro_append_args;

/* Returns 0 after a valid call, 1 when the metadata was flagged. */
int fqro_append_paged(const fqro_append_args* a);

/* ---- the MLA latent concat ---------------------------------------------- */
typedef struct {
  uint16_t* q;                /* bf16, rope part rotated in place             */
  int32_t T, B, Hq, nope_dim, rope_dim;
  int64_t q_token_stride, q_head_stride;  /* elements                        */
  const uint16_t* kv_c;       /* bf16 [T, kv_c_stride], first kv_lora_rank   */
  int32_t kv_lora_rank;
  int64_t kv_c_stride;        /* elements per token row                      */
  const uint16_t* k_pe;       /* bf16 [T, k_pe_stride], first rope_dim       */
  int64_t k_pe_stride;
  const float* cos_sin;       /* fp32 [cos_sin_rows, rope_dim]               */
  int32_t cos_sin_rows, rope_style;
  const int64_t* positions;
  const int32_t* q_indptr;
  const int32_t* seq_lens;
  const int32_t* block_table; /* [B, max_blocks]                             */
  int32_t max_blocks;
  void* latent_cache;         /* [num_blocks, block_size, rank + rope_dim]   */
  int32_t num_blocks, block_size;
  int32_t cache_fp8;          /* 1: e4m3 codes (x / kv_scale), 0: bf16 bits   */
  float kv_scale;
  int32_t* flags;             /* [B]                                         */
  /* Q quantisation: 0 none (rope part rotated in place, BF16); otherwise q is
   * read-only and q_out [T, Hq, nope + rope] receives e4m3 codes of
   * v = [nope | rope(rope part)] (fp32):
   *   1 static per-tensor:     e4m3(v * q_scale_inv)
   *   2 dynamic per-token:     s = max(max |v| over the token, 1e-6) / upper_max,
   *                            e4m3(v / s), q_scale [T]
   *   3 dynamic per-head:      the same with the max over one head, q_scale [T, Hq]
   *   4 dynamic per-group:     the same with the max over each group of q_group
   *                            consecutive values of a head (the last group of a
   *                            head may be shorter), q_scale [T, Hq, ceil(W / q_group)] */
  int32_t q_quant;
  float q_scale_inv, upper_max;
  uint8_t* q_out;
  float* q_scale;
  int32_t q_group;            /* elements per group (q_quant 4), >= 1          */
} fqro_mla_args;

int fqro_concat_mla_cache(const fqro_mla_args* a);

#ifdef __cplusplus
}
#endif
#endif /* FQR_ORACLE_H */
