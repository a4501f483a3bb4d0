/*
 * fqr_oracle.c -- plain, slow, obviously correct CPU oracle of the fused
 * pre-attention preparation path.  TEST INFRASTRUCTURE ONLY (see the header):
 * nothing in the product path includes, links or calls this file.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math (no FMA
 * contraction: every product and every sum is rounded to fp32 on its own).
 *
 * Sources (pages about the method, cited by title and section):
 *  [FI]  FlashInfer PR #5956, "fused QK RMSNorm + NeoX RoPE + FP8 E4M3
 *        quantize + NHD paged-KV append", sections "Contract", "What changes"
 *        (test list) and the review thread on device-side validation.
 *  [TRT] TensorRT-LLM PR #16024 "Fuse Qwen3.5 gated QKV preprocessing",
 *        review excerpt of the fused QK norm (rsqrt(sum_sq / head_size + eps)).
 *  [SGL] SGLang PR #43425 (fused Q/K RMSNorm + RoPE on SM100), "Modifications".
 *  [VLLM] vLLM issue #24678 "ROPE + KV-Cache-Write + pre-attn prepare-ops
 *        fusion" (MLA latent concat, interleaved RoPE for DeepSeek R1).
 *
 * parity pinned: every function below is checked by tests/test_oracle_*.py
 * against closed forms, invariants, exhaustive brute force (encoders) or an
 * inverse-direction brute-force model (slots, tails, flags).
 */
#include "fqr_oracle.h"

#include <math.h>
#include <string.h>

#define D FQRO_HEAD_DIM

/* ------------------------------------------------------------------------ */
/* Formats                                                                   */
/* ------------------------------------------------------------------------ */

/* BF16 is the top half of an IEEE binary32: widening is exact. */
float fqro_bf16_to_f32(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* Round-to-nearest, ties-to-even, from binary32 to bfloat16 (8-bit
 * significand, same exponent range).  Computed from the definition: find the
 * binade of |x|, count quanta of that binade in exact double arithmetic, round
 * the count to the nearest integer (ties to even), and rebuild.  Overflow past
 * the largest finite value goes to infinity, NaN stays a (quiet) NaN. */
uint16_t fqro_f32_to_bf16_rne(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  if (isnan(x)) return (uint16_t)((u >> 16) | 0x0040u);
  uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  if (isinf(x)) return (uint16_t)(sign | 0x7F80u);
  double a = fabs((double)x);
  if (a == 0.0) return sign;
  int e;
  (void)frexp(a, &e);
  int E = e - 1;                       /* a in [2^E, 2^(E+1)) */
  if (E < -126) E = -126;              /* subnormal binade spacing */
  double quantum = ldexp(1.0, E - 7);  /* 7 stored fraction bits */
  double r = rint(a / quantum) * quantum;
  if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80u);
  float rf = (float)r;                 /* exact: r has <= 8 significant bits */
  uint32_t ur;
  memcpy(&ur, &rf, 4);
  return (uint16_t)(sign | (uint16_t)(ur >> 16));
}

/* OCP FP8 E4M3 ("fn" variant): 1 sign, 4 exponent (bias 7), 3 fraction bits;
 * no infinities; S.1111.111 is NaN; largest finite 448 = S.1111.110;
 * subnormals m * 2^-9.  Round to nearest, ties to even on the fraction, and
 * saturate: every |x| >= 448 (infinity included) becomes +-448, as the
 * satfinite conversion the FlashInfer page names ("RN satfinite FP8") does.
 * NaN becomes 0x7F. */
uint8_t fqro_f32_to_e4m3_rn_satfinite(float x) {
  if (isnan(x)) return 0x7F;
  uint8_t sign = signbit(x) ? 0x80 : 0x00;
  double a = fabs((double)x);
  if (a >= 448.0) return (uint8_t)(sign | 0x7E);
  if (a == 0.0) return sign;
  int e;
  (void)frexp(a, &e);
  int E = e - 1;
  if (E < -6) E = -6;                  /* below 2^-6 the spacing is 2^-9 */
  double quantum = ldexp(1.0, E - 3);  /* 3 fraction bits */
  double n = rint(a / quantum);        /* exact division by a power of two */
  if (E == -6 && n < 8.0) return (uint8_t)(sign | (uint8_t)n); /* subnormal */
  if (n >= 16.0) {                     /* rounded up into the next binade */
    E += 1;
    n = 8.0;
  }
  return (uint8_t)(sign | (uint8_t)(((E + 7) << 3) | ((int)n - 8)));
}

void fqro_f32_to_e4m3_array(const float* x, uint8_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = fqro_f32_to_e4m3_rn_satfinite(x[i]);
}

void fqro_f32_to_bf16_array(const float* x, uint16_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = fqro_f32_to_bf16_rne(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Per-head steps                                                            */
/* ------------------------------------------------------------------------ */

/* RMSNorm over one head ([TRT] review excerpt; [FI] "per-head RMSNorm eps
 * 1e-6"): mean square over all n elements, eps inside the square root, then
 * scale and weight.
 *
 * The mean square is the fp32 rounding of the exact mean of the squares
 * ([FI] "What changes": an fp32 reference of the norm; the sum itself has no
 * stated order, so no order is taken).  The squares are formed and summed in
 * binary64: a BF16 value has 8 significant bits, so its square has 16, and
 * the binary64 sum of 128 of them is exact whenever the head's nonzero
 * magnitudes span at most 2^15 (2 * 15 + 16 + 7 <= 53 bits); beyond that it
 * is within 2^-46 of the exact sum, far inside one fp32 rounding.  The sum is
 * then divided by n and rounded once to fp32; eps is added, and the square
 * root and the reciprocal are taken, each as one correctly rounded fp32
 * operation. */
void fqro_rmsnorm(const float* x, const float* w, int n, float eps, float* y) {
  double ss = 0.0;
  for (int i = 0; i < n; ++i) {
    double sq = (double)x[i] * (double)x[i];
    ss = ss + sq;
  }
  float ms = (float)(ss / (double)n);
  float inv = 1.0f / sqrtf(ms + eps);
  for (int i = 0; i < n; ++i) {
    float t = x[i] * inv;
    y[i] = w ? t * w[i] : t;
  }
}

/* NeoX ("rotate half") RoPE ([SGL] "full-width NeoX rotation", [FI] "NeoX
 * RoPE"): element i pairs with i + rot/2; the cache row is [cos | sin]. */
void fqro_rope_neox(float* y, const float* cs_row, int rot) {
  int half = rot / 2;
  for (int i = 0; i < half; ++i) {
    float c = cs_row[i], s = cs_row[half + i];
    float a = y[i], b = y[i + half];
    float ac = a * c, bs = b * s, bc = b * c, as = a * s;
    y[i] = ac - bs;
    y[i + half] = bc + as;
  }
}

/* GPT-J (interleaved) RoPE ([VLLM] "RoPE/NoPE interleaved" for DeepSeek R1):
 * element 2i pairs with 2i + 1; the cache row is [cos | sin]. */
void fqro_rope_gptj(float* y, const float* cs_row, int rot) {
  int half = rot / 2;
  for (int i = 0; i < half; ++i) {
    float c = cs_row[i], s = cs_row[half + i];
    float a = y[2 * i], b = y[2 * i + 1];
    float ac = a * c, bs = b * s, bc = b * c, as = a * s;
    y[2 * i] = ac - bs;
    y[2 * i + 1] = bc + as;
  }
}

static void rope(float* y, const float* cs_row, int rot, int style) {
  if (style == 0)
    fqro_rope_neox(y, cs_row, rot);
  else
    fqro_rope_gptj(y, cs_row, rot);
}

/* ------------------------------------------------------------------------ */
/* Validation ([FI] "Contract": malformed q_indptr -> all flags -1 and nothing */
/* written; the review thread adds seq_lens < new tokens, page-table overrun  */
/* and cos/sin row overrun to the same rule).                                */
/* ------------------------------------------------------------------------ */
int fqro_validate(const int32_t* q_indptr, const int32_t* seq_lens, int32_t B,
                  int32_t T, int32_t max_pages, int32_t page_size,
                  int32_t cos_sin_rows, const int64_t* positions,
                  int32_t max_seqlen, int32_t paged) {
  if (q_indptr[0] != 0) return 1;
  if (q_indptr[B] != T) return 1;
  for (int32_t b = 0; b < B; ++b) {
    int64_t lo = q_indptr[b], hi = q_indptr[b + 1], L = seq_lens[b];
    if (hi < lo) return 1;
    if (L < hi - lo) return 1;  /* derived positions would go negative */
    if (paged && L > (int64_t)max_pages * page_size) return 1;
    if (!positions && L > cos_sin_rows) return 1;
    /* dynamic-Q prefill: a request may not outgrow its q_scale rows */
    if (max_seqlen > 0 && hi - lo > max_seqlen) return 1;
  }
  if (positions) {
    for (int32_t t = 0; t < T; ++t)
      if (positions[t] < 0 || positions[t] >= cos_sin_rows) return 1;
  }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Paged append ([FI] "Contract")                                            */
/* ------------------------------------------------------------------------ */

static void widen_head(const uint16_t* src, float* x, int n) {
  for (int i = 0; i < n; ++i) x[i] = fqro_bf16_to_f32(src[i]);
}

/* Norm weights as fp32; the Gemma-style norm scales by 1 + w, formed in fp32
 * ([TRT] "qk_norm_use_gemma"). */
static void norm_weights(const uint16_t* w, int gemma, float* out) {
  widen_head(w, out, D);
  if (gemma)
    for (int i = 0; i < D; ++i) out[i] = 1.0f + out[i];
}

int fqro_append_paged(const fqro_append_args* a) {
  /* the dynamic-Q prefill layout and its max_seqlen check exist for policy 1
   * only; with caller-owned K/V outputs no page is addressed */
  const int32_t msl = a->quant_policy == 1 ? a->max_seqlen : 0;
  const int paged = a->out_k == NULL;
  if (fqro_validate(a->q_indptr, a->seq_lens, a->B, a->T, a->max_pages,
                    a->page_size, a->cos_sin_rows, a->positions, msl, paged)) {
    for (int32_t b = 0; b < a->B; ++b) a->flags[b] = -1;
    return 1;
  }
  const int P = a->page_size;
  const int fp8 = a->quant_policy != 0;
  const int64_t ld = ((int64_t)msl + 127) / 128 * 128;  /* prefill q_scale row */
  float wq[D], wk[D], x[D], y[D];
  if (a->q_norm_w) norm_weights(a->q_norm_w, a->norm_style == 1, wq);
  if (a->k_norm_w) norm_weights(a->k_norm_w, a->norm_style == 1, wk);

  for (int32_t b = 0; b < a->B; ++b) {
    int64_t lo = a->q_indptr[b], hi = a->q_indptr[b + 1], L = a->seq_lens[b];
    for (int64_t r = lo; r < hi; ++r) {
      /* seq_lens is the length after the append: token r sits at
       * r + L - q_indptr[b + 1]; the KV slot always uses that position. */
      int64_t p_slot = r + L - hi;
      int64_t pos = a->positions ? a->positions[r] : p_slot;
      int64_t page = paged ? a->page_table[(int64_t)b * a->max_pages + p_slot / P] : 0;
      int64_t row = p_slot % P;
      const float* cs = a->cos_sin + pos * a->rot_dim;
      const uint16_t* src = a->qkv + r * a->row_stride;

      for (int h = 0; h < a->Hq; ++h) {
        widen_head(src + (int64_t)h * D, x, D);
        if (a->q_norm_w)
          fqro_rmsnorm(x, wq, D, a->eps, y);
        else
          memcpy(y, x, sizeof y);
        rope(y, cs, a->rot_dim, a->rope_style);
        int64_t o = (r * a->Hq + h) * D;
        if (a->quant_policy == 0) {
          uint16_t* q = (uint16_t*)a->out_q + o;
          for (int i = 0; i < D; ++i) q[i] = fqro_f32_to_bf16_rne(y[i]);
        } else if (a->quant_policy == 1) {
          /* dynamic per-token/per-head scale: max(max|q|, 1e-6) / upper_max,
           * payload q / q_scale ([FI] "Contract" and test list) */
          float amax = 0.0f;
          for (int i = 0; i < D; ++i) amax = fmaxf(amax, fabsf(y[i]));
          float qs = fmaxf(amax, 1e-6f) / a->upper_max;
          /* decode layout [T, Hq]; prefill layout [B, Hq, ld] addressed by
           * the token's index inside its request ([FI] "Contract") */
          if (msl > 0)
            a->q_scale[((int64_t)b * a->Hq + h) * ld + (r - lo)] = qs;
          else
            a->q_scale[r * a->Hq + h] = qs;
          uint8_t* q = (uint8_t*)a->out_q + o;
          for (int i = 0; i < D; ++i) q[i] = fqro_f32_to_e4m3_rn_satfinite(y[i] / qs);
        } else {
          /* static per-tensor: payload q * q_scale_inv */
          uint8_t* q = (uint8_t*)a->out_q + o;
          for (int i = 0; i < D; ++i)
            q[i] = fqro_f32_to_e4m3_rn_satfinite(y[i] * a->q_scale_inv);
        }
      }
      void* kdst = paged ? a->k_cache : a->out_k;
      void* vdst = paged ? a->v_cache : a->out_v;
      for (int kh = 0; kh < a->Hkv; ++kh) {
        /* the cache slot, or row r of the caller-owned K / V outputs */
        int64_t ko = paged ? page * a->k_page_stride + (row * a->Hkv + kh) * D
                           : (r * a->Hkv + kh) * D;
        int64_t vo = paged ? page * a->v_page_stride + (row * a->Hkv + kh) * D
                           : (r * a->Hkv + kh) * D;
        /* K head */
        widen_head(src + (int64_t)(a->Hq + kh) * D, x, D);
        if (a->k_norm_w)
          fqro_rmsnorm(x, wk, D, a->eps, y);
        else
          memcpy(y, x, sizeof y);
        rope(y, cs, a->rot_dim, a->rope_style);
        if (!fp8) {
          uint16_t* k = (uint16_t*)kdst + ko;
          for (int i = 0; i < D; ++i) k[i] = fqro_f32_to_bf16_rne(y[i]);
        } else {
          uint8_t* k = (uint8_t*)kdst + ko;
          for (int i = 0; i < D; ++i) k[i] = fqro_f32_to_e4m3_rn_satfinite(y[i] / a->k_scale);
        }
        /* V head: a bit copy in BF16, x / v_scale in FP8 */
        const uint16_t* vs = src + (int64_t)(a->Hq + a->Hkv + kh) * D;
        if (!fp8) {
          memcpy((uint16_t*)vdst + vo, vs, D * sizeof(uint16_t));
        } else {
          uint8_t* v = (uint8_t*)vdst + vo;
          for (int i = 0; i < D; ++i)
            v[i] = fqro_f32_to_e4m3_rn_satfinite(fqro_bf16_to_f32(vs[i]) / a->v_scale);
        }
      }
    }
  }

  /* Rows [last + 1, page_size) of every request's last page are zeroed in
   * both caches ([FI] "Contract"); a request with L == 0 has no last page.
   * Redirected K/V writes leave the caches alone ([FI] review). */
  const int64_t esize = fp8 ? 1 : 2;
  for (int32_t b = 0; paged && b < a->B; ++b) {
    int64_t L = a->seq_lens[b];
    if (L <= 0) continue;
    int64_t last = (L - 1) % P;
    int64_t page = a->page_table[(int64_t)b * a->max_pages + (L - 1) / P];
    for (int64_t row = last + 1; row < P; ++row) {
      int64_t ko = page * a->k_page_stride + row * a->Hkv * D;
      int64_t vo = page * a->v_page_stride + row * a->Hkv * D;
      memset((char*)a->k_cache + ko * esize, 0, (size_t)(a->Hkv * D * esize));
      memset((char*)a->v_cache + vo * esize, 0, (size_t)(a->Hkv * D * esize));
    }
  }
  for (int32_t b = 0; b < a->B; ++b) a->flags[b] = 0;
  return 0;
}

/* ------------------------------------------------------------------------ */
/* MLA latent concat ([VLLM] concat_and_cache_mla; interleaved RoPE on the    */
/* rope part of Q and on k_pe; latent row = [kv_c | rope(k_pe)])             */
/* ------------------------------------------------------------------------ */
/* The fp32 values v = [nope | rope(rope part)] of head h of row r. */
static void mla_q_values(const fqro_mla_args* a, int64_t r, int h, const float* cs, float* v) {
  const uint16_t* qp = a->q + r * a->q_token_stride + h * a->q_head_stride;
  widen_head(qp, v, a->nope_dim + a->rope_dim);
  rope(v + a->nope_dim, cs, a->rope_dim, a->rope_style);
}

/* Q quantisation of row r ([VLLM] "static per-tensor, dynamic per-token, and
 * dynamic per-group"; the scale and payload forms of the dynamic per-head Q
 * scale of [FI] "Contract"). */
static void quantize_q(const fqro_mla_args* a, int64_t r, const float* cs) {
  const int W = a->nope_dim + a->rope_dim;
  float v[1024];
  float s = 0.0f;
  if (a->q_quant == 4) {  /* one scale per group of q_group values of a head */
    const int G = a->q_group, ng = (W + G - 1) / G;
    for (int h = 0; h < a->Hq; ++h) {
      mla_q_values(a, r, h, cs, v);
      uint8_t* out = a->q_out + (r * a->Hq + h) * W;
      for (int k = 0; k < ng; ++k) {
        const int lo = k * G, hi = lo + G < W ? lo + G : W;
        float amax = 0.0f;
        for (int i = lo; i < hi; ++i) amax = fmaxf(amax, fabsf(v[i]));
        s = fmaxf(amax, 1e-6f) / a->upper_max;
        a->q_scale[(r * a->Hq + h) * ng + k] = s;
        for (int i = lo; i < hi; ++i) out[i] = fqro_f32_to_e4m3_rn_satfinite(v[i] / s);
      }
    }
    return;
  }
  if (a->q_quant == 2) {  /* one scale for the whole token */
    float amax = 0.0f;
    for (int h = 0; h < a->Hq; ++h) {
      mla_q_values(a, r, h, cs, v);
      for (int i = 0; i < W; ++i) amax = fmaxf(amax, fabsf(v[i]));
    }
    s = fmaxf(amax, 1e-6f) / a->upper_max;
    a->q_scale[r] = s;
  }
  for (int h = 0; h < a->Hq; ++h) {
    mla_q_values(a, r, h, cs, v);
    if (a->q_quant == 3) {  /* one scale per head */
      float amax = 0.0f;
      for (int i = 0; i < W; ++i) amax = fmaxf(amax, fabsf(v[i]));
      s = fmaxf(amax, 1e-6f) / a->upper_max;
      a->q_scale[r * a->Hq + h] = s;
    }
    uint8_t* out = a->q_out + (r * a->Hq + h) * W;
    for (int i = 0; i < W; ++i)
      out[i] = fqro_f32_to_e4m3_rn_satfinite(a->q_quant == 1 ? v[i] * a->q_scale_inv : v[i] / s);
  }
}

int fqro_concat_mla_cache(const fqro_mla_args* a) {
  if (fqro_validate(a->q_indptr, a->seq_lens, a->B, a->T, a->max_blocks,
                    a->block_size, a->cos_sin_rows, a->positions, 0, 1)) {
    for (int32_t b = 0; b < a->B; ++b) a->flags[b] = -1;
    return 1;
  }
  const int R = a->rope_dim, K = a->kv_lora_rank, W = K + R;
  float y[512];
  if (R > 512 || a->nope_dim + R > 1024) return 2;
  if (a->q_quant == 4 && a->q_group < 1) return 2;
  for (int32_t b = 0; b < a->B; ++b) {
    int64_t lo = a->q_indptr[b], hi = a->q_indptr[b + 1], L = a->seq_lens[b];
    for (int64_t r = lo; r < hi; ++r) {
      int64_t p_slot = r + L - hi;
      int64_t pos = a->positions ? a->positions[r] : p_slot;
      int64_t blk = a->block_table[(int64_t)b * a->max_blocks + p_slot / a->block_size];
      int64_t row = p_slot % a->block_size;
      const float* cs = a->cos_sin + pos * R;
      if (a->q_quant == 0) {
        /* Q: rotate the rope part in place, the nope part is left as it is */
        for (int h = 0; h < a->Hq; ++h) {
          uint16_t* qp = a->q + r * a->q_token_stride + h * a->q_head_stride + a->nope_dim;
          widen_head(qp, y, R);
          rope(y, cs, R, a->rope_style);
          for (int i = 0; i < R; ++i) qp[i] = fqro_f32_to_bf16_rne(y[i]);
        }
      } else {
        quantize_q(a, r, cs);
      }
      /* latent row */
      int64_t base = (blk * a->block_size + row) * W;
      const uint16_t* kc = a->kv_c + r * a->kv_c_stride;
      widen_head(a->k_pe + r * a->k_pe_stride, y, R);
      rope(y, cs, R, a->rope_style);
      if (a->cache_fp8) {
        uint8_t* dst = (uint8_t*)a->latent_cache + base;
        for (int i = 0; i < K; ++i)
          dst[i] = fqro_f32_to_e4m3_rn_satfinite(fqro_bf16_to_f32(kc[i]) / a->kv_scale);
        for (int i = 0; i < R; ++i)
          dst[K + i] = fqro_f32_to_e4m3_rn_satfinite(y[i] / a->kv_scale);
      } else {
        uint16_t* dst = (uint16_t*)a->latent_cache + base;
        memcpy(dst, kc, (size_t)K * sizeof(uint16_t));
        for (int i = 0; i < R; ++i) dst[K + i] = fqro_f32_to_bf16_rne(y[i]);
      }
    }
  }
  for (int32_t b = 0; b < a->B; ++b) a->flags[b] = 0;
  return 0;
}
