// fqr_api.cu -- the extern "C" entry points of libfqr.so (declared in
// include/fqr.h).  Each entry point checks every argument the host can check,
// returns an error code before any CUDA call if one is wrong, and otherwise
// enqueues exactly one kernel on the caller's stream.  Nothing is allocated,
// nothing is synchronised.
#include <cmath>
#include <cstdint>

#include "fqr.h"
#include "fqr_launch.h"

namespace {

inline bool aligned(const void* p, uintptr_t n) {
  return (reinterpret_cast<uintptr_t>(p) & (n - 1)) == 0;
}

}  // namespace

namespace fqr {

int check_append(const fqr_append_params* p) {
  if (p == nullptr) return FQR_EINVAL;
  if (p->T < 0 || p->B < 0 || p->B > FQR_MAX_BATCH) return FQR_EINVAL;
  if (p->B == 0 && p->T > 0) return FQR_EINVAL;  // q_indptr[0] must equal T
  if (p->head_dim != FQR_HEAD_DIM) return FQR_EINVAL;
  if (p->Hq <= 0 || p->Hkv <= 0 || p->Hq % p->Hkv != 0) return FQR_EINVAL;
  if (p->quant_policy < 0 || p->quant_policy > 2) return FQR_EINVAL;
  if (p->rope_style != 0 && p->rope_style != 1) return FQR_EINVAL;
  if (p->rot_dim < 2 || p->rot_dim > FQR_HEAD_DIM || (p->rot_dim & 1)) return FQR_EINVAL;
  if (!(std::isfinite(p->eps) && p->eps >= 0.0f)) return FQR_EINVAL;
  if (p->quant_policy == 1 &&
      !(std::isfinite(p->upper_max) && p->upper_max > 0.0f && p->upper_max <= 448.0f))
    return FQR_EINVAL;
  if (p->cos_sin_rows <= 0) return FQR_EINVAL;
  // caller-owned K/V rows (both or neither) replace the paged caches
  const bool owned = p->out_k != nullptr || p->out_v != nullptr;
  if (owned && (!p->out_k || !p->out_v || !aligned(p->out_k, 16) || !aligned(p->out_v, 16)))
    return FQR_EINVAL;
  const int64_t H = static_cast<int64_t>(p->Hq) + 2 * static_cast<int64_t>(p->Hkv);
  if (p->qkv_row_stride < H * FQR_HEAD_DIM || p->qkv_row_stride % 8 != 0) return FQR_EINVAL;
  const int64_t esize = p->quant_policy == 0 ? 2 : 1;
  if (!owned) {
    if (p->page_size <= 0 || p->num_pages <= 0 || p->max_pages <= 0) return FQR_EINVAL;
    // tail rows of the whole batch are counted in 32 bits
    if (2 * static_cast<int64_t>(p->B) * (p->page_size - 1) >= (int64_t{1} << 31))
      return FQR_EINVAL;
    const int64_t page_elems = static_cast<int64_t>(p->page_size) * p->Hkv * FQR_HEAD_DIM;
    if (p->k_page_stride < page_elems || p->v_page_stride < page_elems) return FQR_EINVAL;
    if ((p->k_page_stride * esize) % 16 != 0 || (p->v_page_stride * esize) % 16 != 0)
      return FQR_EINVAL;
    if (!p->page_table || !p->k_cache || !p->v_cache) return FQR_EINVAL;
    if (!aligned(p->k_cache, 16) || !aligned(p->v_cache, 16) || !aligned(p->page_table, 4))
      return FQR_EINVAL;
  }
  // the dynamic-Q prefill layout [B, Hq, round_up(max_seqlen, 128)] is indexed in 32 bits
  if (p->max_seqlen < 0) return FQR_EINVAL;
  if (p->quant_policy == 1 && p->max_seqlen > 0 &&
      static_cast<int64_t>(p->B) * p->Hq * ((static_cast<int64_t>(p->max_seqlen) + 127) / 128 * 128) >=
          (int64_t{1} << 31))
    return FQR_ENOTSUP;
  if (p->norm_style != FQR_NORM_RMS && p->norm_style != FQR_NORM_GEMMA) return FQR_EINVAL;
  // required pointers and their alignment
  if (!p->q_indptr || !p->seq_lens || !p->flags || !p->cos_sin_cache) return FQR_EINVAL;
  if (!aligned(p->cos_sin_cache, 16)) return FQR_EINVAL;
  if (!aligned(p->q_indptr, 4) || !aligned(p->seq_lens, 4) || !aligned(p->flags, 4) ||
      !aligned(p->positions, 8))
    return FQR_EINVAL;
  if (p->T > 0) {
    if (!p->qkv || !p->out_q || !aligned(p->qkv, 16) || !aligned(p->out_q, 16))
      return FQR_EINVAL;
  }
  if ((p->q_norm_w && !aligned(p->q_norm_w, 16)) || (p->k_norm_w && !aligned(p->k_norm_w, 16)))
    return FQR_EINVAL;
  if (p->quant_policy == 1 && (!p->q_scale || !aligned(p->q_scale, 4))) return FQR_EINVAL;
  if (p->quant_policy == 2 && !p->q_scale_inv) return FQR_EINVAL;
  if (p->quant_policy != 0 && (!p->k_scale || !p->v_scale)) return FQR_EINVAL;
  if (p->schedule < FQR_SCHEDULE_AUTO || p->schedule > FQR_SCHEDULE_STREAMING) return FQR_EINVAL;
  if (p->rope_style == 0 && p->rot_dim != FQR_HEAD_DIM) return FQR_ENOTSUP;
  return FQR_OK;
}

}  // namespace fqr

namespace {

int check_mla(const fqr_mla_params* p) {
  if (p == nullptr) return FQR_EINVAL;
  if (p->T < 0 || p->B < 0 || p->B > FQR_MAX_BATCH) return FQR_EINVAL;
  if (p->B == 0 && p->T > 0) return FQR_EINVAL;
  if (p->Hq <= 0 || p->nope_dim < 0 || p->kv_lora_rank <= 0) return FQR_EINVAL;
  if (p->rope_style != 0 && p->rope_style != 1) return FQR_EINVAL;
  if (p->rope_dim <= 0 || (p->rope_dim & 1)) return FQR_EINVAL;
  if (p->block_size <= 0 || p->num_blocks <= 0 || p->max_blocks <= 0 || p->cos_sin_rows <= 0)
    return FQR_EINVAL;
  if (p->cache_fp8 != 0 && p->cache_fp8 != 1) return FQR_EINVAL;
  if (!p->q_indptr || !p->seq_lens || !p->block_table || !p->flags || !p->latent_cache ||
      !p->cos_sin_cache)
    return FQR_EINVAL;
  if (p->cache_fp8 && !p->kv_scale) return FQR_EINVAL;
  if (!aligned(p->latent_cache, 16) || !aligned(p->cos_sin_cache, 4) ||
      !aligned(p->q_indptr, 4) || !aligned(p->seq_lens, 4) || !aligned(p->block_table, 4) ||
      !aligned(p->flags, 4) || !aligned(p->positions, 8))
    return FQR_EINVAL;
  if (p->T > 0) {
    if (!p->q || !p->kv_c || !p->k_pe) return FQR_EINVAL;
    if (!aligned(p->q, 16) || !aligned(p->kv_c, 16) || !aligned(p->k_pe, 16)) return FQR_EINVAL;
    if (p->q_head_stride < p->nope_dim + p->rope_dim) return FQR_EINVAL;
    if (p->q_token_stride < static_cast<int64_t>(p->Hq) * p->q_head_stride) return FQR_EINVAL;
    if (p->kv_c_stride < p->kv_lora_rank || p->k_pe_stride < p->rope_dim) return FQR_EINVAL;
  }
  if (p->q_quant < FQR_MLA_Q_NONE || p->q_quant > FQR_MLA_Q_GROUP) return FQR_EINVAL;
  if (p->q_quant == FQR_MLA_Q_GROUP && (p->q_group < 8 || p->q_group % 8)) return FQR_EINVAL;
  if (p->q_quant != FQR_MLA_Q_NONE) {
    if (p->T > 0 && (!p->q_out || !aligned(p->q_out, 16))) return FQR_EINVAL;
    if (p->q_quant == FQR_MLA_Q_STATIC && !p->q_scale_inv) return FQR_EINVAL;
    if (p->q_quant != FQR_MLA_Q_STATIC) {
      if (!p->q_scale || !aligned(p->q_scale, 4)) return FQR_EINVAL;
      if (!(std::isfinite(p->upper_max) && p->upper_max > 0.0f && p->upper_max <= 448.0f))
        return FQR_EINVAL;
    }
  }
  if (p->rope_dim != 64) return FQR_ENOTSUP;
  if (p->nope_dim % 4 || p->q_token_stride % 4 || p->q_head_stride % 4 || p->kv_lora_rank % 8 ||
      p->kv_c_stride % 8 || p->k_pe_stride % 4)
    return FQR_ENOTSUP;
  // quantised Q keeps a head's nope part (at most 256 dims) in registers,
  // loaded in 16-byte vectors
  if (p->q_quant != FQR_MLA_Q_NONE &&
      (p->nope_dim % 8 || p->nope_dim > 256 || p->q_token_stride % 8 || p->q_head_stride % 8))
    return FQR_ENOTSUP;
  return FQR_OK;
}

}  // namespace

extern "C" {

int fqr_append_paged(const fqr_append_params* p, void* stream) {
  if (p != nullptr && p->T == 0 && p->B == 0) return FQR_OK;  // empty batch: no launch
  const int rc = fqr::check_append(p);
  if (rc != FQR_OK) return rc;
  return fqr::launch_append(*p, static_cast<cudaStream_t>(stream));
}

int fqr_append_plan_query(const fqr_append_params* p, fqr_append_plan* plan) {
  if (plan == nullptr) return FQR_EINVAL;
  *plan = fqr_append_plan{0, 0, 0, 0, 0, 0, 0};
  if (p != nullptr && p->T == 0 && p->B == 0) return FQR_OK;  // nothing would launch
  const int rc = fqr::check_append(p);
  if (rc != FQR_OK) return rc;
  return fqr::launch_append(*p, nullptr, plan);
}

int fqr_concat_mla_cache(const fqr_mla_params* p, void* stream) {
  if (p != nullptr && p->T == 0 && p->B == 0) return FQR_OK;
  const int rc = check_mla(p);
  if (rc != FQR_OK) return rc;
  return fqr::launch_mla(*p, static_cast<cudaStream_t>(stream));
}

const char* fqr_strerror(int code) {
  switch (code) {
    case FQR_OK: return "ok";
    case FQR_EINVAL: return "invalid argument (nothing was launched)";
    case FQR_ENOTSUP: return "unsupported argument combination (nothing was launched)";
    case FQR_ECUDA: return "the CUDA runtime refused the launch";
    default: return "unknown fqr error code";
  }
}

}  // extern "C"
