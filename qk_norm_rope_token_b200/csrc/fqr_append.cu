// fqr_append.cu -- fqr_append_paged's launcher: builds the per-head
// parameters and picks one of the two schedules of the same computation.
//
//   latency schedule   (fqr_append_warp.cu): independent warp tasks, all
//                       resident at once -- small batches such as decode.
//   streaming schedule (fqr_append_pipe.cu): per-block bulk-copy pipeline
//                       through shared memory -- large batches such as prefill.
//
// Both write identical results (same arithmetic in fqr_head.cuh); the choice
// only changes how rows are spread over the GPU.
#include "fqr_head.cuh"
#include "fqr_launch.h"

namespace fqr {

constexpr int64_t kLargeTail = 48 * 1024;  // expected tail bytes per row (both caches)
constexpr int64_t kLargeTailPasses = 8;

int launch_append(const fqr_append_params& p, cudaStream_t stream, fqr_append_plan* plan) {
  HeadParams hp;
  const int es = p.quant_policy == 0 ? 2 : 1;
  const bool owned = p.out_k != nullptr;
  // with caller-owned K/V no page is addressed: a page size of 1 keeps the
  // slot arithmetic defined (its results are not used)
  const int page_size = owned ? 1 : p.page_size;
  hp.pdiv = FastDiv(static_cast<uint32_t>(page_size));
  hp.Hq = p.Hq;
  hp.Hkv = p.Hkv;
  hp.page_size = page_size;
  hp.row_bytes = p.Hkv * kHeadDim * es;
  hp.rot = p.rot_dim;
  hp.has_qw = p.q_norm_w != nullptr;
  hp.has_kw = p.k_norm_w != nullptr;
  hp.eps = p.eps;
  hp.upper_max = p.upper_max;
  hp.k_cache = static_cast<char*>(p.k_cache);
  hp.v_cache = static_cast<char*>(p.v_cache);
  hp.k_page_bytes = p.k_page_stride * es;
  hp.v_page_bytes = p.v_page_stride * es;
  hp.q_scale_inv = p.q_scale_inv;
  hp.k_scale = p.k_scale;
  hp.v_scale = p.v_scale;
  hp.out_q = p.out_q;
  hp.q_scale = p.q_scale;
  hp.gemma = p.norm_style == FQR_NORM_GEMMA;
  hp.qs_prefill = p.quant_policy == 1 && p.max_seqlen > 0;
  hp.qs_ld = hp.qs_prefill ? (p.max_seqlen + 127) / 128 * 128 : 1;
  hp.out_k = static_cast<char*>(p.out_k);
  hp.out_v = static_cast<char*>(p.out_v);

  int schedule = p.schedule;
  if (schedule == FQR_SCHEDULE_AUTO) {
    // Latency while every warp task has a resident warp of its own (one pass,
    // no task waits for another); streaming once the tasks outnumber the
    // resident warps and a pipeline hides the rest -- except for decode-like
    // batches (a row per request) whose last-page tails are large (an
    // expected kLargeTail bytes or more per row, half a page of both caches):
    // the latency schedule writes those with bulk copies while its warps move
    // on, and stays ahead up to kLargeTailPasses passes of tasks (measured on
    // B200 with 64 FP8 Q heads, 8 KV heads and 64-slot pages).
    const int64_t cap = latency_capacity(p);
    if (cap < 0) return FQR_ECUDA;
    const int64_t tasks = latency_tasks(p);
    const int64_t tail_per_row =
        owned ? 0 : static_cast<int64_t>(p.page_size - 1) * hp.row_bytes;  // (P-1)/2 rows x 2 caches
    const bool decode_like = p.T <= p.B;
    schedule = tasks <= cap || (decode_like && tail_per_row >= kLargeTail &&
                                tasks <= kLargeTailPasses * cap)
                   ? FQR_SCHEDULE_LATENCY
                   : FQR_SCHEDULE_STREAMING;
  }
  return schedule == FQR_SCHEDULE_STREAMING ? launch_append_pipe(p, hp, stream, plan)
                                            : launch_append_warp(p, hp, stream, plan);
}

}  // namespace fqr
