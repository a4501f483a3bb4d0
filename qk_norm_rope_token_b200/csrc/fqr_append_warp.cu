// fqr_append_warp.cu -- latency schedule of the fused append (small batches,
// e.g. decode): many independent warp tasks, all resident at once.
//
// Method: FlashInfer PR #5956, section "Contract" (see fqr_head.cuh for the
// per-head arithmetic).
//
//   * head task = 4 heads of one packed row (8 lanes per head), in quad-major
//     order (consecutive warps take the same quad of consecutive rows); the
//     task's two 16-byte loads per lane need no metadata and are issued before
//     the validation prologue; the next task's loads are issued before the
//     current task is computed.
//   * the first task also reads its own request's metadata in that first
//     round trip (request guessed as b = t) and, when it is consistent and
//     in bounds, issues its page-id and cos/sin loads before the prologue, so
//     the second dependent round trip overlaps the batch validation.
//   * every block stages q_indptr / seq_lens in shared memory and validates the
//     whole batch (stage_and_validate); a malformed batch writes only flags.
//     When every warp holds one task and the batch is small, every warp
//     validates the batch on its own instead (WarpBatchCheck): no barrier.
//   * the warps of a request's last new row split that request's last-page
//     tail (both caches) evenly between them and store their share of zeros
//     before their heads (the stores drain while the heads are computed);
//     one "request task" per request zeroes the tail of requests that append
//     nothing -- or, when tails are small and every warp holds one task,
//     every request's whole tail, so that the head tasks share none.
//   * blocks of 8 warps, or of 12 when that spreads a one-pass grid evenly
//     over the SMs (warp_block_threads).
#include "fqr_head.cuh"
#include "fqr_launch.h"

namespace fqr {

struct WarpArgs {
  HeadParams hp;
  FastDiv qdiv;  // division by quads (tail shares)
  FastDiv tdiv;  // division by T (head task -> quad, row)
  const uint16_t* qkv;
  int64_t row_stride;
  int T, B, H, quads, n_head;
  const uint16_t* qw;
  const uint16_t* kw;
  const float* cs;
  int cs_rows;
  const int64_t* positions;
  const int32_t* q_indptr;
  const int32_t* seq_lens;
  const int32_t* page_table;
  int max_pages;
  int64_t slot_cap;  // max_pages * page_size; INT64_MAX with caller-owned K/V
  int max_seqlen;    // > 0: the dynamic-Q prefill check n_b <= max_seqlen
  int bulk_tail;     // tails by bulk copies (warps with several tasks)
  int own_tails;     // request tasks zero whole tails (head tasks share none)
  int32_t* flags;
};

// Shared memory: fp32 weights [256], q_indptr [B + 1], seq_lens [B], then the
// zero buffer of the bulk tails (16-byte aligned).
__host__ __device__ __forceinline__ int warp_zero_offset(int B) {
  return ((2 * kHeadDim + 2 * B + 1) * static_cast<int>(sizeof(int)) + 15) & ~15;
}

// Packed row t and quad of head task w, in quad-major order (w = quad * T +
// t): consecutive warps take the same quad of consecutive rows, so a block's
// warps serve different requests and each writes one share of its request's
// tail -- an SM zeroes parts of many requests' tails, not all of one.
// (Measured on B200 against row-major order, which put a row's quads on
// consecutive warps: Qwen3-style decode 3.51 -> 3.20 us per launch, FP8
// decode with 256 rows 8.58 -> 8.28 us, tiny decode 2.49 -> 2.25 us; there
// the SMs with the largest tails set the launch time.)
__device__ __forceinline__ void head_task(const WarpArgs& a, int w, int& t, int& quad) {
  quad = static_cast<int>(a.tdiv.div(static_cast<uint32_t>(w)));
  t = w - quad * a.T;
}

__device__ __forceinline__ void warp_load_head(const WarpArgs& a, int w, int g, int l8, uint4& xa,
                                               uint4& xb) {
  int t, quad;
  head_task(a, w, t, quad);
  const int h = quad * 4 + g;
  if (h < a.H) {
    const uint16_t* src = a.qkv + static_cast<int64_t>(t) * a.row_stride + h * kHeadDim + 8 * l8;
    xa = ld_stream_v4(src);
    xb = ld_stream_v4(src + 64);
  }
}

// Pull into L2 the lines task w's second round trip will read -- its
// page-table entry and its row's cos/sin values -- while the warp still works
// on its current task (the request comes from the staged q_indptr, so this
// runs after the prologue).  A warp with several tasks otherwise pays a full
// DRAM round trip for these at the start of each later task.
__device__ __forceinline__ void prefetch_task_lines(const WarpArgs& a, int w, const int* s_indptr,
                                                    const int* s_seq, int lane, bool paged) {
  int t, quad;
  head_task(a, w, t, quad);
  const int h0 = quad * 4;
  const int b = request_of_row(s_indptr, a.B, t);
  const int end = s_indptr[b + 1];
  const int p_slot = t + s_seq[b] - end;
  if (lane == 0) {
    if (paged && (h0 + 3 >= a.hp.Hq || t == end - 1))
      prefetch_l2(a.page_table + static_cast<int64_t>(b) * a.max_pages +
                  a.hp.pdiv.div(static_cast<uint32_t>(p_slot)));
  } else if (a.positions == nullptr && 32 * (lane - 1) < a.hp.rot && h0 < a.hp.Hq + a.hp.Hkv) {
    prefetch_l2(a.cs + static_cast<int64_t>(p_slot) * a.hp.rot + 32 * (lane - 1));
  }
}

// WV: every warp validates the batch itself (WarpBatchCheck, batches of at
// most kWarpCheckMaxB requests) and reads metadata and weights from global
// memory: no block barrier, no shared-memory staging, so no warp waits for
// the slowest first round trip of its block.  Chosen for launches in which
// every warp holds one task; correct for any.  Measured on B200 against the
// block-staged prologue: Qwen3-style decode (128 requests, Hq/Hkv 32/8)
// 3.82 -> 3.50 us per launch, tiny decode 2.48 -> 2.24 us.

template <int POLICY, int STYLE, int NT, bool WV>
__global__ void __launch_bounds__(NT, NT == kThreads ? 2 : 0) warp_append_kernel(const WarpArgs a) {
  constexpr int NW = NT / 32;  // warps per block
  // a warp with one task waits on its own chain: the short form of the
  // mean square (inv_rms_n) -- in the wide block, whose threads have no
  // register cap (the short form needs more registers than 128)
  constexpr int kForm = WV && NT == kWideThreads ? kSumShort : kSumMixed;
  extern __shared__ __align__(16) int smem[];
  float* s_w = reinterpret_cast<float*>(smem);  // 256 fp32 weights
  int* s_indptr = smem + 2 * kHeadDim;          // B + 1
  int* s_seq = s_indptr + a.B + 1;              // B
  unsigned char* s_zero =                       // kZeroBytes (bulk tails)
      reinterpret_cast<unsigned char*>(smem) + warp_zero_offset(a.B);

  // (a shuffled warp index is known to the compiler to be warp-uniform, so
  // the task loop and the head-kind dispatch branch uniformly)
  const int lane = threadIdx.x & 31;
  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x >> 5), 0);
  const int g = lane >> 3, l8 = lane & 7;
  const unsigned gmask = 0xFFu << (8 * g);
  const int gwarp = blockIdx.x * NW + warp;
  const int nwarps = gridDim.x * NW;

  const bool paged = a.hp.out_k == nullptr;
  // The first task's coordinates need only the kernel parameters: computed
  // once, for the prefetches below and for the loads after the wait.
  const bool head0 = gwarp < a.n_head;
  int t0 = 0, h0 = a.H, gb = 0;
  const uint16_t* src0 = a.qkv;
  if (head0) {
    int q0;
    head_task(a, gwarp, t0, q0);
    h0 = q0 * 4 + g;
    gb = t0 < a.B - 1 ? t0 : a.B - 1;
    src0 = a.qkv + static_cast<int64_t>(t0) * a.row_stride + h0 * kHeadDim + 8 * l8;
  }
  const bool own0 = head0 && h0 < a.H;  // this group has a head in the first task

  // While the preceding grid finishes: pull into L2 the lines of the first
  // round trip below (metadata, weights, the first task's packed row and its
  // own request's metadata), one prefetch per 128-byte line.
  {
    const int tid = threadIdx.x;
    if (32 * tid <= a.B) {
      prefetch_l2(a.q_indptr + 32 * tid);
      if (32 * tid < a.B) prefetch_l2(a.seq_lens + 32 * tid);
    }
    const uint16_t* w = tid < 2 ? a.qw : a.kw;
    if (tid < 4 && w != nullptr) prefetch_l2(w + 64 * (tid & 1));
    if (head0) {
      if (l8 == 0 && own0) {
        prefetch_l2(src0);
        prefetch_l2(src0 + 64);
      }
      // ... and, from a possibly stale read of that metadata (L2 only), the
      // lines of the second round trip: the page-table entry and the cos/sin
      // row (a wrong guess costs only a useless prefetch).  Only for paged
      // K/V: the read's latency delays the warp's arrival at the dependency
      // wait, which a cos/sin row alone does not repay (measured on B200,
      // decode into caller-owned K/V, 128 requests, Hq/Hkv 32/8: 2.90 ->
      // 2.75 us per launch without it; the paged Qwen3-style decode loses
      // 3.48 -> 3.55 us without it).
      int lo = 0, hi = 0, L = 0;
      int64_t ps = 0;
      if (lane == 0 && paged) {
        lo = ld_cg_s32(a.q_indptr + gb);
        hi = ld_cg_s32(a.q_indptr + gb + 1);
        L = ld_cg_s32(a.seq_lens + gb);
        if (a.positions != nullptr) ps = ld_cg_s64(a.positions + t0);
      }
      lo = __shfl_sync(0xffffffffu, lo, 0);
      hi = __shfl_sync(0xffffffffu, hi, 0);
      L = __shfl_sync(0xffffffffu, L, 0);
      ps = __shfl_sync(0xffffffffu, ps, 0);
      if (lo <= t0 && t0 < hi) {
        const int p = t0 + L - hi;
        const int64_t pos = a.positions != nullptr ? ps : static_cast<int64_t>(p);
        if (p >= 0 && p < a.slot_cap && pos >= 0 && pos < a.cs_rows) {
          if (lane == 0 && paged)
            prefetch_l2(a.page_table + static_cast<int64_t>(gb) * a.max_pages +
                        a.hp.pdiv.div(static_cast<uint32_t>(p)));
          if (lane >= 1 && 32 * (lane - 1) < a.hp.rot && h0 < a.hp.Hq + a.hp.Hkv)
            prefetch_l2(a.cs + pos * a.hp.rot + 32 * (lane - 1));
        }
      }
    }
  }
  grid_dependency_wait();
  grid_launch_dependents();

  // ---- first round trip: every load that needs no metadata -- the batch
  // metadata this thread stages, the norm weights, the first task's packed
  // heads and its own request's metadata (request guessed as b = t: one new
  // row per request, the decode case).
  const Meta m{a.q_indptr, a.seq_lens, a.positions, a.flags, a.T,
               a.B,         a.slot_cap,  a.cs_rows,  a.max_seqlen};
  MetaRegs meta{0, 0, 0, 0};
  WeightRegs<NT> wreg;
  WarpBatchCheck<kWarpCheckMaxB / 32> check;
  RegWeights wq{make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u), a.hp.gemma};
  if (WV) {
    check.load(m, lane);
    // the lane's own weight slices for its first head (Q or K; none for V)
    const uint16_t* wsrc = h0 < a.hp.Hq ? a.qw : (h0 < a.hp.Hq + a.hp.Hkv ? a.kw : nullptr);
    if (own0 && wsrc != nullptr) {
      wq.wa = __ldg(reinterpret_cast<const uint4*>(wsrc + 8 * l8));
      wq.wb = __ldg(reinterpret_cast<const uint4*>(wsrc + 64 + 8 * l8));
    }
  } else {
    meta = meta_prefetch(a.q_indptr, a.seq_lens, a.B);
    wreg = weight_prefetch_nt<NT>(a.qw, a.kw, a.hp.gemma);
  }
  uint4 pa = make_uint4(0u, 0u, 0u, 0u), pb = pa;
  int e_lo = 0, e_hi = 0, e_L = 0;
  int64_t e_pos = 0;
  if (head0) {
    if (own0) {
      pa = ld_stream_v4(src0);
      pb = ld_stream_v4(src0 + 64);
    }
    e_lo = __ldg(a.q_indptr + gb);
    e_hi = __ldg(a.q_indptr + gb + 1);
    e_L = __ldg(a.seq_lens + gb);
    if (a.positions != nullptr) e_pos = __ldg(a.positions + t0);
  }
  // ---- second round trip, started before the validation prologue when the
  // row's own metadata is consistent and every address it yields is in
  // bounds (the prologue still decides whether anything is written).
  RowCtx r0{t0, 0, 0, 0, 0, 0};
  float2 c0[4], s0[4];
  bool early = false;
  if (head0 && h0 < a.H && e_lo <= t0 && t0 < e_hi) {
    const int p = t0 + e_L - e_hi;
    const int64_t pos = a.positions != nullptr ? e_pos : static_cast<int64_t>(p);
    if (p >= 0 && p < a.slot_cap && pos >= 0 && pos < a.cs_rows) {
      early = true;
      const int pidx = static_cast<int>(a.hp.pdiv.div(static_cast<uint32_t>(p)));
      r0.slot_row = p - pidx * a.hp.page_size;
      r0.pos = static_cast<int>(pos);
      r0.is_last = t0 == e_hi - 1;
      r0.qs = q_scale_row(a.hp, t0, gb, t0 - e_lo);
      // K/V slot, or the tail share of the last row
      if (paged && (h0 >= a.hp.Hq || (r0.is_last && !a.own_tails)))
        r0.page = __ldg(a.page_table + static_cast<int64_t>(gb) * a.max_pages + pidx);
      if (h0 < a.hp.Hq + a.hp.Hkv)
        load_cs<STYLE, false>(a.cs + pos * a.hp.rot, a.hp.rot, l8, c0, s0);
    }
  }
  const bool bulk = !WV && a.bulk_tail;  // (WV: no block-wide zero buffer)
  bool issued = false;                    // bulk copies in flight (lane 0)
  if (WV) {
    const bool bad = check.bad(m, lane);
    write_flags(m, bad);
    if (bad) return;
  } else {
    weight_store_nt<NT>(s_w, wreg);
    if (bulk) zero_buffer_init(s_zero);  // (the prologue's barrier follows)
    if (stage_and_validate(m, s_indptr, s_seq, meta)) return;
  }
  const GlobalWeights wg{a.qw, a.kw, a.hp.gemma};

  const int n_tasks = a.n_head + a.B;
  for (int w = gwarp; w < n_tasks; w += nwarps) {
    if (w < a.n_head) {
      const uint4 xa = pa, xb = pb;
      if (w + nwarps < a.n_head) {
        warp_load_head(a, w + nwarps, g, l8, pa, pb);
        if (!WV) prefetch_task_lines(a, w + nwarps, s_indptr, s_seq, lane, paged);
      }
      int t, quad;
      head_task(a, w, t, quad);
      if (w == gwarp && early) {  // the batch is valid: the early lookups stand
        // (the tail stores need nothing from the head: issue them first so they
        // drain while the head is computed)
        if (paged && r0.is_last && !a.own_tails) {
          if (bulk)
            issued |= zero_tail_share_bulk(a.hp, r0.page, r0.slot_row, quad, a.qdiv, lane, s_zero);
          else
            zero_tail_share(a.hp, r0.page, r0.slot_row, quad, a.qdiv, lane);
        }
        if (WV)
          process_quad_cs<POLICY, STYLE, kForm>(a.hp, r0, 4 * quad, a.H, g, xa, xb, c0, s0, wq,
                                                l8, gmask);
        else
          process_quad_cs<POLICY, STYLE, kForm>(a.hp, r0, 4 * quad, a.H, g, xa, xb, c0, s0, s_w,
                                                l8, gmask);
        continue;
      }
      const int h = quad * 4 + g;
      const int b = WV ? request_of_row_global(a.q_indptr, a.B, t) : request_of_row(s_indptr, a.B, t);
      const int beg = WV ? __ldg(a.q_indptr + b) : s_indptr[b];
      const int end = WV ? __ldg(a.q_indptr + b + 1) : s_indptr[b + 1];
      const int p_slot = t + (WV ? __ldg(a.seq_lens + b) : s_seq[b]) - end;
      const int pidx = static_cast<int>(a.hp.pdiv.div(static_cast<uint32_t>(p_slot)));
      RowCtx r;
      r.t = t;
      r.slot_row = p_slot - pidx * a.hp.page_size;
      r.pos = a.positions != nullptr ? static_cast<int>(a.positions[t]) : p_slot;
      r.is_last = t == end - 1;
      r.qs = q_scale_row(a.hp, t, b, t - beg);
      const bool share = paged && r.is_last && !a.own_tails;
      r.page = paged && (h >= a.hp.Hq || share)
                   ? __ldg(a.page_table + static_cast<int64_t>(b) * a.max_pages + pidx)
                   : 0;
      if (share) {
        if (bulk)
          issued |= zero_tail_share_bulk(a.hp, r.page, r.slot_row, quad, a.qdiv, lane, s_zero);
        else
          zero_tail_share(a.hp, r.page, r.slot_row, quad, a.qdiv, lane);
      }
      // (a group past the last head only helps with the tail)
      const float* cs_row = a.cs + static_cast<int64_t>(r.pos) * a.hp.rot;
      if (WV)
        process_quad<POLICY, STYLE, false, kForm>(a.hp, r, 4 * quad, a.H, g, xa, xb, cs_row, wg,
                                                  l8, gmask);
      else
        process_quad<POLICY, STYLE, false, kForm>(a.hp, r, 4 * quad, a.H, g, xa, xb, cs_row,
                                                  s_w, l8, gmask);
    } else {
      // request task: the tail of a request without new rows (whose tail no
      // head task shares), or of every request when request tasks own tails
      const int b = w - a.n_head;
      const int L = WV ? __ldg(a.seq_lens + b) : s_seq[b];
      const bool empty = WV ? __ldg(a.q_indptr + b) == __ldg(a.q_indptr + b + 1)
                            : s_indptr[b] == s_indptr[b + 1];
      if (paged && L > 0 && (a.own_tails || empty))
        zero_request_tail<POLICY == 0 ? 2 : 1>(a.hp, a.page_table, a.max_pages, b, L, lane);
    }
  }
  if (issued) bulk_wait_all();  // the zero buffer must outlive the copies
}

using WarpKernel = void (*)(const WarpArgs);

template <int NT, bool WV>
static WarpKernel select_warp_nt(int policy, int style) {
  if (style == 0) {
    if (policy == 0) return warp_append_kernel<0, 0, NT, WV>;
    if (policy == 1) return warp_append_kernel<1, 0, NT, WV>;
    return warp_append_kernel<2, 0, NT, WV>;
  }
  if (policy == 0) return warp_append_kernel<0, 1, NT, WV>;
  if (policy == 1) return warp_append_kernel<1, 1, NT, WV>;
  return warp_append_kernel<2, 1, NT, WV>;
}

static WarpKernel select_warp(int policy, int style, int nt, bool wv = false) {
  if (wv)
    return nt == kWideThreads ? select_warp_nt<kWideThreads, true>(policy, style)
                              : select_warp_nt<kThreads, true>(policy, style);
  return nt == kWideThreads ? select_warp_nt<kWideThreads, false>(policy, style)
                            : select_warp_nt<kThreads, false>(policy, style);
}

static size_t warp_smem(const fqr_append_params& p) {
  return static_cast<size_t>(warp_zero_offset(p.B)) + kZeroBytes;
}

int64_t latency_tasks(const fqr_append_params& p) {
  return static_cast<int64_t>(p.T) * ((p.Hq + 2 * p.Hkv + 3) / 4) + p.B;
}

// Threads per block of the latency schedule.  Blocks of kThreads while one
// pass of them leaves every SM at most one block; when it would put two
// blocks on some SMs and one on the others, and one block of kWideThreads
// per SM holds every task, the wide block spreads the warps evenly: an SM
// with twice the warps of its neighbours takes longer in every phase of the
// launch (load round trips, prologue, stores), and it sets the launch time.
// Measured on B200 (decode, Hq/Hkv 32/8, 128 requests: 1,664 warp tasks;
// 208 blocks of 8 warps leave 60 SMs with 16 warps, 139 blocks of 12 one
// per SM): paged K/V 3.55 -> 3.49 us per launch, caller-owned K/V 3.01 ->
// 2.91 us (with the warp-level batch check; 4.04 -> 3.81 us before it).
int warp_block_threads(const fqr_append_params& p) {
  DeviceInfo d;
  if (device_info(&d) != FQR_OK) return kThreads;
  const int64_t tasks = latency_tasks(p);
  const int64_t narrow_blocks = (tasks + kWarps - 1) / kWarps;
  const int64_t wide_blocks = (tasks + kWideThreads / 32 - 1) / (kWideThreads / 32);
  return narrow_blocks > d.sms && wide_blocks <= d.sms ? kWideThreads : kThreads;
}

int64_t latency_capacity(const fqr_append_params& p) {
  DeviceInfo d;
  int per_sm = 0;
  const int nt = kThreads;  // (the wide block only serves grids of at most one block per SM)
  const void* fn = reinterpret_cast<const void*>(select_warp(p.quant_policy, p.rope_style, nt));
  if (device_info(&d) != FQR_OK || resident_blocks(fn, nt, warp_smem(p), &per_sm) != FQR_OK)
    return -1;
  return static_cast<int64_t>(per_sm) * d.sms * (nt / 32);
}

// Request tasks zero whole tails (and the head tasks none) when every warp
// holds one task and a request's expected tail, (P - 1) / 2 rows of both
// caches, is at most this many bytes: one warp then writes it in a few
// stores while the heads run without a tail share.  Larger tails are split
// over the warps of the request's last row.  Measured on B200 (decode, one
// row per request): Hq/Hkv 8/1, page 16 (3.75 KiB): 2.99 -> 2.47 us at 1
// request, 3.50 -> 2.86 us at 128; Hq/Hkv 32/8, page 16 (30 KiB): 2.75 ->
// 3.57 us at 4 requests with whole tails, so those keep the shares.
constexpr int64_t kOwnTailsMaxBytes = 4096;

int launch_append_warp(const fqr_append_params& p, const HeadParams& hp, cudaStream_t stream,
                       fqr_append_plan* plan) {
  WarpArgs a;
  a.hp = hp;
  a.qkv = p.qkv;
  a.row_stride = p.qkv_row_stride;
  a.T = p.T;
  a.B = p.B;
  a.H = p.Hq + 2 * p.Hkv;
  a.quads = (a.H + 3) / 4;
  const int64_t n_head = static_cast<int64_t>(p.T) * a.quads;
  if (n_head + p.B >= (int64_t{1} << 31)) return FQR_ENOTSUP;
  a.n_head = static_cast<int>(n_head);
  a.qdiv = FastDiv(static_cast<uint32_t>(a.quads));
  a.tdiv = FastDiv(static_cast<uint32_t>(p.T > 0 ? p.T : 1));
  a.qw = p.q_norm_w;
  a.kw = p.k_norm_w;
  a.cs = p.cos_sin_cache;
  a.cs_rows = p.cos_sin_rows;
  a.positions = p.positions;
  a.q_indptr = p.q_indptr;
  a.seq_lens = p.seq_lens;
  a.page_table = p.page_table;
  a.max_pages = p.max_pages;
  a.slot_cap = hp.out_k != nullptr ? INT64_MAX : static_cast<int64_t>(p.max_pages) * p.page_size;
  a.max_seqlen = p.quant_policy == 1 ? p.max_seqlen : 0;
  a.flags = p.flags;
  const size_t smem = warp_smem(p);
  const int nt = warp_block_threads(p);
  // Warp-level validation when every warp holds one task (the launch is one
  // pass) and the batch is small enough for one warp to check.
  const int64_t cap = latency_capacity(p);
  const bool wv = cap >= n_head + p.B && p.B <= kWarpCheckMaxB &&
                  (p.positions == nullptr || p.T <= kWarpCheckMaxPositions);
  WarpKernel k = select_warp(p.quant_policy, p.rope_style, nt, wv);
  return launch_persistent(
      reinterpret_cast<const void*>(k), n_head + p.B, smem, stream,
      [&](int grid) {
        // bulk tails once warps have more than one task
        a.bulk_tail = static_cast<int64_t>(grid) * (nt / 32) < n_head + p.B;
        a.own_tails = !a.bulk_tail && static_cast<int64_t>(p.page_size - 1) * hp.row_bytes <=
                                          kOwnTailsMaxBytes;
        if (plan != nullptr) {
          *plan = fqr_append_plan{FQR_SCHEDULE_LATENCY, grid, nt, a.n_head + p.B, wv ? 1 : 0,
                                  a.bulk_tail, a.own_tails};
          return FQR_OK;
        }
        return launch_pdl(k, grid, nt, smem, stream, a);
      },
      nt);
}

}  // namespace fqr
