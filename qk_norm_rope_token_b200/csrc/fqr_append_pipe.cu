// fqr_append_pipe.cu -- streaming schedule of the fused append (large
// batches, e.g. prefill): each block pipelines its rows through shared memory.
//
// Method: FlashInfer PR #5956, section "Contract" (see fqr_head.cuh for the
// per-head arithmetic).
//
// One block = 1 producer warp + 7 consumer warps; persistent grid, every
// block resident; each block owns a contiguous range of units (a unit is one
// packed row, or a chunk of its heads for very wide rows).
//   * the producer streams each unit into a ring of shared-memory stages with
//     1-D bulk copies (cp.async.bulk, the TMA engine; never multicast): the
//     packed heads and the token's cos/sin row, completing on a "full"
//     mbarrier.  The first stages' packed heads are requested before the
//     validation prologue.  The producer's 32 lanes resolve request, position
//     and page id of 32 units in parallel; the cos/sin copy is issued before
//     the page id is known, and the stage header (slot, page, position, last
//     row, q_scale index) is published by the arrive that completes the phase.
//   * consumer warps take 4 heads at a time from the stage (fqr_head.cuh),
//     store straight to out_q / the cache slot and release the stage on its
//     "empty" mbarrier; the quad -> warp assignment rotates every unit.
//   * the consumer warps split the last-page tail of a request's last row
//     evenly between them (after releasing the stage); consumer warps of the
//     grid zero the tails of requests that append nothing.
//   * every block validates the whole batch first; every wait is bounded
//     (kWaitLimitNs) and a wait that gives up sets every flag to kFlagTimeout.
#include "fqr_head.cuh"
#include "fqr_launch.h"

namespace fqr {

constexpr int kConsumers = 7;
constexpr int kPipeThreads = (kConsumers + 1) * 32;
constexpr int kMaxStages = 8;
constexpr int kFixedSmem = 1280;  // barriers (128) + fp32 weights (1024) + spare
constexpr int kHeader = 32;       // stage header bytes (keeps the copies 16-byte aligned)
// A NeoX cos/sin row (512 bytes) is staged as four 128-byte quarters with 16
// bytes between them (kCsPadded in fqr_head.cuh), which makes the lanes'
// 32-byte slices of it fall on distinct bank groups.
constexpr uint32_t kCsQuarter = 128;

// Stage header, written by the producer before it arrives on "full".
struct StageInfo {
  int slot_row, page, pos, is_last, qs;
};
static_assert(sizeof(StageInfo) <= kHeader, "stage header");

struct PipeArgs {
  HeadParams hp;
  FastDiv cdiv;  // division by nchunks
  FastDiv wdiv;  // division by kConsumers (tail shares)
  const uint16_t* qkv;
  int64_t row_stride;
  int T, B, H;
  int chunk_heads, nchunks;
  int64_t units;
  const uint16_t* qw;
  const uint16_t* kw;
  const float* cs;
  int cs_rows, cs_bulk, cs_bytes;
  const int64_t* positions;
  const int32_t* q_indptr;
  const int32_t* seq_lens;
  const int32_t* page_table;
  int max_pages;
  int64_t slot_cap;  // max_pages * page_size; INT64_MAX with caller-owned K/V
  int max_seqlen;    // > 0: the dynamic-Q prefill check n_b <= max_seqlen
  int32_t* flags;
  int stages, stage_bytes;
};

__device__ __forceinline__ uint4 ld_smem_v4(const void* p) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(smem_addr(p)));
  return r;
}
__device__ __forceinline__ float4 ld_smem_f4(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}

__device__ void report_timeout(const PipeArgs& a) { flag_timeout(a.flags, a.B, threadIdx.x & 31); }

// Unit u: packed row t, heads [h0, h0 + nh).
__device__ __forceinline__ void unit_heads(const PipeArgs& a, int64_t u, int& t, int& h0,
                                           int& nh) {
  t = static_cast<int>(a.cdiv.div(static_cast<uint32_t>(u)));
  h0 = (static_cast<int>(u) - t * a.nchunks) * a.chunk_heads;
  nh = min(a.H - h0, a.chunk_heads);
}

// Producer lane: bulk-copy the packed heads of unit u into stage `st`.
__device__ __forceinline__ void issue_heads(const PipeArgs& a, unsigned char* st, int64_t u,
                                            uint64_t* bar) {
  int t, h0, nh;
  unit_heads(a, u, t, h0, nh);
  const uint32_t bytes = static_cast<uint32_t>(nh) * kHeadDim * 2;
  mbar_expect_tx(bar, bytes);
  bulk_g2s(st + kHeader + a.cs_bytes,
           a.qkv + static_cast<int64_t>(t) * a.row_stride + static_cast<int64_t>(h0) * kHeadDim,
           bytes, bar);
}

// ------------------------------------------------------------- producer --
template <int STYLE>
__device__ void produce(const PipeArgs& a, unsigned char* stages, uint64_t* full,
                        uint64_t* empty, const int* s_indptr, const int* s_seq, int64_t u0,
                        int nunits, int pre) {
  const int lane = threadIdx.x & 31;
  const int S = a.stages;
  int ok = 1;
  int issued = pre;  // stages whose head copies are in flight or consumed
  int s = 0;         // stage of unit i
  uint32_t eph = 1;  // parity of the empty-phase to wait for (previous use of stage s)
  for (int i0 = 0; i0 < nunits && ok; i0 += 32) {
    // lane j prepares unit i0 + j in parallel with the others
    StageInfo info{0, 0, 0, 0, 0};  // slot_row, page, pos, is_last, qs
    int need_cs = 0;
    if (i0 + lane < nunits) {
      int t, h0, nh;
      unit_heads(a, u0 + i0 + lane, t, h0, nh);
      const int b = request_of_row(s_indptr, a.B, t);
      const int end = s_indptr[b + 1];
      const int p = t + s_seq[b] - end;
      const int pidx = static_cast<int>(a.hp.pdiv.div(static_cast<uint32_t>(p)));
      info.slot_row = p - pidx * a.hp.page_size;
      info.pos = a.positions != nullptr ? static_cast<int>(a.positions[t]) : p;
      info.is_last = t == end - 1;
      info.qs = q_scale_row(a.hp, t, b, t - s_indptr[b]);
      // a unit with K or V heads, or of a last row (tail), needs the page id
      // (unless K/V go to owned rows)
      if ((h0 + nh > a.hp.Hq || info.is_last) && a.hp.out_k == nullptr)
        info.page = __ldg(a.page_table + static_cast<int64_t>(b) * a.max_pages + pidx);
      need_cs = (h0 < a.hp.Hq + a.hp.Hkv) && a.cs_bulk;
    }
    const int n = min(32, nunits - i0);
    for (int j = 0; j < n; ++j) {
      // position first: the cos/sin copy must not wait for the page-id load
      const int posj = __shfl_sync(0xffffffffu, info.pos, j);
      const int csj = __shfl_sync(0xffffffffu, need_cs, j);
      const int i = i0 + j;
      uint64_t* fb = &full[s];
      unsigned char* st = stages + static_cast<size_t>(s) * a.stage_bytes;
      if (lane == 0) {
        if (i >= S && !mbar_wait(&empty[s], eph)) ok = 0;
        if (ok) {
          fence_proxy_async_smem();
          if (i >= pre) {
            issue_heads(a, st, u0 + i, fb);
            ++issued;
          }
          if (csj) {
            const float* src = a.cs + static_cast<int64_t>(posj) * a.hp.rot;
            if (STYLE == 0) {  // NeoX rows: four 128-byte quarters, 16 bytes apart (kCsPadded)
              mbar_expect_tx(fb, 4 * kCsQuarter);
              for (int k = 0; k < 4; ++k)
                bulk_g2s(st + kHeader + k * (kCsQuarter + 16), src + k * (kCsQuarter / 4),
                         kCsQuarter, fb);
            } else {
              const uint32_t cb = static_cast<uint32_t>(a.hp.rot) * 4;
              mbar_expect_tx(fb, cb);
              bulk_g2s(st + kHeader, src, cb, fb);
            }
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const StageInfo sj{__shfl_sync(0xffffffffu, info.slot_row, j),
                         __shfl_sync(0xffffffffu, info.page, j), posj,
                         __shfl_sync(0xffffffffu, info.is_last, j),
                         __shfl_sync(0xffffffffu, info.qs, j)};
      if (lane == 0) {
        *reinterpret_cast<StageInfo*>(st) = sj;
        mbar_arrive(fb);  // release: the header is visible once the phase completes
      }
      if (++s == S) {
        s = 0;
        eph ^= 1u;
      }
    }
  }
  if (!ok) {
    report_timeout(a);
    if (lane == 0) {  // let the copies already issued land before the block leaves
      const int first = issued > S ? issued - S : 0;
      for (int i = first; i < issued; ++i) mbar_wait(&full[i % S], (i / S) & 1);
    }
  }
}

// ------------------------------------------------------------ consumers --
template <int POLICY, int STYLE, bool CSB>
__device__ void consume(const PipeArgs& a, const unsigned char* stages, uint64_t* full,
                        uint64_t* empty, const float* s_w, int64_t u0, int nunits) {
  // (a shuffled warp index is known to the compiler to be warp-uniform, so the
  // quad loop below and the kind dispatch inside it branch uniformly)
  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x >> 5), 0);
  const int lane = threadIdx.x & 31;
  const int g = lane >> 3, l8 = lane & 7;
  const unsigned gmask = 0xFFu << (8 * g);
  const int S = a.stages;
  // (row, chunk) of the current unit, advanced without dividing
  int t = static_cast<int>(u0 / a.nchunks);
  int c = static_cast<int>(u0 - static_cast<int64_t>(t) * a.nchunks);
  int rot = 0;  // quad -> warp rotation, advanced by nq every unit
  int s = 0;
  uint32_t ph = 0;
  for (int i = 0; i < nunits; ++i) {
    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph))) {
      report_timeout(a);
      return;
    }
    const unsigned char* st = stages + static_cast<size_t>(s) * a.stage_bytes;
    const StageInfo info = *reinterpret_cast<const StageInfo*>(st);
    const RowCtx r{t, info.slot_row, info.pos, info.page, info.is_last, info.qs};
    const float* cs_row = CSB ? reinterpret_cast<const float*>(st + kHeader)
                              : a.cs + static_cast<int64_t>(info.pos) * a.hp.rot;
    const int h0 = c * a.chunk_heads, nh = min(a.H - h0, a.chunk_heads);
    const int nq = (nh + 3) >> 2;
    int q = warp - rot;
    if (q < 0) q += kConsumers;
    for (; q < nq; q += kConsumers) {
      const int hl = 4 * q + g;
      uint4 xa = make_uint4(0u, 0u, 0u, 0u), xb = xa;
      if (hl < nh) {
        const unsigned char* src = st + kHeader + a.cs_bytes + hl * (kHeadDim * 2) + 16 * l8;
        xa = ld_smem_v4(src);
        xb = ld_smem_v4(src + 128);
      }
      process_quad<POLICY, STYLE, CSB>(a.hp, r, h0 + 4 * q, h0 + nh, g, xa, xb, cs_row, s_w, l8,
                                       gmask);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    // the request's last row: the block's consumer warps split its last-page
    // tail (both caches) evenly, once per row (its first chunk)
    if (info.is_last && c == 0 && a.hp.out_k == nullptr)
      zero_tail_share(a.hp, info.page, info.slot_row, static_cast<uint32_t>(warp), a.wdiv, lane);
    if (++s == S) {
      s = 0;
      ph ^= 1u;
    }
    rot = (rot + nq) % kConsumers;
    if (++c == a.nchunks) {
      c = 0;
      ++t;
    }
  }
}

// Tails of requests that append no row in this call, spread over every
// consumer warp of the grid.
template <int POLICY>
__device__ void zero_empty_request_tails(const PipeArgs& a, const int* s_indptr, const int* s_seq) {
  if (a.hp.out_k != nullptr) return;  // caller-owned K/V: the caches are not touched
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int W = gridDim.x * kConsumers;
  for (int b = blockIdx.x * kConsumers + warp; b < a.B; b += W) {
    const int L = s_seq[b];
    if (s_indptr[b] == s_indptr[b + 1] && L > 0)
      zero_request_tail<POLICY == 0 ? 2 : 1>(a.hp, a.page_table, a.max_pages, b, L, lane);
  }
}

// Two resident blocks per SM: 16 warps, 4 on each of the 4 sub-partition
// register files (16K registers each), so up to 128 registers a thread.
// (Eight consumer warps a block would put 5 warps on some sub-partitions and
// cap a thread at 96 registers: measured slower, 86.1 -> 79.5 us per launch of
// the ragged FP8 prefill with seven.)
template <int POLICY, int STYLE>
__global__ void __launch_bounds__(kPipeThreads, 2) pipe_append_kernel(const PipeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kMaxStages;
  float* s_w = reinterpret_cast<float*>(smem + 128);   // staged fp32 weights (fqr_head.cuh)
  unsigned char* stages = smem + kFixedSmem;
  int* s_indptr = reinterpret_cast<int*>(stages + static_cast<size_t>(a.stages) * a.stage_bytes);
  int* s_seq = s_indptr + a.B + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool producer = warp == kConsumers;
  const int64_t u0 = static_cast<int64_t>(blockIdx.x) * a.units / gridDim.x;
  const int64_t u1 = static_cast<int64_t>(blockIdx.x + 1) * a.units / gridDim.x;
  const int nunits = static_cast<int>(u1 - u0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers);
    }
    mbar_init_fence();
  }
  // While the preceding grid finishes: pull into L2 the metadata, the
  // weights and the packed rows of this block's first two units, one
  // prefetch per 128-byte line (L2 is the point of coherence: the reads after
  // the wait still see the preceding grid's writes).
  {
    const int tid = threadIdx.x;
    if (32 * tid <= a.B) {
      prefetch_l2(a.q_indptr + 32 * tid);
      if (32 * tid < a.B) prefetch_l2(a.seq_lens + 32 * tid);
    }
    const uint16_t* w = tid < 2 ? a.qw : a.kw;
    if (tid < 4 && w != nullptr) prefetch_l2(w + 64 * (tid & 1));
    for (int i = 0; i < 2 && i < nunits; ++i) {
      int t, h0, nh;
      unit_heads(a, u0 + i, t, h0, nh);
      const uint16_t* src =
          a.qkv + static_cast<int64_t>(t) * a.row_stride + static_cast<int64_t>(h0) * kHeadDim;
      for (int l = tid; l < nh * 2; l += kPipeThreads) prefetch_l2(src + 64 * l);
    }
  }
  // Programmatic dependent launch: everything above touched only shared
  // memory (and prefetched); wait for the preceding grid before reading any
  // input, and let the next grid in the stream start its own set-up early.
  grid_dependency_wait();
  grid_launch_dependents();
  __syncthreads();

  // The first stages' packed heads need no metadata: start them now so their
  // latency overlaps the validation prologue.
  int pre = 0;
  if (producer && lane == 0) {
    pre = min(a.stages, nunits);
    for (int i = 0; i < pre; ++i)
      issue_heads(a, stages + static_cast<size_t>(i) * a.stage_bytes, u0 + i, &full[i]);
  }
  const MetaRegs meta = meta_prefetch(a.q_indptr, a.seq_lens, a.B);
  weight_store(s_w, weight_prefetch(a.qw, a.kw, a.hp.gemma));

  const Meta m{a.q_indptr, a.seq_lens, a.positions, a.flags, a.T,
               a.B,         a.slot_cap,  a.cs_rows,  a.max_seqlen};
  if (stage_and_validate(m, s_indptr, s_seq, meta)) {
    if (producer && lane == 0) {  // drain the copies issued before the verdict
      for (int i = 0; i < pre; ++i) {
        mbar_arrive(&full[i]);
        mbar_wait(&full[i], 0);
      }
    }
    return;
  }

  if (producer) {
    produce<STYLE>(a, stages, full, empty, s_indptr, s_seq, u0, nunits, pre);
  } else {
    zero_empty_request_tails<POLICY>(a, s_indptr, s_seq);
    if constexpr (STYLE == 0) {  // NeoX rows are 128 wide: always staged
      consume<POLICY, STYLE, true>(a, stages, full, empty, s_w, u0, nunits);
    } else {
      if (a.cs_bulk)
        consume<POLICY, STYLE, true>(a, stages, full, empty, s_w, u0, nunits);
      else
        consume<POLICY, STYLE, false>(a, stages, full, empty, s_w, u0, nunits);
    }
  }
}

using PipeKernel = void (*)(const PipeArgs);

static PipeKernel select_pipe(int policy, int style) {
  if (style == 0) {
    if (policy == 0) return pipe_append_kernel<0, 0>;
    if (policy == 1) return pipe_append_kernel<1, 0>;
    return pipe_append_kernel<2, 0>;
  }
  if (policy == 0) return pipe_append_kernel<0, 1>;
  if (policy == 1) return pipe_append_kernel<1, 1>;
  return pipe_append_kernel<2, 1>;
}

int launch_append_pipe(const fqr_append_params& p, const HeadParams& hp, cudaStream_t stream,
                       fqr_append_plan* plan) {
  PipeArgs a;
  a.hp = hp;
  a.qkv = p.qkv;
  a.row_stride = p.qkv_row_stride;
  a.T = p.T;
  a.B = p.B;
  a.H = p.Hq + 2 * p.Hkv;
  a.qw = p.q_norm_w;
  a.kw = p.k_norm_w;
  a.cs = p.cos_sin_cache;
  a.cs_rows = p.cos_sin_rows;
  a.cs_bulk = (p.rot_dim * 4) % 16 == 0 ? 1 : 0;
  a.cs_bytes = !a.cs_bulk ? 0 : p.rope_style == 0 ? kCsPaddedBytes : p.rot_dim * 4;
  a.positions = p.positions;
  a.q_indptr = p.q_indptr;
  a.seq_lens = p.seq_lens;
  a.page_table = p.page_table;
  a.max_pages = p.max_pages;
  a.slot_cap = hp.out_k != nullptr ? INT64_MAX : static_cast<int64_t>(p.max_pages) * p.page_size;
  a.max_seqlen = p.quant_policy == 1 ? p.max_seqlen : 0;
  a.flags = p.flags;

  DeviceInfo d;
  if (device_info(&d) != FQR_OK) return FQR_ECUDA;
  const int sms = d.sms, smem_optin = d.smem_optin, smem_sm = d.smem_sm;

  const int64_t meta = static_cast<int64_t>(2 * p.B + 1) * sizeof(int);
  auto stage_bytes = [&](int hc) { return kHeader + a.cs_bytes + hc * kHeadDim * 2; };
  // a row that does not fit two stages beside the metadata is split into
  // chunks of whole quads
  int hc = a.H;
  while (hc > 4 && kFixedSmem + meta + 2 * stage_bytes(hc) > smem_optin) hc = ((hc / 2 + 3) / 4) * 4;
  if (kFixedSmem + meta + stage_bytes(hc) > smem_optin) return FQR_ENOTSUP;
  a.chunk_heads = hc;
  a.nchunks = (a.H + hc - 1) / hc;
  a.units = static_cast<int64_t>(p.T) * a.nchunks;
  if (a.units >= (int64_t{1} << 31)) return FQR_ENOTSUP;
  a.cdiv = FastDiv(static_cast<uint32_t>(a.nchunks));
  a.wdiv = FastDiv(static_cast<uint32_t>(kConsumers));
  a.stage_bytes = stage_bytes(hc);
  // pipeline depth: aim at two resident blocks per SM (the register budget of
  // the consumers), never deeper than the units a block will see
  const int64_t per_block_budget = smem_sm / 2 - 1024;
  int S = static_cast<int>((per_block_budget - kFixedSmem - meta) / a.stage_bytes);
  S = S < 1 ? 1 : (S > kMaxStages ? kMaxStages : S);
  const int64_t upb = (a.units + 2 * sms - 1) / (2 * sms);
  if (upb >= 1 && S > upb) S = static_cast<int>(upb);
  while (S > 1 && kFixedSmem + meta + static_cast<int64_t>(S) * a.stage_bytes > smem_optin) --S;
  a.stages = S;
  const size_t smem = static_cast<size_t>(kFixedSmem + meta + static_cast<int64_t>(S) * a.stage_bytes);

  PipeKernel k = select_pipe(p.quant_policy, p.rope_style);
  int per_sm = 0;
  if (resident_blocks(reinterpret_cast<const void*>(k), kPipeThreads, smem, &per_sm) != FQR_OK)
    return FQR_ECUDA;
  const int64_t cap = static_cast<int64_t>(per_sm) * sms;
  const int64_t want = a.units > sms ? a.units : sms;
  const int grid = static_cast<int>(want < cap ? want : cap);
  if (plan != nullptr) {
    *plan = fqr_append_plan{FQR_SCHEDULE_STREAMING, grid, kPipeThreads, static_cast<int32_t>(a.units),
                            0, 0, 0};
    return FQR_OK;
  }
  return launch_pdl(k, grid, kPipeThreads, smem, stream, a);
}

}  // namespace fqr
