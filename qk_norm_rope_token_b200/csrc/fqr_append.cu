// fqr_append.cu -- fused per-head Q/K RMSNorm + RoPE + (optional) FP8 E4M3
// quantisation + paged K/V append + last-page tail zeroing, one launch.
//
// Method: FlashInfer PR #5956 (fused QK RMSNorm + NeoX RoPE + FP8 E4M3
// quantize + NHD paged-KV append), section "Contract"; RMSNorm as in the
// TensorRT-LLM PR #16024 review excerpt; fp32 cos/sin cache RoPE as in SGLang
// PR #43425 "Modifications".
//
// Structure (one block = 1 producer warp + 8 consumer warps, persistent grid
// with every block resident):
//   * work unit = one packed row (or, for very wide rows, a chunk of its
//     heads).  Each block owns a contiguous range of units.
//   * the producer warp streams each unit into a ring of shared-memory stages
//     with 1-D bulk copies (cp.async.bulk, the TMA engine; never multicast):
//     the packed Q|K|V heads and the token's cos/sin row, completing on a
//     "full" mbarrier.  The packed-row copies of the first stages are issued
//     before the validation prologue (their addresses need no metadata).  The
//     producer's 32 lanes look up each unit's request, position and page id in
//     parallel and write them into the stage header.
//   * consumer warps take 4 heads at a time (8 lanes per head, lane l holding
//     elements [8l, 8l+8) and [64+8l, 64+8l+8), so NeoX pairs never cross
//     lanes), normalise (xor shuffle inside the 8-lane group), rotate and
//     quantise in fp32 (sm_100 f32x2 instructions, every product rounded on
//     its own), store straight to out_q / the cache slot, and release the
//     stage on its "empty" mbarrier.  Heads are dealt to warps in a rotating
//     order so no warp always gets the extra quad.
//   * before the rows, the consumer warps zero the last-page tails: the
//     concatenated tail rows of all requests are split evenly over every
//     consumer warp of the grid (an exclusive scan gives each request's
//     offset).
//   * every block first validates the whole batch (stage_and_validate): a
//     malformed batch writes only the flags.
//   * every wait is bounded (kWaitLimitNs); a wait that gives up sets every
//     flag to kFlagTimeout and the block leaves after its copies drain.
#include "fqr_device.cuh"
#include "fqr_launch.h"

namespace fqr {

constexpr int kConsumers = 8;
constexpr int kPipeThreads = (kConsumers + 1) * 32;
constexpr int kMaxStages = 8;
constexpr int kFixedSmem = 1280;  // barriers (128) + fp32 weights (1024) + scan scratch

struct StageInfo {
  int b, p_slot, page, pos;
};

struct PipeArgs {
  const uint16_t* qkv;
  int64_t row_stride;
  int T, B, Hq, Hkv, H;
  int chunk_heads, nchunks;
  int64_t units;
  const uint16_t* qw;
  const uint16_t* kw;
  float eps;
  const float* cs;
  int cs_rows, rot, cs_bulk, cs_bytes;
  const int64_t* positions;
  const int32_t* q_indptr;
  const int32_t* seq_lens;
  const int32_t* page_table;
  int max_pages;
  char* k_cache;
  char* v_cache;
  int page_size, row_bytes;
  int64_t k_page_bytes, v_page_bytes;
  const float* q_scale_inv;
  const float* k_scale;
  const float* v_scale;
  float upper_max;
  void* out_q;
  float* q_scale;
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

__device__ void report_timeout(const PipeArgs& a) {
  for (int b = threadIdx.x & 31; b < a.B; b += 32) a.flags[b] = kFlagTimeout;
}

// Unit u: packed row t, heads [h0, h0 + nh).
__device__ __forceinline__ void unit_heads(const PipeArgs& a, int64_t u, int& t, int& h0,
                                           int& nh) {
  t = static_cast<int>(u / a.nchunks);
  h0 = static_cast<int>(u - static_cast<int64_t>(t) * a.nchunks) * a.chunk_heads;
  nh = min(a.H - h0, a.chunk_heads);
}

// Producer lane: bulk-copy the packed heads of unit u into stage `st`.
__device__ __forceinline__ void issue_heads(const PipeArgs& a, unsigned char* st, int64_t u,
                                            uint64_t* bar) {
  int t, h0, nh;
  unit_heads(a, u, t, h0, nh);
  const uint32_t bytes = static_cast<uint32_t>(nh) * kHeadDim * 2;
  mbar_expect_tx(bar, bytes);
  bulk_g2s(st + 16 + a.cs_bytes,
           a.qkv + static_cast<int64_t>(t) * a.row_stride + static_cast<int64_t>(h0) * kHeadDim,
           bytes, bar);
}

// ------------------------------------------------------------- producer --
__device__ void produce(const PipeArgs& a, unsigned char* stages, uint64_t* full,
                        uint64_t* empty, const int* s_indptr, const int* s_seq, int64_t u0,
                        int nunits, int pre) {
  const int lane = threadIdx.x & 31;
  const int S = a.stages;
  int ok = 1;
  int issued = pre;  // stages whose head copies are in flight or consumed
  for (int i0 = 0; i0 < nunits && ok; i0 += 32) {
    // lane j prepares unit i0 + j in parallel with the others
    StageInfo info{0, 0, 0, 0};
    int need_cs = 0;
    if (i0 + lane < nunits) {
      int t, h0, nh;
      unit_heads(a, u0 + i0 + lane, t, h0, nh);
      const int b = request_of_row(s_indptr, a.B, t);
      const int p = t + s_seq[b] - s_indptr[b + 1];
      info.b = b;
      info.p_slot = p;
      info.pos = a.positions != nullptr ? static_cast<int>(a.positions[t]) : p;
      if (h0 + nh > a.Hq)  // the unit holds K or V heads: it needs the page id
        info.page = __ldg(a.page_table + static_cast<int64_t>(b) * a.max_pages + p / a.page_size);
      need_cs = (h0 < a.Hq + a.Hkv) && a.cs_bulk;
    }
    const int n = min(32, nunits - i0);
    for (int j = 0; j < n; ++j) {
      const StageInfo sj{__shfl_sync(0xffffffffu, info.b, j),
                         __shfl_sync(0xffffffffu, info.p_slot, j),
                         __shfl_sync(0xffffffffu, info.page, j),
                         __shfl_sync(0xffffffffu, info.pos, j)};
      const int csj = __shfl_sync(0xffffffffu, need_cs, j);
      if (lane == 0) {
        const int i = i0 + j, s = i % S;
        uint64_t* fb = &full[s];
        if (i >= S && !mbar_wait(&empty[s], ((i / S) - 1) & 1)) ok = 0;
        if (ok) {
          unsigned char* st = stages + static_cast<size_t>(s) * a.stage_bytes;
          *reinterpret_cast<StageInfo*>(st) = sj;
          fence_proxy_async_smem();
          if (i >= pre) {
            issue_heads(a, st, u0 + i, fb);
            ++issued;
          }
          if (csj) {
            const uint32_t cb = static_cast<uint32_t>(a.rot) * 4;
            mbar_arrive_expect_tx(fb, cb);
            bulk_g2s(st + 16, a.cs + static_cast<int64_t>(sj.pos) * a.rot, cb, fb);
          } else {
            mbar_arrive(fb);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
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
template <int POLICY, int STYLE>
__device__ __forceinline__ void process_quad(const PipeArgs& a, const unsigned char* st,
                                             const StageInfo& info, int t, int h0, int nh, int q,
                                             int g, int l8, const float* s_w) {
  const int hl = 4 * q + g;
  if (hl >= nh) return;  // the whole 8-lane group leaves together
  const int h = h0 + hl;
  const unsigned gmask = 0xFFu << (8 * g);
  const unsigned char* src = st + 16 + a.cs_bytes + hl * (kHeadDim * 2) + 16 * l8;
  const uint4 xa = ld_smem_v4(src), xb = ld_smem_v4(src + 128);
  const int P = a.page_size;
  constexpr int es = POLICY == 0 ? 2 : 1;

  float y[16];
  unpack8(xa, y);
  unpack8(xb, y + 8);

  if (h >= a.Hq + a.Hkv) {  // ---------------------------------- V head
    const int kh = h - a.Hq - a.Hkv;
    char* dst = a.v_cache + static_cast<int64_t>(info.page) * a.v_page_bytes +
                (static_cast<int64_t>(info.p_slot % P) * a.Hkv + kh) * kHeadDim * es;
    if (POLICY == 0) {  // bit copy
      st_v4(dst + 16 * l8, xa);
      st_v4(dst + 128 + 16 * l8, xb);
    } else {
      const float vs = __ldg(a.v_scale);
#pragma unroll
      for (int k = 0; k < 16; ++k) y[k] = __fdiv_rn(y[k], vs);
      st_v2(dst + 8 * l8, pack8_e4m3(y));
      st_v2(dst + 64 + 8 * l8, pack8_e4m3(y + 8));
    }
    return;
  }

  const bool is_q = h < a.Hq;
  // cos/sin of this lane's pairs
  float c[8], s[8];
  const float* row = a.cs_bulk ? reinterpret_cast<const float*>(st + 16)
                               : a.cs + static_cast<int64_t>(info.pos) * a.rot;
  if (STYLE == 0) {  // NeoX, rot == 128: pairs (8l+k, 64+8l+k); cs_bulk always holds
    const float4 c0 = ld_smem_f4(row + 8 * l8), c1 = ld_smem_f4(row + 8 * l8 + 4);
    const float4 s0 = ld_smem_f4(row + 64 + 8 * l8), s1 = ld_smem_f4(row + 68 + 8 * l8);
    c[0] = c0.x; c[1] = c0.y; c[2] = c0.z; c[3] = c0.w;
    c[4] = c1.x; c[5] = c1.y; c[6] = c1.z; c[7] = c1.w;
    s[0] = s0.x; s[1] = s0.y; s[2] = s0.z; s[3] = s0.w;
    s[4] = s1.x; s[5] = s1.y; s[6] = s1.z; s[7] = s1.w;
  } else {  // GPT-J: chunk A pairs i = 4l + j, chunk B pairs i = 32 + 4l + j
    const int half = a.rot >> 1;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = (j < 4 ? 4 * l8 + j : 32 + 4 * l8 + (j - 4));
      const bool on = i < half;
      c[j] = on ? row[i] : 1.0f;
      s[j] = on ? row[half + i] : 0.0f;
    }
  }

  // ----------------------------------------------------------- RMSNorm
  if ((is_q ? a.qw : a.kw) != nullptr) {
    float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int k = 0; k < 16; k += 2) {
      const float2 v = make_float2(y[k], y[k + 1]);
      acc = fma2(v, v, acc);
    }
    float ss = acc.x + acc.y;
    ss += __shfl_xor_sync(gmask, ss, 4);
    ss += __shfl_xor_sync(gmask, ss, 2);
    ss += __shfl_xor_sync(gmask, ss, 1);
    const float inv = __frcp_rn(__fsqrt_rn(__fadd_rn(ss * (1.0f / kHeadDim), a.eps)));
    const float* wv = s_w + (is_q ? 0 : kHeadDim);
    const float4 w0 = ld_smem_f4(wv + 8 * l8), w1 = ld_smem_f4(wv + 8 * l8 + 4);
    const float4 w2 = ld_smem_f4(wv + 64 + 8 * l8), w3 = ld_smem_f4(wv + 68 + 8 * l8);
    const float w[16] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w,
                         w2.x, w2.y, w2.z, w2.w, w3.x, w3.y, w3.z, w3.w};
    const float2 iv = make_float2(inv, inv);
#pragma unroll
    for (int k = 0; k < 16; k += 2) {
      const float2 r = mul2(mul2(make_float2(y[k], y[k + 1]), iv), make_float2(w[k], w[k + 1]));
      y[k] = r.x;
      y[k + 1] = r.y;
    }
  }

  // -------------------------------------------------------------- RoPE
  if (STYLE == 0) {
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      const float2 av = make_float2(y[k], y[k + 1]), bv = make_float2(y[8 + k], y[9 + k]);
      const float2 cv = make_float2(c[k], c[k + 1]), sv = make_float2(s[k], s[k + 1]);
      const float2 ac = mul2(av, cv), bs = mul2(bv, sv), bc = mul2(bv, cv), as = mul2(av, sv);
      const float2 na = add2(ac, make_float2(-bs.x, -bs.y)), nb = add2(bc, as);
      y[k] = na.x; y[k + 1] = na.y; y[8 + k] = nb.x; y[9 + k] = nb.y;
    }
  } else {
    const int half = a.rot >> 1;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = (j < 4 ? 4 * l8 + j : 32 + 4 * l8 + (j - 4));
      const int e = (j < 4 ? 2 * j : 8 + 2 * (j - 4));
      if (i < half) rotate_pair(y[e], y[e + 1], c[j], s[j]);
    }
  }

  // ------------------------------------------------------------ output
  if (is_q) {
    const int64_t o = (static_cast<int64_t>(t) * a.Hq + h) * kHeadDim;
    if (POLICY == 0) {
      uint16_t* out = static_cast<uint16_t*>(a.out_q) + o;
      st_v4(out + 8 * l8, pack8_bf16(y));
      st_v4(out + 64 + 8 * l8, pack8_bf16(y + 8));
    } else {
      if (POLICY == 1) {
        float amax = 0.0f;
#pragma unroll
        for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(y[k]));
        amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, 4));
        amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, 1));
        const float qs = __fdiv_rn(fmaxf(amax, 1e-6f), a.upper_max);
        if (l8 == 0) a.q_scale[static_cast<int64_t>(t) * a.Hq + h] = qs;
#pragma unroll
        for (int k = 0; k < 16; ++k) y[k] = __fdiv_rn(y[k], qs);
      } else {
        const float qsi = __ldg(a.q_scale_inv);
        const float2 qv = make_float2(qsi, qsi);
#pragma unroll
        for (int k = 0; k < 16; k += 2) {
          const float2 r = mul2(make_float2(y[k], y[k + 1]), qv);
          y[k] = r.x;
          y[k + 1] = r.y;
        }
      }
      uint8_t* out = static_cast<uint8_t*>(a.out_q) + o;
      st_v2(out + 8 * l8, pack8_e4m3(y));
      st_v2(out + 64 + 8 * l8, pack8_e4m3(y + 8));
    }
  } else {
    const int kh = h - a.Hq;
    char* dst = a.k_cache + static_cast<int64_t>(info.page) * a.k_page_bytes +
                (static_cast<int64_t>(info.p_slot % P) * a.Hkv + kh) * kHeadDim * es;
    if (POLICY == 0) {
      st_v4(dst + 16 * l8, pack8_bf16(y));
      st_v4(dst + 128 + 16 * l8, pack8_bf16(y + 8));
    } else {
      const float ks = __ldg(a.k_scale);
#pragma unroll
      for (int k = 0; k < 16; ++k) y[k] = __fdiv_rn(y[k], ks);
      st_v2(dst + 8 * l8, pack8_e4m3(y));
      st_v2(dst + 64 + 8 * l8, pack8_e4m3(y + 8));
    }
  }
}

template <int POLICY, int STYLE>
__device__ void consume(const PipeArgs& a, const unsigned char* stages, uint64_t* full,
                        uint64_t* empty, const float* s_w, int64_t u0, int nunits) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 3, l8 = lane & 7;
  const int S = a.stages;
  // (row, chunk) of the current unit, advanced without dividing
  int t = static_cast<int>(u0 / a.nchunks);
  int c = static_cast<int>(u0 - static_cast<int64_t>(t) * a.nchunks);
  int rot = 0;  // quad -> warp rotation, advanced by nq every unit
  for (int i = 0; i < nunits; ++i) {
    const int s = i % S;
    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (i / S) & 1))) {
      report_timeout(a);
      return;
    }
    const unsigned char* st = stages + static_cast<size_t>(s) * a.stage_bytes;
    const StageInfo info = *reinterpret_cast<const StageInfo*>(st);
    const int h0 = c * a.chunk_heads, nh = min(a.H - h0, a.chunk_heads);
    const int nq = (nh + 3) >> 2;
    int q = warp - rot;
    if (q < 0) q += kConsumers;
    for (; q < nq; q += kConsumers) process_quad<POLICY, STYLE>(a, st, info, t, h0, nh, q, g, l8, s_w);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    rot = (rot + nq) & (kConsumers - 1);
    if (++c == a.nchunks) {
      c = 0;
      ++t;
    }
  }
}

// Consumer warps of the whole grid split the concatenated tail rows evenly.
// s_tail[b] = first tail row of request b (each request: its K rows, then
// its V rows); s_tail[B] = total.
__device__ void zero_tails(const PipeArgs& a, const int* s_seq, const int* s_tail) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t W = static_cast<int64_t>(gridDim.x) * kConsumers;
  const int64_t cw = static_cast<int64_t>(blockIdx.x) * kConsumers + warp;
  const int64_t Z = s_tail[a.B];
  int64_t r = cw * Z / W;
  const int64_t r_end = (cw + 1) * Z / W;
  if (r >= r_end) return;
  int b = upper_bound(s_tail, a.B + 1, static_cast<int>(r)) - 1;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  const int P = a.page_size;
  while (r < r_end) {
    const int64_t lo = s_tail[b], hi = s_tail[b + 1];
    if (hi <= r) {
      ++b;
      continue;
    }
    const int L = s_seq[b];
    const int last = (L - 1) % P, n = P - 1 - last;
    const int64_t page = __ldg(a.page_table + static_cast<int64_t>(b) * a.max_pages + (L - 1) / P);
    const int64_t j0 = r - lo, j1 = (r_end < hi ? r_end : hi) - lo;   // rows of [0, 2n)
    // K rows [0, n), V rows [n, 2n)
    for (int cache = 0; cache < 2; ++cache) {
      const int64_t c0 = max(j0, static_cast<int64_t>(cache * n)) - cache * n;
      const int64_t c1 = min(j1, static_cast<int64_t>((cache + 1) * n)) - cache * n;
      if (c0 >= c1) continue;
      char* base = cache == 0 ? a.k_cache + page * a.k_page_bytes : a.v_cache + page * a.v_page_bytes;
      const int64_t beg = (last + 1 + c0) * a.row_bytes, end = (last + 1 + c1) * a.row_bytes;
      for (int64_t off = beg + 16 * lane; off < end; off += 512) st_v4(base + off, z);
    }
    r = lo + j1;
    ++b;
  }
}

template <int POLICY, int STYLE>
__global__ void __launch_bounds__(kPipeThreads) append_kernel(const PipeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kMaxStages;
  float* s_w = reinterpret_cast<float*>(smem + 128);   // fp32 weights: [0,128) Q, [128,256) K
  int* s_scan = reinterpret_cast<int*>(smem + 1152);   // one int per warp
  unsigned char* stages = smem + kFixedSmem;
  int* s_indptr = reinterpret_cast<int*>(stages + static_cast<size_t>(a.stages) * a.stage_bytes);
  int* s_seq = s_indptr + a.B + 1;
  int* s_tail = s_seq + a.B;

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
  __syncthreads();

  // The first stages' packed heads need no metadata: start them now so their
  // latency overlaps the validation prologue.
  int pre = 0;
  if (producer && lane == 0) {
    pre = min(a.stages, nunits);
    for (int i = 0; i < pre; ++i)
      issue_heads(a, stages + static_cast<size_t>(i) * a.stage_bytes, u0 + i, &full[i]);
  }
  for (int i = threadIdx.x; i < 2 * kHeadDim; i += blockDim.x) {
    const uint16_t* w = i < kHeadDim ? a.qw : a.kw;
    s_w[i] = w != nullptr ? __uint_as_float(static_cast<uint32_t>(w[i & (kHeadDim - 1)]) << 16)
                          : 1.0f;
  }

  const Meta m{a.q_indptr, a.seq_lens, a.positions, a.flags, a.T, a.B,
               static_cast<int64_t>(a.max_pages) * a.page_size, a.cs_rows};
  if (stage_and_validate(m, s_indptr, s_seq)) {
    if (producer && lane == 0) {  // drain the copies issued before the verdict
      for (int i = 0; i < pre; ++i) {
        mbar_arrive(&full[i]);
        mbar_wait(&full[i], 0);
      }
    }
    return;
  }

  // tail rows per request (K then V), exclusive scan
  const int P = a.page_size;
  for (int b = threadIdx.x; b < a.B; b += blockDim.x) {
    const int L = s_seq[b];
    s_tail[b] = L > 0 ? 2 * (P - 1 - (L - 1) % P) : 0;
  }
  __syncthreads();
  block_exclusive_scan(s_tail, a.B, s_scan);

  if (producer) {
    produce(a, stages, full, empty, s_indptr, s_seq, u0, nunits, pre);
  } else {
    zero_tails(a, s_seq, s_tail);
    consume<POLICY, STYLE>(a, stages, full, empty, s_w, u0, nunits);
  }
}

using AppendKernel = void (*)(const PipeArgs);

static AppendKernel select_append(int policy, int style) {
  if (style == 0) {
    if (policy == 0) return append_kernel<0, 0>;
    if (policy == 1) return append_kernel<1, 0>;
    return append_kernel<2, 0>;
  }
  if (policy == 0) return append_kernel<0, 1>;
  if (policy == 1) return append_kernel<1, 1>;
  return append_kernel<2, 1>;
}

int launch_append(const fqr_append_params& p, cudaStream_t stream) {
  PipeArgs a;
  const int esize = p.quant_policy == 0 ? 2 : 1;
  a.qkv = p.qkv;
  a.row_stride = p.qkv_row_stride;
  a.T = p.T; a.B = p.B; a.Hq = p.Hq; a.Hkv = p.Hkv;
  a.H = p.Hq + 2 * p.Hkv;
  a.qw = p.q_norm_w; a.kw = p.k_norm_w; a.eps = p.eps;
  a.cs = p.cos_sin_cache; a.cs_rows = p.cos_sin_rows; a.rot = p.rot_dim;
  a.cs_bulk = (p.rot_dim * 4) % 16 == 0 ? 1 : 0;
  a.cs_bytes = a.cs_bulk ? p.rot_dim * 4 : 0;
  a.positions = p.positions;
  a.q_indptr = p.q_indptr; a.seq_lens = p.seq_lens; a.page_table = p.page_table;
  a.max_pages = p.max_pages;
  a.k_cache = static_cast<char*>(p.k_cache);
  a.v_cache = static_cast<char*>(p.v_cache);
  a.page_size = p.page_size;
  a.row_bytes = p.Hkv * kHeadDim * esize;
  a.k_page_bytes = p.k_page_stride * esize;
  a.v_page_bytes = p.v_page_stride * esize;
  a.q_scale_inv = p.q_scale_inv; a.k_scale = p.k_scale; a.v_scale = p.v_scale;
  a.upper_max = p.upper_max;
  a.out_q = p.out_q; a.q_scale = p.q_scale; a.flags = p.flags;

  int dev = 0, sms = 0, smem_optin = 0, smem_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
          cudaSuccess)
    return FQR_ECUDA;

  const int64_t meta = static_cast<int64_t>(3 * p.B + 2) * sizeof(int);
  auto stage_bytes = [&](int hc) { return 16 + a.cs_bytes + hc * kHeadDim * 2; };
  // a row that does not fit two stages beside the metadata is split into
  // chunks of whole quads
  int hc = a.H;
  while (hc > 4 && kFixedSmem + meta + 2 * stage_bytes(hc) > smem_optin) hc = ((hc / 2 + 3) / 4) * 4;
  if (kFixedSmem + meta + stage_bytes(hc) > smem_optin) return FQR_ENOTSUP;
  a.chunk_heads = hc;
  a.nchunks = (a.H + hc - 1) / hc;
  a.units = static_cast<int64_t>(p.T) * a.nchunks;
  a.stage_bytes = stage_bytes(hc);
  // pipeline depth: aim at two resident blocks per SM, never deeper than the
  // units a block will see
  const int64_t per_block_budget = smem_sm / 2 - 1024;
  int S = static_cast<int>((per_block_budget - kFixedSmem - meta) / a.stage_bytes);
  S = S < 1 ? 1 : (S > kMaxStages ? kMaxStages : S);
  const int64_t upb = (a.units + 2 * sms - 1) / (2 * sms);
  if (upb >= 1 && S > upb) S = static_cast<int>(upb);
  while (S > 1 && kFixedSmem + meta + static_cast<int64_t>(S) * a.stage_bytes > smem_optin) --S;
  a.stages = S;
  const size_t smem = static_cast<size_t>(kFixedSmem + meta + static_cast<int64_t>(S) * a.stage_bytes);

  AppendKernel k = select_append(p.quant_policy, p.rope_style);
  const void* fn = reinterpret_cast<const void*>(k);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return FQR_ECUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kPipeThreads, smem) !=
          cudaSuccess ||
      per_sm < 1)
    return FQR_ECUDA;
  const int64_t cap = static_cast<int64_t>(per_sm) * sms;
  const int64_t want = a.units > sms ? a.units : sms;
  const int grid = static_cast<int>(want < cap ? want : cap);
  k<<<grid, kPipeThreads, smem, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? FQR_OK : FQR_ECUDA;
}

}  // namespace fqr
