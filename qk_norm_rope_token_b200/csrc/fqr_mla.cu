// fqr_mla.cu -- MLA variant: RoPE on the rope part of Q (in place) and the
// latent-cache write [kv_c | rope(k_pe)] (FP8 E4M3 with a per-tensor scale, or
// BF16), one launch.
//
// Method: vLLM issue #24678 ("ROPE + KV-Cache-Write + pre-attn prepare-ops
// fusion": concat_and_cache_mla fused with RoPE; DeepSeek R1 model table:
// 64 qk_rope dims, RoPE/NoPE interleaved), with the slot, position and
// device-side validation rules of the FlashInfer PR #5956 "Contract".
//
// Tasks (persistent grid, one warp each):
//   * latent tasks (one per packed row): 32 lanes stream kv_c in 16-byte
//     vectors; 8 lanes rotate k_pe; the encoded row goes to its block slot.
//   * Q tasks (one per row and 4 heads): 8 lanes per head, each holding
//     elements [4l, 4l+4) and [32+4l, 32+4l+4) of the 64 rope dims, which
//     covers the NeoX pairs (i, i+32) and the GPT-J pairs (2i, 2i+1) alike.
// With Q quantisation the 8 lanes of a head also hold its nope part in
// 16-byte chunks: static and per-head scales keep the warp tasks
// (mla_quant_kernel); per-token scales give a thread-block cluster of
// kTokenCluster blocks a whole row of Q at a time (mla_token_kernel), its
// maximum reduced over the cluster (distributed shared memory) before any
// payload store.
#include <cooperative_groups.h>

#include "fqr_head.cuh"
#include "fqr_launch.h"

namespace fqr {

constexpr int kRope = 64;

struct MlaArgs {
  uint16_t* q;
  int64_t q_tok, q_head;
  int T, B, Hq, nope, qgroups;
  const uint16_t* kv_c;
  int rank;
  int64_t kv_c_stride;
  const uint16_t* k_pe;
  int64_t k_pe_stride;
  const float* cs;
  int cs_rows;
  const int64_t* positions;
  const int32_t* q_indptr;
  const int32_t* seq_lens;
  const int32_t* block_table;
  int max_blocks;
  char* latent;
  int block_size;
  int64_t row_bytes;
  const float* kv_scale;
  int32_t* flags;
  int q_quant;
  const float* q_scale_inv;
  float upper_max;
  unsigned char* q_out;
  float* q_scale;
  int q_ng;      // per-group Q scales: groups per head, ceil((nope + 64) / q_group)
  FastDiv gdiv;  // division by q_group
};

__device__ __forceinline__ uint2 ld_v2(const void* p) {
  uint2 r;
  asm volatile("ld.global.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}

// cos/sin for this lane's 4 pairs; element layout A = [4l, 4l+4), B = [32+4l, ...)
template <int STYLE>
__device__ __forceinline__ void mla_cos_sin(const float* row, int l, float* c, float* s) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    // NeoX: pair j is (A_j, B_j), index 4l + j.  GPT-J: pairs (A0,A1), (A2,A3),
    // (B0,B1), (B2,B3) with indices 2l, 2l+1, 16+2l, 16+2l+1.
    const int i = STYLE == 0 ? 4 * l + j : (j < 2 ? 2 * l + j : 16 + 2 * l + (j - 2));
    c[j] = __ldg(row + i);
    s[j] = __ldg(row + kRope / 2 + i);
  }
}

template <int STYLE>
__device__ __forceinline__ void mla_rotate(float* y /* A[0..4) B[4..8) */, const float* c,
                                           const float* s) {
  if (STYLE == 0) {
#pragma unroll
    for (int j = 0; j < 4; ++j) rotate_pair(y[j], y[4 + j], c[j], s[j]);
  } else {
    rotate_pair(y[0], y[1], c[0], s[0]);
    rotate_pair(y[2], y[3], c[1], s[1]);
    rotate_pair(y[4], y[5], c[2], s[2]);
    rotate_pair(y[6], y[7], c[3], s[3]);
  }
}

// E4M3 latent payloads x / kv_scale for 8 values: the guarded Markstein
// division of fqr_head.cuh (divide_pairs: codes equal to IEEE division's).
__device__ __forceinline__ void divide8(float* y, float d) {
  float2 v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) v[j] = make_float2(y[2 * j], y[2 * j + 1]);
  divide_pairs<4>(v, d);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    y[2 * j] = v[j].x;
    y[2 * j + 1] = v[j].y;
  }
}

// A latent row's inputs as one lane holds them: kv_c chunks lane + 32 k
// (8 elements each; kLatentChunks in registers, any further ones are loaded
// when stored) and, for lanes < 8, the k_pe elements [4l, 4l+4) and
// [32+4l, 32+4l+4).
constexpr int kLatentChunks = 2;  // kv_lora_rank 512
struct LatentIn {
  uint4 kv[kLatentChunks];
  uint2 pe0, pe1;
};

__device__ __forceinline__ void load_latent(const MlaArgs& a, int t, int lane, LatentIn& in) {
  const uint16_t* kc = a.kv_c + static_cast<int64_t>(t) * a.kv_c_stride;
#pragma unroll
  for (int k = 0; k < kLatentChunks; ++k)
    if (lane + 32 * k < a.rank / 8) in.kv[k] = ld_stream_v4(kc + 8 * (lane + 32 * k));
  if (lane < kRope / 8) {
    const uint16_t* kp = a.k_pe + static_cast<int64_t>(t) * a.k_pe_stride;
    in.pe0 = ld_stream_v2(kp + 4 * lane);
    in.pe1 = ld_stream_v2(kp + kRope / 2 + 4 * lane);
  }
}

// Latent row of packed row t (request b, slot position p_slot) from `in`:
// the encoded row goes to its block slot.
template <int FP8, int STYLE>
__device__ __forceinline__ void store_latent(const MlaArgs& a, int t, int b, int p_slot,
                                             const float* row, int lane, const LatentIn& in) {
  const int64_t blk =
      __ldg(a.block_table + static_cast<int64_t>(b) * a.max_blocks + p_slot / a.block_size);
  char* dst = a.latent + (blk * a.block_size + p_slot % a.block_size) * a.row_bytes;
  const uint16_t* kc = a.kv_c + static_cast<int64_t>(t) * a.kv_c_stride;
  const float sc = FP8 ? __ldg(a.kv_scale) : 1.0f;
  for (int k = 0, c8 = lane; c8 < a.rank / 8; ++k, c8 += 32) {
    uint4 v;
    if (k < kLatentChunks) {
#pragma unroll
      for (int j = 0; j < kLatentChunks; ++j)
        if (j == k) v = in.kv[j];
    } else {
      v = ld_stream_v4(kc + 8 * c8);
    }
    if (FP8) {
      float y[8];
      unpack8(v, y);
      divide8(y, sc);
      st_v2(dst + 8 * c8, pack8_e4m3(y));
    } else {
      st_v4(dst + 16 * c8, v);
    }
  }
  if (lane < kRope / 8) {
    float y[8], c[4], s[4];
    unpack4(in.pe0, y);
    unpack4(in.pe1, y + 4);
    mla_cos_sin<STYLE>(row, lane, c, s);
    mla_rotate<STYLE>(y, c, s);
    const int64_t e0 = a.rank + 4 * lane, e1 = a.rank + kRope / 2 + 4 * lane;
    if (FP8) {
      divide8(y, sc);
      st_u32(dst + e0, pack4_e4m3(y));
      st_u32(dst + e1, pack4_e4m3(y + 4));
    } else {
      st_v2(dst + 2 * e0, pack4_bf16(y));
      st_v2(dst + 2 * e1, pack4_bf16(y + 4));
    }
  }
}

template <int FP8, int STYLE>
__device__ __forceinline__ void latent_row(const MlaArgs& a, int t, int b, int p_slot,
                                           const float* row, int lane) {
  LatentIn in;
  load_latent(a, t, lane, in);
  store_latent<FP8, STYLE>(a, t, b, p_slot, row, lane, in);
}

// Before griddepcontrol.wait: pull into L2 the metadata lines and the inputs
// of this warp's first task (latent row: kv_c and k_pe; Q quad: the rows of
// its heads' rope part), one prefetch per 128-byte line.  L2 is the point of
// coherence, so the reads after the wait still see the preceding grid's
// writes.
// Then, from a possibly stale read of the task's own request metadata (L2
// only: the values only steer prefetches, and a later load cannot hit a
// stale L1 line; the request is guessed as b = t, one row per request), the
// block-table entry and the cos/sin row of that row.
__device__ __forceinline__ void mla_prefetch(const MlaArgs& a, int64_t gwarp, int lane) {
  const int tid = threadIdx.x;
  if (32 * tid <= a.B) {
    prefetch_l2(a.q_indptr + 32 * tid);
    if (32 * tid < a.B) prefetch_l2(a.seq_lens + 32 * tid);
  }
  int64_t t = -1;
  if (gwarp < a.T) {
    t = gwarp;
    const uint16_t* kc = a.kv_c + gwarp * a.kv_c_stride;
    for (int l = lane; l < a.rank / 64; l += 32) prefetch_l2(kc + 64 * l);
    if (lane == 0) prefetch_l2(a.k_pe + gwarp * a.k_pe_stride);
  } else if (gwarp < a.T + static_cast<int64_t>(a.T) * a.qgroups) {
    const int64_t qw = gwarp - a.T;
    t = qw / a.qgroups;
    const int h = static_cast<int>(qw - t * a.qgroups) * 4 + lane;
    if (lane < 4 && h < a.Hq) prefetch_l2(a.q + t * a.q_tok + h * a.q_head + a.nope);
  }
  if (t < 0) return;  // (warp-uniform)
  const int gb = t < a.B - 1 ? static_cast<int>(t) : a.B - 1;
  int lo = 0, hi = 0, L = 0;
  int64_t ps = 0;
  if (lane == 0) {
    lo = ld_cg_s32(a.q_indptr + gb);
    hi = ld_cg_s32(a.q_indptr + gb + 1);
    L = ld_cg_s32(a.seq_lens + gb);
    if (a.positions != nullptr) ps = ld_cg_s64(a.positions + t);
  }
  lo = __shfl_sync(0xffffffffu, lo, 0);
  hi = __shfl_sync(0xffffffffu, hi, 0);
  L = __shfl_sync(0xffffffffu, L, 0);
  ps = __shfl_sync(0xffffffffu, ps, 0);
  if (lo <= t && t < hi) {
    const int64_t p = t + L - hi;
    const int64_t pos = a.positions != nullptr ? ps : p;
    if (p >= 0 && p < static_cast<int64_t>(a.max_blocks) * a.block_size && pos >= 0 &&
        pos < a.cs_rows) {
      if (lane == 0 && gwarp < a.T)
        prefetch_l2(a.block_table + static_cast<int64_t>(gb) * a.max_blocks + p / a.block_size);
      if (lane == 1 || lane == 2) prefetch_l2(a.cs + pos * kRope + 32 * (lane - 1));
    }
  }
}

template <int FP8, int STYLE>
__global__ void __launch_bounds__(kThreads) mla_kernel(const MlaArgs a) {
  extern __shared__ int smem[];
  int* s_indptr = smem;
  int* s_seq = s_indptr + a.B + 1;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 3, l8 = lane & 7;
  const int64_t gwarp = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;

  mla_prefetch(a, gwarp, lane);
  grid_dependency_wait();
  grid_launch_dependents();

  // the first task's inputs need no metadata: load them before the
  // validation prologue (a latent row, or this group's head of a Q quad)
  const int64_t n_lat = a.T;
  const int64_t n_tasks = n_lat + static_cast<int64_t>(a.T) * a.qgroups;
  LatentIn in0;
  uint2 q0a = make_uint2(0u, 0u), q0b = q0a;
  if (gwarp < n_lat) {
    load_latent(a, static_cast<int>(gwarp), lane, in0);
  } else if (gwarp < n_tasks) {
    const int64_t qw = gwarp - n_lat;
    const int64_t t = qw / a.qgroups;
    const int h = static_cast<int>(qw - t * a.qgroups) * 4 + g;
    if (h < a.Hq) {
      const uint16_t* qp = a.q + t * a.q_tok + h * a.q_head + a.nope;
      q0a = ld_v2(qp + 4 * l8);
      q0b = ld_v2(qp + kRope / 2 + 4 * l8);
    }
  }

  const Meta m{a.q_indptr, a.seq_lens, a.positions, a.flags, a.T, a.B,
               static_cast<int64_t>(a.max_blocks) * a.block_size, a.cs_rows};
  if (stage_and_validate(m, s_indptr, s_seq)) return;

  for (int64_t w = gwarp; w < n_tasks; w += nwarps) {
    const bool lat = w < n_lat;
    const int64_t qw = w - n_lat;
    const int t = lat ? static_cast<int>(w) : static_cast<int>(qw / a.qgroups);
    const int b = request_of_row(s_indptr, a.B, t);
    const int p_slot = t + s_seq[b] - s_indptr[b + 1];
    const int64_t pos = a.positions != nullptr ? a.positions[t] : static_cast<int64_t>(p_slot);
    const float* row = a.cs + pos * kRope;

    if (lat) {
      if (w == gwarp)
        store_latent<FP8, STYLE>(a, t, b, p_slot, row, lane, in0);
      else
        latent_row<FP8, STYLE>(a, t, b, p_slot, row, lane);
    } else {
      const int h = static_cast<int>(qw - static_cast<int64_t>(t) * a.qgroups) * 4 + g;
      if (h < a.Hq) {
        uint16_t* qp = a.q + static_cast<int64_t>(t) * a.q_tok + h * a.q_head + a.nope;
        float y[8], c[4], s[4];
        unpack4(w == gwarp ? q0a : ld_v2(qp + 4 * l8), y);
        unpack4(w == gwarp ? q0b : ld_v2(qp + kRope / 2 + 4 * l8), y + 4);
        mla_cos_sin<STYLE>(row, l8, c, s);
        mla_rotate<STYLE>(y, c, s);
        st_v2(qp + 4 * l8, pack4_bf16(y));
        st_v2(qp + kRope / 2 + 4 * l8, pack4_bf16(y + 4));
      }
    }
  }
}

using MlaKernel = void (*)(const MlaArgs);

// ---------------------------------------------------------------- Q FP8 --

// E4M3 codes of 8 values: x * qsi (static) or x / sc with rc = 1 / sc
// (dynamic, |x / sc| <= upper_max: div2_bounded, see fqr_head.cuh).
template <int QMODE>
__device__ __forceinline__ void quantize8(float* x, float qsi, float sc, float rc) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float2 v = make_float2(x[2 * j], x[2 * j + 1]);
    v = QMODE == FQR_MLA_Q_STATIC ? mul2(v, make_float2(qsi, qsi))
                                  : div2_bounded(v, make_float2(sc, sc), make_float2(rc, rc));
    x[2 * j] = v.x;
    x[2 * j + 1] = v.y;
  }
}

// The rope part of the head at qp, rotated: y[0..4) = elements [4 l8, 4 l8 + 4),
// y[4..8) = [32 + 4 l8, ...) of the 64 rope dims.
template <int STYLE>
__device__ __forceinline__ void rope_part(const uint16_t* qp, int nope, int l8, const float* c,
                                          const float* s, float* y) {
  unpack4(ld_stream_v2(qp + nope + 4 * l8), y);
  unpack4(ld_stream_v2(qp + nope + kRope / 2 + 4 * l8), y + 4);
  mla_rotate<STYLE>(y, c, s);
}

// Quantisation of head h = quad*4 + g of packed row t (Q FP8).  The lane
// holds the head's nope chunks l8, l8 + 8, ... (8 elements each, kept as
// packed bf16: at most kMaxChunks) and its rotated rope part y.
constexpr int kMaxChunks = 4;  // nope_dim <= 256

struct QHead {
  uint4 nope[kMaxChunks];
  float y[8];
};

template <int STYLE>
__device__ __forceinline__ void load_q_head(const uint16_t* qp, int nope, int l8, const float* c,
                                            const float* s, QHead& v) {
#pragma unroll
  for (int k = 0; k < kMaxChunks; ++k)
    if (l8 + 8 * k < nope / 8) v.nope[k] = ld_stream_v4(qp + 8 * (l8 + 8 * k));
  rope_part<STYLE>(qp, nope, l8, c, s, v.y);
}

__device__ __forceinline__ float q_head_amax(const QHead& v, int nope, int l8) {
  float m = 0.0f;
#pragma unroll
  for (int k = 0; k < 8; ++k) m = fmaxf(m, fabsf(v.y[k]));
#pragma unroll
  for (int k = 0; k < kMaxChunks; ++k) {
    if (l8 + 8 * k < nope / 8) {
      float x[8];
      unpack8(v.nope[k], x);
#pragma unroll
      for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(x[j]));
    }
  }
  return m;
}

template <int QMODE>
__device__ __forceinline__ void store_q_head(QHead& v, unsigned char* op, int nope, int l8,
                                             float qsi, float sc, float rc) {
#pragma unroll
  for (int k = 0; k < kMaxChunks; ++k) {
    const int c = l8 + 8 * k;
    if (c < nope / 8) {
      float x[8];
      unpack8(v.nope[k], x);
      quantize8<QMODE>(x, qsi, sc, rc);
      st_v2(op + 8 * c, pack8_e4m3(x));
    }
  }
  quantize8<QMODE>(v.y, qsi, sc, rc);
  st_u32(op + nope + 4 * l8, pack4_e4m3(v.y));
  st_u32(op + nope + kRope / 2 + 4 * l8, pack4_e4m3(v.y + 4));
}

// Per-group scales (FQR_MLA_Q_GROUP): groups of q_group consecutive values of
// a head's v = [nope | rope(rope part)].  Each of the lane's runs -- its nope
// chunks l8 + 8k (8 values) and its two 4-value rope runs -- lies inside one
// group: q_group is a multiple of 8, nope a multiple of 8, and every run
// starts on a multiple of 4 inside an 8-aligned block.  The groups' maxima
// are reduced one group at a time over the head's 8 lanes; lane k % 8 stores
// the scale of group k.
constexpr int kRuns = kMaxChunks + 2;
struct RunScales {
  float sc[kRuns], rc[kRuns];
};

__device__ __forceinline__ void group_scales(const MlaArgs& a, const QHead& v, int l8,
                                             unsigned gmask, float* qs, RunScales& rs) {
  float m[kRuns];
  int grp[kRuns];
#pragma unroll
  for (int k = 0; k < kMaxChunks; ++k) {
    const int c = l8 + 8 * k;
    m[k] = 0.0f;
    grp[k] = -1;
    if (c < a.nope / 8) {
      float x[8];
      unpack8(v.nope[k], x);
#pragma unroll
      for (int j = 0; j < 8; ++j) m[k] = fmaxf(m[k], fabsf(x[j]));
      grp[k] = static_cast<int>(a.gdiv.div(static_cast<uint32_t>(8 * c)));
    }
  }
  m[kMaxChunks] = fmaxf(fmaxf(fabsf(v.y[0]), fabsf(v.y[1])), fmaxf(fabsf(v.y[2]), fabsf(v.y[3])));
  m[kMaxChunks + 1] =
      fmaxf(fmaxf(fabsf(v.y[4]), fabsf(v.y[5])), fmaxf(fabsf(v.y[6]), fabsf(v.y[7])));
  grp[kMaxChunks] = static_cast<int>(a.gdiv.div(static_cast<uint32_t>(a.nope + 4 * l8)));
  grp[kMaxChunks + 1] =
      static_cast<int>(a.gdiv.div(static_cast<uint32_t>(a.nope + kRope / 2 + 4 * l8)));
#pragma unroll
  for (int r = 0; r < kRuns; ++r) rs.sc[r] = 1.0f;
  for (int k = 0; k < a.q_ng; ++k) {
    float mk = 0.0f;
#pragma unroll
    for (int r = 0; r < kRuns; ++r)
      if (grp[r] == k) mk = fmaxf(mk, m[r]);
    mk = fmaxf(mk, __shfl_xor_sync(gmask, mk, 4));
    mk = fmaxf(mk, __shfl_xor_sync(gmask, mk, 2));
    mk = fmaxf(mk, __shfl_xor_sync(gmask, mk, 1));
    const float sk = __fdiv_rn(fmaxf(mk, 1e-6f), a.upper_max);
    if (l8 == (k & 7)) qs[k] = sk;
#pragma unroll
    for (int r = 0; r < kRuns; ++r)
      if (grp[r] == k) rs.sc[r] = sk;
  }
#pragma unroll
  for (int r = 0; r < kRuns; ++r) rs.rc[r] = __frcp_rn(rs.sc[r]);
}

// E4M3 codes of n values x / sc (|x / sc| <= upper_max: div2_bounded).
template <int N>
__device__ __forceinline__ void quantize_dyn(float* x, float sc, float rc) {
#pragma unroll
  for (int j = 0; j < N / 2; ++j) {
    const float2 q = div2_bounded(make_float2(x[2 * j], x[2 * j + 1]), make_float2(sc, sc),
                                  make_float2(rc, rc));
    x[2 * j] = q.x;
    x[2 * j + 1] = q.y;
  }
}

__device__ __forceinline__ void store_q_head_groups(QHead& v, unsigned char* op, int nope, int l8,
                                                    const RunScales& rs) {
#pragma unroll
  for (int k = 0; k < kMaxChunks; ++k) {
    const int c = l8 + 8 * k;
    if (c < nope / 8) {
      float x[8];
      unpack8(v.nope[k], x);
      quantize_dyn<8>(x, rs.sc[k], rs.rc[k]);
      st_v2(op + 8 * c, pack8_e4m3(x));
    }
  }
  quantize_dyn<4>(v.y, rs.sc[kMaxChunks], rs.rc[kMaxChunks]);
  quantize_dyn<4>(v.y + 4, rs.sc[kMaxChunks + 1], rs.rc[kMaxChunks + 1]);
  st_u32(op + nope + 4 * l8, pack4_e4m3(v.y));
  st_u32(op + nope + kRope / 2 + 4 * l8, pack4_e4m3(v.y + 4));
}

// Static, per-head and per-group scales: persistent warp tasks
// [latent rows | row x quad].
template <int QMODE, int FP8, int STYLE>
__global__ void __launch_bounds__(kThreads) mla_quant_kernel(const MlaArgs a) {
  extern __shared__ int smem[];
  int* s_indptr = smem;
  int* s_seq = s_indptr + a.B + 1;
  const int lane = threadIdx.x & 31;
  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x >> 5), 0);
  const int g = lane >> 3, l8 = lane & 7;
  const unsigned gmask = 0xFFu << (8 * g);
  const int64_t gwarp = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;

  mla_prefetch(a, gwarp, lane);
  grid_dependency_wait();
  grid_launch_dependents();
  const Meta m{a.q_indptr, a.seq_lens, a.positions, a.flags, a.T, a.B,
               static_cast<int64_t>(a.max_blocks) * a.block_size, a.cs_rows};
  if (stage_and_validate(m, s_indptr, s_seq)) return;

  const int W = a.nope + kRope;
  const float qsi = QMODE == FQR_MLA_Q_STATIC ? __ldg(a.q_scale_inv) : 0.0f;
  const int64_t n_tasks = a.T + static_cast<int64_t>(a.T) * a.qgroups;
  for (int64_t w = gwarp; w < n_tasks; w += nwarps) {
    const bool lat = w < a.T;
    const int64_t qw = w - a.T;
    const int t = lat ? static_cast<int>(w) : static_cast<int>(qw / a.qgroups);
    const int b = request_of_row(s_indptr, a.B, t);
    const int p_slot = t + s_seq[b] - s_indptr[b + 1];
    const int64_t pos = a.positions != nullptr ? a.positions[t] : static_cast<int64_t>(p_slot);
    const float* row = a.cs + pos * kRope;
    if (lat) {
      latent_row<FP8, STYLE>(a, t, b, p_slot, row, lane);
      continue;
    }
    const int h = static_cast<int>(qw - static_cast<int64_t>(t) * a.qgroups) * 4 + g;
    if (h >= a.Hq) continue;  // (the whole group)
    float c[4], s[4];
    mla_cos_sin<STYLE>(row, l8, c, s);
    QHead v;
    load_q_head<STYLE>(a.q + static_cast<int64_t>(t) * a.q_tok + static_cast<int64_t>(h) * a.q_head,
                       a.nope, l8, c, s, v);
    if (QMODE == FQR_MLA_Q_GROUP) {
      RunScales rs;
      group_scales(a, v, l8, gmask,
                   a.q_scale + (static_cast<int64_t>(t) * a.Hq + h) * a.q_ng, rs);
      store_q_head_groups(v, a.q_out + (static_cast<int64_t>(t) * a.Hq + h) * W, a.nope, l8, rs);
      continue;
    }
    float sc = 0.0f, rc = 0.0f;
    if (QMODE == FQR_MLA_Q_HEAD) {
      float mx = q_head_amax(v, a.nope, l8);
      mx = fmaxf(mx, __shfl_xor_sync(gmask, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(gmask, mx, 2));
      mx = fmaxf(mx, __shfl_xor_sync(gmask, mx, 1));
      sc = __fdiv_rn(fmaxf(mx, 1e-6f), a.upper_max);
      rc = __frcp_rn(sc);
      if (l8 == 0) a.q_scale[static_cast<int64_t>(t) * a.Hq + h] = sc;
    }
    store_q_head<QMODE>(v, a.q_out + (static_cast<int64_t>(t) * a.Hq + h) * W, a.nope, l8, qsi,
                        sc, rc);
  }
}

// Per-token scales: a thread-block cluster of kTokenCluster blocks per row of
// Q at a time.  The row's quads are spread over the cluster's warps (block r
// takes quads r * nw + warp, then + kTokenCluster * nw, ...; each warp keeps
// its first quad in registers and reads any further ones again for the
// payloads).  The row's maximum is reduced over each warp (shuffles), each
// block (shared memory) and the cluster: every block reads its peers'
// partial maxima from their shared memory (distributed shared memory, after
// a cluster barrier), so no global memory and no second kernel is involved.
// The latent rows are warp tasks spread over the clusters.
constexpr int kTokenWarps = 16;   // warps per block at most
constexpr int kTokenCluster = 4;  // blocks per cluster (one row of Q)

template <int FP8, int STYLE>
__global__ void __launch_bounds__(kTokenWarps * 32) mla_token_kernel(const MlaArgs a) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ int smem[];
  int* s_indptr = smem;
  int* s_seq = s_indptr + a.B + 1;
  float* s_red = reinterpret_cast<float*>(s_seq + a.B);  // one float per warp, then the block's
  const int lane = threadIdx.x & 31;
  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x >> 5), 0);
  const int nw = blockDim.x >> 5;
  const int g = lane >> 3, l8 = lane & 7;
  const int crank = static_cast<int>(cluster.block_rank());
  const int cid = blockIdx.x / kTokenCluster;       // this block's cluster
  const int ncl = gridDim.x / kTokenCluster;        // clusters in the grid
  const int cw = crank * nw + warp;                 // warp index inside the cluster
  const int cwarps = kTokenCluster * nw;
  // latent rows: warp task pw, pw + (all warps), ... with the warps ordered
  // cluster-minor, so that consecutive rows go to different clusters
  const int pw = cw * ncl + cid;
  const int nwarps = gridDim.x * nw;

  // before the wait: metadata, this warp's first latent row and this block's
  // quads of the cluster's first row of Q into L2 (see mla_prefetch)
  mla_prefetch(a, pw < a.T ? pw : INT64_MAX, lane);
  if (cid < a.T) {
    const uint16_t* qrow = a.q + static_cast<int64_t>(cid) * a.q_tok;
    const int h = (crank * nw + warp) * 4 + lane;
    if (lane < 4 && h < a.Hq) {
      const uint16_t* hp = qrow + static_cast<int64_t>(h) * a.q_head;
      for (int e = 0; e < a.nope + kRope; e += 64) prefetch_l2(hp + e);
    }
  }
  grid_dependency_wait();
  grid_launch_dependents();
  const Meta m{a.q_indptr, a.seq_lens, a.positions, a.flags, a.T, a.B,
               static_cast<int64_t>(a.max_blocks) * a.block_size, a.cs_rows};
  // (every block of every cluster reaches the same verdict: a malformed batch
  // returns them all before any cluster barrier)
  if (stage_and_validate(m, s_indptr, s_seq)) return;

  for (int t = pw; t < a.T; t += nwarps) {  // latent rows
    const int b = request_of_row(s_indptr, a.B, t);
    const int p_slot = t + s_seq[b] - s_indptr[b + 1];
    const int64_t pos = a.positions != nullptr ? a.positions[t] : static_cast<int64_t>(p_slot);
    latent_row<FP8, STYLE>(a, t, b, p_slot, a.cs + pos * kRope, lane);
  }
  const int W = a.nope + kRope;
  for (int t = cid; t < a.T; t += ncl) {  // Q rows (cluster-uniform loop)
    const int b = request_of_row(s_indptr, a.B, t);
    const int p_slot = t + s_seq[b] - s_indptr[b + 1];
    const int64_t pos = a.positions != nullptr ? a.positions[t] : static_cast<int64_t>(p_slot);
    float c[4], s[4];
    mla_cos_sin<STYLE>(a.cs + pos * kRope, l8, c, s);
    const uint16_t* qrow = a.q + static_cast<int64_t>(t) * a.q_tok;
    // pass 1: the maximum over this warp's quads
    const int hA = cw * 4 + g;
    const bool okA = hA < a.Hq;  // (group-uniform)
    QHead va;
    if (okA) load_q_head<STYLE>(qrow + static_cast<int64_t>(hA) * a.q_head, a.nope, l8, c, s, va);
    float mx = okA ? q_head_amax(va, a.nope, l8) : 0.0f;
    for (int h = hA + 4 * cwarps; h - g < a.Hq; h += 4 * cwarps) {
      if (h < a.Hq) {
        QHead v;
        load_q_head<STYLE>(qrow + static_cast<int64_t>(h) * a.q_head, a.nope, l8, c, s, v);
        mx = fmaxf(mx, q_head_amax(v, a.nope, l8));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) s_red[warp] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
      float bm = s_red[0];
      for (int i = 1; i < nw; ++i) bm = fmaxf(bm, s_red[i]);
      s_red[nw] = bm;
    }
    cluster.sync();  // every block's partial maximum is in its shared memory
    mx = 0.0f;
#pragma unroll
    for (int r = 0; r < kTokenCluster; ++r) mx = fmaxf(mx, *cluster.map_shared_rank(s_red + nw, r));
    cluster.sync();  // read everywhere before any block reuses s_red or exits
    const float sc = __fdiv_rn(fmaxf(mx, 1e-6f), a.upper_max);
    const float rc = __frcp_rn(sc);
    if (crank == 0 && threadIdx.x == 0) a.q_scale[t] = sc;
    // pass 2: payloads
    unsigned char* orow = a.q_out + static_cast<int64_t>(t) * a.Hq * W;
    if (okA) store_q_head<FQR_MLA_Q_TOKEN>(va, orow + static_cast<int64_t>(hA) * W, a.nope, l8, 0.0f, sc, rc);
    for (int h = hA + 4 * cwarps; h - g < a.Hq; h += 4 * cwarps) {
      if (h < a.Hq) {
        QHead v;
        load_q_head<STYLE>(qrow + static_cast<int64_t>(h) * a.q_head, a.nope, l8, c, s, v);
        store_q_head<FQR_MLA_Q_TOKEN>(v, orow + static_cast<int64_t>(h) * W, a.nope, l8, 0.0f, sc, rc);
      }
    }
  }
}

template <int QMODE>
static MlaKernel select_quant(int fp8, int style) {
  if (fp8) return style == 0 ? mla_quant_kernel<QMODE, 1, 0> : mla_quant_kernel<QMODE, 1, 1>;
  return style == 0 ? mla_quant_kernel<QMODE, 0, 0> : mla_quant_kernel<QMODE, 0, 1>;
}



int launch_mla(const fqr_mla_params& p, cudaStream_t stream) {
  MlaArgs a;
  a.q = p.q; a.q_tok = p.q_token_stride; a.q_head = p.q_head_stride;
  a.T = p.T; a.B = p.B; a.Hq = p.Hq; a.nope = p.nope_dim;
  a.qgroups = (p.Hq + 3) / 4;
  a.kv_c = p.kv_c; a.rank = p.kv_lora_rank; a.kv_c_stride = p.kv_c_stride;
  a.k_pe = p.k_pe; a.k_pe_stride = p.k_pe_stride;
  a.cs = p.cos_sin_cache; a.cs_rows = p.cos_sin_rows;
  a.positions = p.positions; a.q_indptr = p.q_indptr; a.seq_lens = p.seq_lens;
  a.block_table = p.block_table; a.max_blocks = p.max_blocks;
  a.latent = static_cast<char*>(p.latent_cache);
  a.block_size = p.block_size;
  a.row_bytes = static_cast<int64_t>(p.kv_lora_rank + p.rope_dim) * (p.cache_fp8 ? 1 : 2);
  a.kv_scale = p.kv_scale; a.flags = p.flags;
  a.q_quant = p.q_quant; a.q_scale_inv = p.q_scale_inv; a.upper_max = p.upper_max;
  a.q_out = static_cast<unsigned char*>(p.q_out); a.q_scale = p.q_scale;
  a.q_ng = 1;
  if (p.q_quant == FQR_MLA_Q_GROUP) {
    const int W = p.nope_dim + p.rope_dim;
    a.q_ng = (W + p.q_group - 1) / p.q_group;
    a.gdiv = FastDiv(static_cast<uint32_t>(p.q_group));
  }

  if (p.q_quant == FQR_MLA_Q_TOKEN) {
    MlaKernel k = p.cache_fp8 ? (p.rope_style == 0 ? mla_token_kernel<1, 0> : mla_token_kernel<1, 1>)
                              : (p.rope_style == 0 ? mla_token_kernel<0, 0> : mla_token_kernel<0, 1>);
    // warps per block: the row's quads spread over the cluster, one per warp
    // while they last (at most kTokenWarps)
    const int per_block = (a.qgroups + kTokenCluster - 1) / kTokenCluster;
    const int nw = per_block < kTokenWarps ? (per_block > 0 ? per_block : 1) : kTokenWarps;
    const size_t smem = static_cast<size_t>(2 * p.B + 1) * sizeof(int) + (nw + 1) * sizeof(float);
    DeviceInfo d;
    int per_sm = 0;
    if (device_info(&d) != FQR_OK ||
        resident_blocks(reinterpret_cast<const void*>(k), 32 * nw, smem, &per_sm) != FQR_OK)
      return FQR_ECUDA;
    // clusters: one per row, at most as many as fit on the device at once
    const int64_t cap = static_cast<int64_t>(per_sm) * d.sms / kTokenCluster;
    const int64_t want = p.T > 0 ? p.T : 1;
    const int clusters = static_cast<int>(want < cap ? want : (cap > 0 ? cap : 1));
    return launch_pdl(k, clusters * kTokenCluster, 32 * nw, smem, stream, a, kTokenCluster);
  }
  if (p.q_quant != FQR_MLA_Q_NONE) {
    MlaKernel k = p.q_quant == FQR_MLA_Q_STATIC ? select_quant<FQR_MLA_Q_STATIC>(p.cache_fp8, p.rope_style)
                  : p.q_quant == FQR_MLA_Q_GROUP ? select_quant<FQR_MLA_Q_GROUP>(p.cache_fp8, p.rope_style)
                                                 : select_quant<FQR_MLA_Q_HEAD>(p.cache_fp8, p.rope_style);
    const int64_t tasks = static_cast<int64_t>(p.T) * (1 + a.qgroups);
    const size_t smem = static_cast<size_t>(2 * p.B + 1) * sizeof(int);
    return launch_persistent(reinterpret_cast<const void*>(k), tasks, smem, stream,
                             [&](int grid) { return launch_pdl(k, grid, kThreads, smem, stream, a); });
  }
  MlaKernel k = p.cache_fp8 ? (p.rope_style == 0 ? mla_kernel<1, 0> : mla_kernel<1, 1>)
                            : (p.rope_style == 0 ? mla_kernel<0, 0> : mla_kernel<0, 1>);
  const int64_t tasks = static_cast<int64_t>(p.T) * (1 + a.qgroups);
  const size_t smem = static_cast<size_t>(2 * p.B + 1) * sizeof(int);
  return launch_persistent(reinterpret_cast<const void*>(k), tasks, smem, stream,
                           [&](int grid) { return launch_pdl(k, grid, kThreads, smem, stream, a); });
}

}  // namespace fqr
