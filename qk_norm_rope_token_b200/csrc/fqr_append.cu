// fqr_append.cu -- fused per-head Q/K RMSNorm + RoPE + (optional) FP8 E4M3
// quantisation + paged K/V append + last-page tail zeroing, one launch.
//
// Method: FlashInfer PR #5956 (fused QK RMSNorm + NeoX RoPE + FP8 E4M3
// quantize + NHD paged-KV append), section "Contract"; RMSNorm as in the
// TensorRT-LLM PR #16024 review excerpt; fp32 cos/sin cache RoPE as in SGLang
// PR #43425 "Modifications".
//
// Work decomposition (persistent grid, warp-granular tasks):
//   * head tasks: one warp handles 4 heads of one packed row; 8 lanes own a
//     head.  Lane l of a group loads elements [8l, 8l+8) and [64+8l, 64+8l+8)
//     with two 16-byte loads, so it holds both halves of its 8 NeoX pairs and
//     the rotation needs no shuffle.  The RMS reduction is a 3-step xor
//     shuffle inside the 8-lane group (group mask, never the whole warp).
//   * tail tasks: one warp zeroes up to 2 KiB of one request's last-page tail
//     in one cache with 16-byte stores; the tasks come from an exclusive scan
//     of per-request chunk counts, so no task is idle.
// Each block first validates the whole batch (see stage_and_validate): a
// malformed batch writes only the flags.
#include "fqr_device.cuh"
#include "fqr_launch.h"

namespace fqr {

struct AppendArgs {
  const uint16_t* qkv;
  int64_t row_stride;
  int T, B, Hq, Hkv, H, quads;
  const uint16_t* qw;
  const uint16_t* kw;
  float eps;
  const float* cs;
  int cs_rows, rot;
  const int64_t* positions;
  const int32_t* q_indptr;
  const int32_t* seq_lens;
  const int32_t* page_table;
  int max_pages;
  char* k_cache;
  char* v_cache;
  int page_size;
  int row_bytes;                  // Hkv * 128 * element size
  int64_t k_page_bytes, v_page_bytes;
  const float* q_scale_inv;
  const float* k_scale;
  const float* v_scale;
  float upper_max;
  void* out_q;
  float* q_scale;
  int32_t* flags;
};

// Packed-row data of head task w for this lane: 16 BF16 elements.
__device__ __forceinline__ void load_head(const AppendArgs& a, int64_t w, int g, int l8,
                                          uint4& xa, uint4& xb) {
  const int64_t t = w / a.quads;
  const int h = static_cast<int>(w - t * a.quads) * 4 + g;
  if (h < a.H) {
    const uint16_t* src = a.qkv + t * a.row_stride + static_cast<int64_t>(h) * kHeadDim + 8 * l8;
    xa = ld_stream_v4(src);
    xb = ld_stream_v4(src + 64);
  }
}

// cos/sin values this lane needs for its 8 pairs.
template <int STYLE>
__device__ __forceinline__ void load_cos_sin(const AppendArgs& a, int64_t pos, int l8,
                                             float* c, float* s) {
  const float* row = a.cs + pos * a.rot;
  if (STYLE == 0) {  // NeoX, rot == 128: pairs (8l+k, 64+8l+k)
    const float4 c0 = ld_shared_ro_f4(row + 8 * l8), c1 = ld_shared_ro_f4(row + 8 * l8 + 4);
    const float4 s0 = ld_shared_ro_f4(row + 64 + 8 * l8), s1 = ld_shared_ro_f4(row + 68 + 8 * l8);
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
      c[j] = on ? __ldg(row + i) : 1.0f;
      s[j] = on ? __ldg(row + half + i) : 0.0f;
    }
  }
}

template <int STYLE>
__device__ __forceinline__ void apply_rope(const AppendArgs& a, int l8, float* y,
                                           const float* c, const float* s) {
  if (STYLE == 0) {
#pragma unroll
    for (int k = 0; k < 8; ++k) rotate_pair(y[k], y[8 + k], c[k], s[k]);
  } else {
    const int half = a.rot >> 1;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = (j < 4 ? 4 * l8 + j : 32 + 4 * l8 + (j - 4));
      const int e = (j < 4 ? 2 * j : 8 + 2 * (j - 4));
      if (i < half) rotate_pair(y[e], y[e + 1], c[j], s[j]);
    }
  }
}

template <int POLICY, int STYLE>
__device__ __forceinline__ void head_task(const AppendArgs& a, int64_t w, int g, int l8,
                                          uint4 xa, uint4 xb, const int* s_indptr,
                                          const int* s_seq) {
  const int64_t t64 = w / a.quads;
  const int t = static_cast<int>(t64);
  const int h = static_cast<int>(w - t64 * a.quads) * 4 + g;
  if (h >= a.H) return;  // the whole 8-lane group leaves together
  const unsigned gmask = 0xFFu << (8 * g);

  const int b = request_of_row(s_indptr, a.B, t);
  const int p_slot = t + s_seq[b] - s_indptr[b + 1];
  const int P = a.page_size;

  float y[16];
  unpack8(xa, y);
  unpack8(xb, y + 8);

  if (h >= a.Hq + a.Hkv) {  // ---------------------------------- V head
    const int kh = h - a.Hq - a.Hkv;
    const int64_t page = __ldg(a.page_table + static_cast<int64_t>(b) * a.max_pages + p_slot / P);
    char* dst = a.v_cache + page * a.v_page_bytes +
                (static_cast<int64_t>(p_slot % P) * a.Hkv + kh) * kHeadDim * (POLICY == 0 ? 2 : 1);
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
  const int64_t pos = a.positions != nullptr ? a.positions[t] : static_cast<int64_t>(p_slot);
  int64_t page = 0;
  if (!is_q) page = __ldg(a.page_table + static_cast<int64_t>(b) * a.max_pages + p_slot / P);
  float c[8], s[8];
  load_cos_sin<STYLE>(a, pos, l8, c, s);

  // ----------------------------------------------------------- RMSNorm
  const uint16_t* wts = is_q ? a.qw : a.kw;
  if (wts != nullptr) {
    float ss = 0.0f;
#pragma unroll
    for (int k = 0; k < 16; ++k) ss = fmaf(y[k], y[k], ss);
    ss += __shfl_xor_sync(gmask, ss, 4);
    ss += __shfl_xor_sync(gmask, ss, 2);
    ss += __shfl_xor_sync(gmask, ss, 1);
    const float inv = __frcp_rn(__fsqrt_rn(__fadd_rn(ss * (1.0f / kHeadDim), a.eps)));
    const uint4 wa = __ldg(reinterpret_cast<const uint4*>(wts + 8 * l8));
    const uint4 wb = __ldg(reinterpret_cast<const uint4*>(wts + 64 + 8 * l8));
    float wv[16];
    unpack8(wa, wv);
    unpack8(wb, wv + 8);
#pragma unroll
    for (int k = 0; k < 16; ++k) y[k] = __fmul_rn(__fmul_rn(y[k], inv), wv[k]);
  }

  // -------------------------------------------------------------- RoPE
  apply_rope<STYLE>(a, l8, y, c, s);

  // ------------------------------------------------------------ output
  if (is_q) {
    const int64_t o = (t64 * a.Hq + h) * kHeadDim;
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
        if (l8 == 0) a.q_scale[t64 * a.Hq + h] = qs;
#pragma unroll
        for (int k = 0; k < 16; ++k) y[k] = __fdiv_rn(y[k], qs);
      } else {
        const float qsi = __ldg(a.q_scale_inv);
#pragma unroll
        for (int k = 0; k < 16; ++k) y[k] = __fmul_rn(y[k], qsi);
      }
      uint8_t* out = static_cast<uint8_t*>(a.out_q) + o;
      st_v2(out + 8 * l8, pack8_e4m3(y));
      st_v2(out + 64 + 8 * l8, pack8_e4m3(y + 8));
    }
  } else {
    const int kh = h - a.Hq;
    char* dst = a.k_cache + page * a.k_page_bytes +
                (static_cast<int64_t>(p_slot % P) * a.Hkv + kh) * kHeadDim * (POLICY == 0 ? 2 : 1);
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

// Zero one 2 KiB chunk of one request's last-page tail in one cache.
__device__ __forceinline__ void tail_task(const AppendArgs& a, int64_t k2, int lane,
                                          const int* s_seq, const int* s_tail) {
  const int which = static_cast<int>(k2 & 1);
  const int m = static_cast<int>(k2 >> 1);
  const int b = upper_bound(s_tail, a.B + 1, m) - 1;   // s_tail[b] <= m < s_tail[b+1]
  const int chunk = m - s_tail[b];
  const int L = s_seq[b];
  const int64_t P = a.page_size;
  const int64_t last = (L - 1) % P;
  const int64_t page = __ldg(a.page_table + static_cast<int64_t>(b) * a.max_pages + (L - 1) / P);
  char* base = which ? a.v_cache + page * a.v_page_bytes : a.k_cache + page * a.k_page_bytes;
  const int64_t start = (last + 1) * a.row_bytes + static_cast<int64_t>(chunk) * kTailChunkBytes;
  const int64_t span_end = P * a.row_bytes;
  const int64_t end = start + kTailChunkBytes < span_end ? start + kTailChunkBytes : span_end;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  for (int64_t off = start + 16 * lane; off < end; off += 512) st_v4(base + off, z);
}

template <int POLICY, int STYLE>
__global__ void __launch_bounds__(kThreads) append_kernel(const AppendArgs a) {
  extern __shared__ int smem[];
  __shared__ int s_warp[kWarps];
  int* s_indptr = smem;            // B + 1
  int* s_seq = s_indptr + a.B + 1; // B
  int* s_tail = s_seq + a.B;       // B + 1

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 3, l8 = lane & 7;
  const int64_t gwarp = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
  const int64_t n_head = static_cast<int64_t>(a.T) * a.quads;

  // The first task's packed-row loads need no metadata: issue them before
  // the validation prologue so the two latencies overlap.
  uint4 pa = make_uint4(0u, 0u, 0u, 0u), pb = pa;
  if (gwarp < n_head) load_head(a, gwarp, g, l8, pa, pb);

  const Meta m{a.q_indptr, a.seq_lens, a.positions, a.flags, a.T, a.B,
               static_cast<int64_t>(a.max_pages) * a.page_size, a.cs_rows};
  if (stage_and_validate(m, s_indptr, s_seq)) return;

  const int64_t P = a.page_size;
  for (int b = threadIdx.x; b < a.B; b += kThreads) {
    const int L = s_seq[b];
    int c = 0;
    if (L > 0) {
      const int64_t bytes = (P - 1 - (L - 1) % P) * a.row_bytes;
      c = static_cast<int>((bytes + kTailChunkBytes - 1) / kTailChunkBytes);
    }
    s_tail[b] = c;
  }
  __syncthreads();
  block_exclusive_scan(s_tail, a.B, s_warp);
  const int64_t n_tasks = n_head + 2 * static_cast<int64_t>(s_tail[a.B]);

  for (int64_t w = gwarp; w < n_tasks; w += nwarps) {
    if (w < n_head) {
      const uint4 xa = pa, xb = pb;
      if (w + nwarps < n_head) load_head(a, w + nwarps, g, l8, pa, pb);  // next task
      head_task<POLICY, STYLE>(a, w, g, l8, xa, xb, s_indptr, s_seq);
    } else {
      tail_task(a, w - n_head, lane, s_seq, s_tail);
    }
  }
}

using AppendKernel = void (*)(const AppendArgs);

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
  AppendArgs a;
  const int esize = p.quant_policy == 0 ? 2 : 1;
  a.qkv = p.qkv;
  a.row_stride = p.qkv_row_stride;
  a.T = p.T; a.B = p.B; a.Hq = p.Hq; a.Hkv = p.Hkv;
  a.H = p.Hq + 2 * p.Hkv;
  a.quads = (a.H + 3) / 4;
  a.qw = p.q_norm_w; a.kw = p.k_norm_w; a.eps = p.eps;
  a.cs = p.cos_sin_cache; a.cs_rows = p.cos_sin_rows; a.rot = p.rot_dim;
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

  const int64_t n_head = static_cast<int64_t>(p.T) * a.quads;
  const int64_t tail_per_cache =
      (static_cast<int64_t>(p.page_size - 1) * a.row_bytes + kTailChunkBytes - 1) / kTailChunkBytes;
  const int64_t tasks = n_head + 2 * static_cast<int64_t>(p.B) * tail_per_cache;
  const size_t smem = static_cast<size_t>(3 * p.B + 2) * sizeof(int);
  AppendKernel k = select_append(p.quant_policy, p.rope_style);
  return launch_persistent(reinterpret_cast<const void*>(k), tasks, smem, stream,
                           [&](int grid) { k<<<grid, kThreads, smem, stream>>>(a); });
}

}  // namespace fqr
