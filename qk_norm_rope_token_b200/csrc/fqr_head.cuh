// fqr_head.cuh -- the per-head arithmetic of the fused append, shared by both
// schedules (fqr_append_warp.cu, fqr_append_pipe.cu).
//
// One 8-lane group owns one 128-element head.  Lane l holds elements
// [8l, 8l+8) (chunk A) and [64+8l, 64+8l+8) (chunk B) as eight float2 pairs:
//   y[j]   = elements (8l+2j, 8l+2j+1)        j = 0..3
//   y[4+j] = elements (64+8l+2j, 64+8l+2j+1)  j = 0..3
// so a NeoX pair (i, i+64) sits in the same lane (y[j].x <-> y[4+j].x) and a
// GPT-J pair (2i, 2i+1) in the same float2.  All arithmetic is fp32 with every
// product and sum rounded on its own (sm_100 f32x2 instructions do two lanes
// of that at once); the reduction is an xor shuffle inside the group.
#pragma once

#include "fqr_device.cuh"

namespace fqr {

// Parameters the head arithmetic needs (a sub-struct of each schedule's args).
struct HeadParams {
  FastDiv pdiv;  // division by page_size
  int Hq, Hkv, page_size, row_bytes, rot;
  int has_qw, has_kw;
  float eps, upper_max;
  char* k_cache;
  char* v_cache;
  int64_t k_page_bytes, v_page_bytes;
  const float* q_scale_inv;
  const float* k_scale;
  const float* v_scale;
  void* out_q;
  float* q_scale;
  int gemma;       // the norm scales by 1 + w (Gemma-style) instead of w
  int qs_prefill;  // q_scale layout [B, Hq, qs_ld] (else [T, Hq])
  int qs_ld;       // round_up(max_seqlen, 128) for the prefill layout
  char* out_k;     // caller-owned K / V rows [T, Hkv, 128], or null: the paged caches
  char* out_v;
};

// q_scale index of head 0 of packed row t, the i-th row of request b (the
// head stride is 1 in the decode layout, qs_ld in the prefill layout).
__device__ __forceinline__ int q_scale_row(const HeadParams& a, int t, int b, int i) {
  return a.qs_prefill ? (b * a.Hq) * a.qs_ld + i : t * a.Hq;
}

// Where one packed row goes.
struct RowCtx {
  int t;         // packed row
  int slot_row;  // row of the KV slot inside its page (p_slot % page_size)
  int pos;       // RoPE position
  int page;      // page id of the KV slot (valid when the row has K/V heads to store)
  int is_last;   // the row is its request's last: its K/V heads also zero the tail
  int qs;        // q_scale index of head 0 (q_scale_row; dynamic Q only)
};

__device__ __forceinline__ float4 lds_f4(const float* p) {
  float4 r;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
               : "r"(smem_addr(p)));
  return r;
}
// cos/sin row reads: shared memory when the row was staged there, else the
// read-only path from global memory.
template <bool CS_SMEM>
__device__ __forceinline__ float4 ld_cs4(const float* p) {
  if (CS_SMEM) return lds_f4(p);
  return __ldg(reinterpret_cast<const float4*>(p));
}
template <bool CS_SMEM>
__device__ __forceinline__ float ld_cs1(const float* p) {
  if (CS_SMEM) {
    float r;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(r) : "r"(smem_addr(p)));
    return r;
  }
  return __ldg(p);
}

// Shared-memory layout of the fp32 norm weights, 128 per tensor: element e of
// lane l's slice is stored so that lane l reads its 16 values as four float4
// at 16-byte lane stride (conflict-free).
__device__ __forceinline__ int weight_slot(int e) {
  const int half = e >> 6, r = e & 63, l = r >> 3, k = r & 7;
  return half * 64 + (k >> 2) * 32 + 4 * l + (k & 3);
}

// Stage both weight vectors (fp32, permuted) in s_w[0, 256); NULL -> ones.
// For blocks of at least 256 threads: weight_prefetch loads one value per
// thread at kernel entry, weight_store writes it after the first round trip.
// gemma: the Gemma-style norm scales by 1 + w (an fp32 add) instead of w.
__device__ __forceinline__ float weight_value(const uint16_t* qw, const uint16_t* kw, int gemma,
                                              int i) {
  if (i >= 2 * kHeadDim) return 0.0f;
  const uint16_t* w = i < kHeadDim ? qw : kw;
  if (w == nullptr) return 1.0f;  // (the norm is off for this tensor)
  const float v = __uint_as_float(static_cast<uint32_t>(__ldg(w + (i & (kHeadDim - 1)))) << 16);
  return gemma ? __fadd_rn(1.0f, v) : v;
}
__device__ __forceinline__ void weight_store_at(float* s_w, float v, int i) {
  if (i < 2 * kHeadDim) s_w[(i & kHeadDim) + weight_slot(i & (kHeadDim - 1))] = v;
}
__device__ __forceinline__ float weight_prefetch(const uint16_t* qw, const uint16_t* kw,
                                                 int gemma) {
  return weight_value(qw, kw, gemma, threadIdx.x);
}
__device__ __forceinline__ void weight_store(float* s_w, float v) {
  weight_store_at(s_w, v, threadIdx.x);
}
// The same for blocks of NT threads: 256 / NT values per thread when NT < 256.
template <int NT>
struct WeightRegs {
  static constexpr int kN = NT >= 2 * kHeadDim ? 1 : 2 * kHeadDim / NT;
  float v[kN];
};
template <int NT>
__device__ __forceinline__ WeightRegs<NT> weight_prefetch_nt(const uint16_t* qw,
                                                             const uint16_t* kw, int gemma) {
  WeightRegs<NT> r;
#pragma unroll
  for (int k = 0; k < WeightRegs<NT>::kN; ++k)
    r.v[k] = weight_value(qw, kw, gemma, static_cast<int>(threadIdx.x) + k * NT);
  return r;
}
template <int NT>
__device__ __forceinline__ void weight_store_nt(float* s_w, const WeightRegs<NT>& r) {
#pragma unroll
  for (int k = 0; k < WeightRegs<NT>::kN; ++k)
    weight_store_at(s_w, r.v[k], static_cast<int>(threadIdx.x) + k * NT);
}

__device__ __forceinline__ void unpack_pairs(uint4 xa, uint4 xb, float2* y) {
  y[0] = make_float2(bf16_lo(xa.x), bf16_hi(xa.x));
  y[1] = make_float2(bf16_lo(xa.y), bf16_hi(xa.y));
  y[2] = make_float2(bf16_lo(xa.z), bf16_hi(xa.z));
  y[3] = make_float2(bf16_lo(xa.w), bf16_hi(xa.w));
  y[4] = make_float2(bf16_lo(xb.x), bf16_hi(xb.x));
  y[5] = make_float2(bf16_lo(xb.y), bf16_hi(xb.y));
  y[6] = make_float2(bf16_lo(xb.z), bf16_hi(xb.z));
  y[7] = make_float2(bf16_lo(xb.w), bf16_hi(xb.w));
}

// Norm-weight sources of the head arithmetic (load_weights): the block's
// staged fp32 copy (a `const float*` filled by weight_store), the lane's two
// 16-byte slices of the BF16 weight vector already in registers (RegWeights:
// wa = elements [8l, 8l+8), wb = [64+8l, 64+8l+8), loaded in a task's first
// round trip), or those slices read from global memory at the norm
// (GlobalWeights).  The last two need no block-wide staging.
struct RegWeights {
  uint4 wa, wb;
  int gemma;
};
struct GlobalWeights {
  const uint16_t* qw;
  const uint16_t* kw;
  int gemma;
};

__device__ __forceinline__ void load_weights(const float* s_w, bool is_q, int l8, float2* w) {
  const float* wv = s_w + (is_q ? 0 : kHeadDim) + 4 * l8;
  const float4 w0 = lds_f4(wv);
  const float4 w1 = lds_f4(wv + 32);
  const float4 w2 = lds_f4(wv + 64);
  const float4 w3 = lds_f4(wv + 96);
  w[0] = make_float2(w0.x, w0.y);
  w[1] = make_float2(w0.z, w0.w);
  w[2] = make_float2(w1.x, w1.y);
  w[3] = make_float2(w1.z, w1.w);
  w[4] = make_float2(w2.x, w2.y);
  w[5] = make_float2(w2.z, w2.w);
  w[6] = make_float2(w3.x, w3.y);
  w[7] = make_float2(w3.z, w3.w);
}
// BF16 slices -> the lane's 8 weight pairs; the Gemma-style norm scales by
// 1 + w, formed in fp32 exactly as weight_value forms it.
__device__ __forceinline__ void unpack_weights(uint4 wa, uint4 wb, int gemma, float2* w) {
  unpack_pairs(wa, wb, w);
  if (gemma) {
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = __fadd2_rn(make_float2(1.0f, 1.0f), w[j]);
  }
}
__device__ __forceinline__ void load_weights(const RegWeights& r, bool /*is_q*/, int /*l8*/,
                                             float2* w) {
  unpack_weights(r.wa, r.wb, r.gemma, w);
}
__device__ __forceinline__ void load_weights(const GlobalWeights& g, bool is_q, int l8,
                                             float2* w) {
  const uint16_t* src = is_q ? g.qw : g.kw;
  unpack_weights(__ldg(reinterpret_cast<const uint4*>(src + 8 * l8)),
                 __ldg(reinterpret_cast<const uint4*>(src + 64 + 8 * l8)), g.gemma, w);
}

__device__ __forceinline__ uint4 pack_bf16_pairs(const float2* y) {
  return make_uint4(pack_bf16x2(y[0].x, y[0].y), pack_bf16x2(y[1].x, y[1].y),
                    pack_bf16x2(y[2].x, y[2].y), pack_bf16x2(y[3].x, y[3].y));
}
__device__ __forceinline__ uint2 pack_e4m3_pairs(const float2* y) {
  return make_uint2(pack_e4m3x2(y[0].x, y[0].y) | (pack_e4m3x2(y[1].x, y[1].y) << 16),
                    pack_e4m3x2(y[2].x, y[2].y) | (pack_e4m3x2(y[3].x, y[3].y) << 16));
}

__device__ __forceinline__ float2 neg2(float2 v) { return make_float2(-v.x, -v.y); }

// a / b for the dynamic Q payload, where the divisor b = q_scale is used for a
// whole head and |a / b| <= upper_max <= 448 by construction.  Given
// r = __frcp_rn(b): one correction step of Markstein's method (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990): q0 = a r, e = a - b q0 (exact
// with an FMA), q = q0 + e r -- written as -(-e r - q0) so that a zero
// dividend keeps its sign.  Two lanes at once (f32x2).  Within that bounded
// domain the E4M3 code of the result equals the code of IEEE a / b for every
// a, and the quotient itself is bit-equal when a = +-0, or |a| >= 2^-100 and
// the quotient is not subnormal (the theorem assumes no underflow; a
// subnormal quotient encodes to a zero code either way).
// tests/test_gpu_division.py checks both over every binary32 dividend for a
// set of q_scale values and over 2^33 random pairs.  Outside the domain --
// |a / b| beyond the float range -- the correction is not used.
__device__ __forceinline__ float2 div2_bounded(float2 a, float2 b, float2 r) {
  const float2 q0 = mul2(a, r);
  const float2 e = fma2(neg2(q0), b, a);
  return neg2(fma2(neg2(e), r, neg2(q0)));
}

// K / V payloads: every value divided by d (k_scale or v_scale, one value for
// the whole call), then encoded to E4M3.  The lane's 2N quotients come from
// div2_bounded when the division cannot overflow or lose the exactness of the
// residual anywhere it matters -- 2^-80 <= d <= 2^80 and max|x| / d < 2^100
// -- which makes every E4M3 code equal to the code of the IEEE quotient
// (tests/test_gpu_division.py checks it over every binary32 dividend for a set
// of scales).  A negative scale would give a zero quotient the wrong sign in
// the correction; it, like any lane outside the guard, divides with __fdiv_rn.
template <int N = 8>
__device__ __forceinline__ void divide_pairs(float2* y, float d) {
  const float r = __frcp_rn(d);
  float m = 0.0f;
#pragma unroll
  for (int j = 0; j < N; ++j) m = fmaxf(m, fmaxf(fabsf(y[j].x), fabsf(y[j].y)));
  if (d >= 0x1p-80f && d <= 0x1p80f && m * r < 0x1p100f) {
    const float2 b2 = make_float2(d, d), r2 = make_float2(r, r);
#pragma unroll
    for (int j = 0; j < N; ++j) y[j] = div2_bounded(y[j], b2, r2);
  } else {
#pragma unroll
    for (int j = 0; j < N; ++j) y[j] = make_float2(__fdiv_rn(y[j].x, d), __fdiv_rn(y[j].y, d));
  }
}

// Store a head (16 values per lane) into a KV slot / out_q row at `dst`
// (the head's first byte): bf16 for policy 0, e4m3 otherwise.
template <int POLICY>
__device__ __forceinline__ void store_head(char* dst, const float2* y, int l8) {
  if (POLICY == 0) {
    st_v4(dst + 16 * l8, pack_bf16_pairs(y));
    st_v4(dst + 128 + 16 * l8, pack_bf16_pairs(y + 4));
  } else {
    st_v2(dst + 8 * l8, pack_e4m3_pairs(y));
    st_v2(dst + 64 + 8 * l8, pack_e4m3_pairs(y + 4));
  }
}

// A NeoX cos/sin row staged in shared memory is four 128-byte quarters
// (cos 0-31, cos 32-63, sin 0-31, sin 32-63), each followed by 16 bytes of
// padding: lane l8's 32-byte slice starts at quarter l8/4, byte 32*(l8%4),
// and the 8 lanes of a quarter-warp phase hit 8 distinct 16-byte bank groups.
constexpr int kCsPaddedBytes = 4 * (128 + 16);
__device__ __forceinline__ int cs_padded_slice(int l8) { return (l8 >> 2) * 36 + (l8 & 3) * 8; }

// The cos/sin values lane l8 needs for its 8 pairs: NeoX (rot 128) pairs
// (8l+k, 64+8l+k); GPT-J pairs 4l+j (chunk A) and 32+4l+j (chunk B), with
// c = s = 0 outside the rotated dims (those pairs are not rotated).  A NeoX
// row in shared memory (CS_SMEM) has the padded layout above; a GPT-J one is
// contiguous.
template <int STYLE, bool CS_SMEM>
__device__ __forceinline__ void load_cs(const float* cs_row, int rot, int l8, float2* c,
                                        float2* s) {
  if (STYLE == 0) {
    const int i0 = CS_SMEM ? cs_padded_slice(l8) : 8 * l8;  // cos slice
    const int is = CS_SMEM ? 72 : 64;                        // sin: two quarters on
    const float4 c0 = ld_cs4<CS_SMEM>(cs_row + i0);
    const float4 c1 = ld_cs4<CS_SMEM>(cs_row + i0 + 4);
    const float4 s0 = ld_cs4<CS_SMEM>(cs_row + is + i0);
    const float4 s1 = ld_cs4<CS_SMEM>(cs_row + is + i0 + 4);
    c[0] = make_float2(c0.x, c0.y); c[1] = make_float2(c0.z, c0.w);
    c[2] = make_float2(c1.x, c1.y); c[3] = make_float2(c1.z, c1.w);
    s[0] = make_float2(s0.x, s0.y); s[1] = make_float2(s0.z, s0.w);
    s[2] = make_float2(s1.x, s1.y); s[3] = make_float2(s1.z, s1.w);
  } else {
    const int half = rot >> 1;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int ia = 4 * l8 + j, ib = 32 + 4 * l8 + j;
      c[j].x = ia < half ? ld_cs1<CS_SMEM>(cs_row + ia) : 0.0f;
      s[j].x = ia < half ? ld_cs1<CS_SMEM>(cs_row + half + ia) : 0.0f;
      c[j].y = ib < half ? ld_cs1<CS_SMEM>(cs_row + ib) : 0.0f;
      s[j].y = ib < half ? ld_cs1<CS_SMEM>(cs_row + half + ib) : 0.0f;
    }
  }
}

// Zero share `part` of `parts` (pdiv divides by parts) of a request's tail
// rows [last+1, P) in both caches -- the K span, then the V span, in 16-byte
// units -- so that all the warps of the request's last row split it evenly.
__device__ __forceinline__ void zero_tail_share(const HeadParams& a, int page, int last,
                                                uint32_t part, const FastDiv& pdiv, int lane) {
  const uint32_t span = static_cast<uint32_t>(a.page_size - 1 - last) * a.row_bytes;  // per cache
  const uint32_t units = span / 8;                                                  // 2 * span / 16
  const uint32_t u0 = pdiv.div(units * part), u1 = pdiv.div(units * (part + 1));
  const int64_t beg = static_cast<int64_t>(last + 1) * a.row_bytes;
  char* kb = a.k_cache + static_cast<int64_t>(page) * a.k_page_bytes + beg;
  char* vb = a.v_cache + static_cast<int64_t>(page) * a.v_page_bytes + beg;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  for (uint32_t u = u0 + lane; u < u1; u += 32) {
    const uint32_t o = u * 16;
    st_v4(o < span ? kb + o : vb + (o - span), z);
  }
}

// The same share written by the TMA engine: lane 0 issues bulk copies from a
// block-wide buffer of kZeroBytes zero bytes in shared memory (filled, and
// fenced for the async proxy, before the block's first barrier) and commits
// them as one bulk async-group; the issuing thread must bulk_wait_all()
// before the block exits.  Returns whether this thread issued any copy.
// The warp is then free for its next task while the zeros stream out, which
// pays off when a warp has several tasks or large shares.
constexpr uint32_t kZeroBytes = 2048;
__device__ __forceinline__ bool zero_tail_share_bulk(const HeadParams& a, int page, int last,
                                                     uint32_t part, const FastDiv& pdiv, int lane,
                                                     const void* zbuf) {
  const uint32_t span = static_cast<uint32_t>(a.page_size - 1 - last) * a.row_bytes;
  const uint32_t units = span / 8;
  const uint32_t u0 = pdiv.div(units * part), u1 = pdiv.div(units * (part + 1));
  if (lane != 0 || u1 <= u0) return false;
  const uint32_t o0 = u0 * 16, o1 = u1 * 16;  // byte range of [K span | V span]
  const int64_t beg = static_cast<int64_t>(last + 1) * a.row_bytes;
  char* kb = a.k_cache + static_cast<int64_t>(page) * a.k_page_bytes + beg;
  char* vb = a.v_cache + static_cast<int64_t>(page) * a.v_page_bytes + beg;
  if (o0 < span) {
    const uint32_t e = o1 < span ? o1 : span;
    for (uint32_t x = o0; x < e; x += kZeroBytes) bulk_s2g(kb + x, zbuf, min(kZeroBytes, e - x));
  }
  if (o1 > span) {
    const uint32_t b = (o0 > span ? o0 : span) - span, e = o1 - span;
    for (uint32_t x = b; x < e; x += kZeroBytes) bulk_s2g(vb + x, zbuf, min(kZeroBytes, e - x));
  }
  bulk_commit();
  return true;
}

// Fill the block's zero buffer (kZeroBytes, 16-byte aligned) and order the
// writes before the bulk copies that read it; a block barrier must follow.
__device__ __forceinline__ void zero_buffer_init(unsigned char* zbuf) {
  for (uint32_t i = threadIdx.x; i < kZeroBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(zbuf)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
}

// What the 4 heads of a quad are, when the whole quad is known to be of one
// kind (a warp-uniform value, so the per-head code has no divergent branch
// on the head type); kAnyHead decides per head.
enum HeadKind { kAnyHead = 0, kQHead = 1, kKHead = 2, kVHead = 3 };

// Kind of heads [h0, h0 + 4) (all of them exist).
__device__ __forceinline__ int quad_kind(const HeadParams& a, int h0) {
  const int qk = a.Hq + a.Hkv;
  if (h0 + 4 <= a.Hq) return kQHead;
  if (h0 >= a.Hq && h0 + 4 <= qk) return kKHead;
  if (h0 >= qk) return kVHead;
  return kAnyHead;
}

// The mean square of the head whose lane slices (8 float2 pairs) are y, over
// the 8-lane group gmask: each value converted to binary64 by the hardware,
// squared and summed there, then rounded once to fp32.  Valid for every input
// (an Inf or a NaN propagates as in the definition); the slow path of
// inv_rms_n.
__device__ __forceinline__ float mean_square_general(const float2* y, unsigned gmask) {
  double ss = 0.0;  // (one chain: a rare path, kept to few registers)
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const double u = y[j].x;
    ss = fma(u, u, ss);
    const double v = y[j].y;
    ss = fma(v, v, ss);
  }
  ss += __shfl_xor_sync(gmask, ss, 4);
  ss += __shfl_xor_sync(gmask, ss, 2);
  ss += __shfl_xor_sync(gmask, ss, 1);
  return __double2float_rn(ss * (1.0 / kHeadDim));
}

// How inv_rms_n forms the binary64 squares (both exact, see there):
// kSumMixed takes fewer instructions (for throughput-bound kernels), kSumShort
// has the shorter dependency chain (for a warp that holds a single task).
enum SumForm { kSumMixed = 0, kSumShort = 1 };

// 1 / sqrt(mean(x^2) + eps) of N heads whose lane slices (8 float2 pairs each,
// BF16 values) are y, over the 8-lane group gmask.  The mean square is the
// fp32 rounding of the exact mean of the squares: a BF16 value has 8
// significant bits, its square 16, and the binary64 sum of a head's 128
// squares is exact whenever its nonzero magnitudes span at most 2^15 -- so no
// summation order (four lane chains, then the group's xor tree) can change
// it.  One rounding to fp32, then +eps, the square root and the reciprocal,
// each correctly rounded (rn_recip_sqrt).
//
// kSumMixed: the values go to binary64 by two conversions, to balance the
// pipes -- the first value of each pair by the hardware conversion, the
// second by integer operations on its fp32 bits u: for a BF16 value (8
// significant bits) the binary64 high word is ((u >> 3) & 0x0FFFFFFF) +
// ((1023 - 127) << 20) with a zero low word (the sign is dropped: only the
// square is used).  That is exact for every finite nonzero normal value; a
// zero or subnormal becomes a value below 2^-126, whose square cannot reach
// the fp32 rounding of any mean square that does not itself round to zero;
// an Inf becomes 2^128, as good as infinite here (the mean square overflows,
// 1/sqrt gives 0); only a NaN would turn finite, so when the mean square
// overflows, the head's values are checked for a NaN (a rare branch), which
// then makes the result NaN.
//
// kSumShort: the squares are formed in fp32 (exact for |x| in [2^-63, 2^64):
// 16 significant bits, no overflow or underflow) and moved to binary64 by a
// shift: the binary32 pattern of a non-negative p shifted right by 3 is the
// high word of the binary64 value p * 2^-896 (the exponent fields line up,
// without the bias difference; zero and subnormal patterns too) with a low
// word of p's three lowest bits -- zero for such an exact square, so the low
// word is left zero (a smaller, rounded square loses bits below 2^-146).  The
// sum is scaled back by 2^889 (2^896 over the 128 values), exactly.  A mean square outside [2^-60, 2^121) (which any
// |x| >= 2^64, an Inf or a NaN puts above, and only heads of tiny values
// below) is recomputed by mean_square_general on a rare branch: inside that
// range every value below 2^-63 is too small to reach the fp32 rounding of
// the exact mean wherever the span condition above holds.
template <int N, int FORM = kSumMixed>
__device__ __forceinline__ void inv_rms_n(float2 (*y)[8], float eps, unsigned gmask, float* inv) {
  double ss[N];
#pragma unroll
  for (int n = 0; n < N; ++n) {
    double s[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      double u, v;
      if (FORM == kSumMixed) {
        u = y[n][j].x;
        v = __hiloint2double(
            static_cast<int>(__umulhi(__float_as_uint(y[n][j].y) & 0x7FFF0000u, 1u << 29) +
                             0x38000000u),
            0);
        s[(j & 1) * 2] = fma(u, u, s[(j & 1) * 2]);
        s[(j & 1) * 2 + 1] = fma(v, v, s[(j & 1) * 2 + 1]);
      } else {
        const float2 p = mul2(y[n][j], y[n][j]);
        u = __hiloint2double(static_cast<int>(__float_as_uint(p.x) >> 3), 0);
        v = __hiloint2double(static_cast<int>(__float_as_uint(p.y) >> 3), 0);
        s[(j & 1) * 2] += u;
        s[(j & 1) * 2 + 1] += v;
      }
    }
    ss[n] = (s[0] + s[1]) + (s[2] + s[3]);
  }
#pragma unroll
  for (int m = 4; m >= 1; m >>= 1) {
#pragma unroll
    for (int n = 0; n < N; ++n) ss[n] += __shfl_xor_sync(gmask, ss[n], m);
  }
#pragma unroll
  for (int n = 0; n < N; ++n) {
    float ms;
    if (FORM == kSumMixed) {
      ms = __double2float_rn(ss[n] * (1.0 / kHeadDim));
      if (__builtin_expect(ms == INFINITY, 0)) {  // the whole 8-lane group agrees on ms
        bool nan = false;
#pragma unroll
        for (int j = 0; j < 8; ++j) nan |= isnan(y[n][j].x) || isnan(y[n][j].y);
        if (__any_sync(gmask, nan)) ms = __int_as_float(0x7FC00000);
      }
    } else {
      ms = __double2float_rn(ss[n] * 0x1p889);
      // ms in [2^-60, 2^121) as one unsigned compare of the bit patterns; the
      // whole 8-lane group agrees on ms
      if (__builtin_expect(__float_as_uint(ms) - 0x21800000u >= 0x7C000000u - 0x21800000u, 0))
        ms = mean_square_general(y[n], gmask);
    }
    inv[n] = rn_recip_sqrt(__fadd_rn(ms, eps));
  }
}
__device__ __forceinline__ float inv_rms(float2* y, float eps, unsigned gmask) {
  float inv;
  inv_rms_n<1>(reinterpret_cast<float2(*)[8]>(y), eps, gmask, &inv);
  return inv;
}

// The RoPE of one head's lane slices y with the lane's cos/sin values c, s
// (NeoX: pairs (i, i + 64) across the two chunks; GPT-J: pairs (2i, 2i + 1)
// inside a float2, dims >= rot passing through).
template <int STYLE>
__device__ __forceinline__ void rope_head(float2* y, const float2* c, const float2* s, int rot,
                                          int l8) {
  if (STYLE == 0) {
#pragma unroll
    for (int j = 0; j < 4; ++j) rotate_pairs2(y[j], y[4 + j], c[j], s[j]);
  } else {  // dims >= rot_dim pass through untouched
    const int half = rot >> 1;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (4 * l8 + j < half) rotate_pair(y[j].x, y[j].y, c[j].x, s[j].x);
      if (32 + 4 * l8 + j < half) rotate_pair(y[4 + j].x, y[4 + j].y, c[j].y, s[j].y);
    }
  }
}

// Quantisation and store of a normed and rotated Q head (out_q) or K head (its
// KV slot, or row r of the caller-owned K output).
template <int POLICY, int KIND>
__device__ __forceinline__ void output_qk_head(const HeadParams& a, const RowCtx& r, int h,
                                               float2* y, int l8, unsigned gmask) {
  constexpr int ES = POLICY == 0 ? 2 : 1;
  if (KIND == kQHead) {
    char* dst = static_cast<char*>(a.out_q) +
                (static_cast<int64_t>(r.t) * a.Hq + h) * kHeadDim * ES;
    if (POLICY == 1) {
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fmaxf(fabsf(y[j].x), fabsf(y[j].y)));
      amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, 4));
      amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, 2));
      amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, 1));
      const float qs = __fdiv_rn(fmaxf(amax, 1e-6f), a.upper_max);
      if (l8 == 0) a.q_scale[r.qs + static_cast<int64_t>(h) * (a.qs_prefill ? a.qs_ld : 1)] = qs;
      const float rq = __frcp_rn(qs);
      const float2 b2 = make_float2(qs, qs), r2 = make_float2(rq, rq);
#pragma unroll
      for (int j = 0; j < 8; ++j) y[j] = div2_bounded(y[j], b2, r2);
    } else if (POLICY == 2) {
      const float qsi = __ldg(a.q_scale_inv);
      const float2 qv = make_float2(qsi, qsi);
#pragma unroll
      for (int j = 0; j < 8; ++j) y[j] = mul2(y[j], qv);
    }
    store_head<POLICY>(dst, y, l8);
  } else {
    const int kh = h - a.Hq;
    char* page_base = a.k_cache + static_cast<int64_t>(r.page) * a.k_page_bytes;
    char* dst = a.out_k != nullptr
                    ? a.out_k + (static_cast<int64_t>(r.t) * a.Hkv + kh) * kHeadDim * ES
                    : page_base + r.slot_row * a.row_bytes + kh * kHeadDim * ES;
    if (POLICY != 0) divide_pairs(y, __ldg(a.k_scale));
    store_head<POLICY>(dst, y, l8);
  }
}

// Norm + RoPE + output of N heads h[0..N) of one kind (KIND: kQHead or
// kKHead) of row r at once, from their lane slices y (unpacked): the heads'
// dependency chains interleave, and they share the cos/sin values and the
// norm weights.
template <int POLICY, int STYLE, int KIND, int N, int FORM, class W>
__device__ __forceinline__ void process_qk_heads(const HeadParams& a, const RowCtx& r, const int* h,
                                                 float2 (*y)[8], const float2* c, const float2* s,
                                                 const W& wts, int l8, unsigned gmask) {
  if (KIND == kQHead ? a.has_qw : a.has_kw) {
    float inv[N];
    inv_rms_n<N, FORM>(y, a.eps, gmask, inv);
    float2 w[8];
    load_weights(wts, KIND == kQHead, l8, w);
#pragma unroll
    for (int n = 0; n < N; ++n) {
      const float2 iv = make_float2(inv[n], inv[n]);
#pragma unroll
      for (int j = 0; j < 8; ++j) y[n][j] = mul2(mul2(y[n][j], iv), w[j]);
    }
  }
#pragma unroll
  for (int n = 0; n < N; ++n) rope_head<STYLE>(y[n], c, s, a.rot, l8);
#pragma unroll
  for (int n = 0; n < N; ++n) output_qk_head<POLICY, KIND>(a, r, h[n], y[n], l8, gmask);
}

// Norm + RoPE + quantisation + store of head h of row r.  xa/xb: the lane's two
// 16-byte slices of the packed head; cs_row: the row's fp32 [cos | sin]
// (shared or global memory); wts: the norm weights (load_weights).  gmask:
// the 8-lane group.  KIND: the head's kind when the caller knows it
// (HeadKind).  Request tails are zeroed by the callers (zero_tail_share), not
// here.
template <int POLICY, int STYLE, int KIND = kAnyHead, int FORM = kSumMixed, class W>
__device__ __forceinline__ void process_head_cs(const HeadParams& a, const RowCtx& r, int h,
                                                uint4 xa, uint4 xb, const float2* c,
                                                const float2* s, const W& wts, int l8,
                                                unsigned gmask) {
  constexpr int ES = POLICY == 0 ? 2 : 1;
  float2 y[8];
  unpack_pairs(xa, xb, y);

  const bool is_v = KIND == kVHead || (KIND == kAnyHead && h >= a.Hq + a.Hkv);
  if (is_v) {  // -------------------------------------------------------- V
    const int kh = h - a.Hq - a.Hkv;
    char* page_base = a.v_cache + static_cast<int64_t>(r.page) * a.v_page_bytes;
    char* dst = a.out_v != nullptr
                    ? a.out_v + (static_cast<int64_t>(r.t) * a.Hkv + kh) * kHeadDim * ES
                    : page_base + r.slot_row * a.row_bytes + kh * kHeadDim * ES;
    if (POLICY == 0) {  // bit copy
      st_v4(dst + 16 * l8, xa);
      st_v4(dst + 128 + 16 * l8, xb);
    } else {
      divide_pairs(y, __ldg(a.v_scale));
      store_head<POLICY>(dst, y, l8);
    }
    return;
  }

  if constexpr (KIND != kVHead) {
    float2 yy[1][8];
#pragma unroll
    for (int j = 0; j < 8; ++j) yy[0][j] = y[j];
    const bool is_q = KIND == kQHead || (KIND == kAnyHead && h < a.Hq);
    if (is_q)
      process_qk_heads<POLICY, STYLE, kQHead, 1, FORM>(a, r, &h, yy, c, s, wts, l8, gmask);
    else
      process_qk_heads<POLICY, STYLE, kKHead, 1, FORM>(a, r, &h, yy, c, s, wts, l8, gmask);
  }
}

// As process_head_cs, loading the cos/sin values from cs_row first (V heads
// need none).
template <int POLICY, int STYLE, bool CS_SMEM, int KIND = kAnyHead, int FORM = kSumMixed,
          class W>
__device__ __forceinline__ void process_head(const HeadParams& a, const RowCtx& r, int h,
                                             uint4 xa, uint4 xb, const float* cs_row,
                                             const W& wts, int l8, unsigned gmask) {
  float2 c[4], s[4];
  if (KIND == kQHead || KIND == kKHead || (KIND == kAnyHead && h < a.Hq + a.Hkv))
    load_cs<STYLE, CS_SMEM>(cs_row, a.rot, l8, c, s);
  process_head_cs<POLICY, STYLE, KIND, FORM>(a, r, h, xa, xb, c, s, wts, l8, gmask);
}

// process_head_cs for one quad whose first head is h0 (warp-uniform), with
// the cos/sin values already loaded; see process_quad.
template <int POLICY, int STYLE, int FORM = kSumMixed, class W>
__device__ __forceinline__ void process_quad_cs(const HeadParams& a, const RowCtx& r, int h0,
                                                int nheads, int g, uint4 xa, uint4 xb,
                                                const float2* c, const float2* s, const W& wts,
                                                int l8, unsigned gmask) {
  const int h = h0 + g;
  const int kind = h0 + 4 <= nheads ? quad_kind(a, h0) : kAnyHead;
  if (kind == kQHead)
    process_head_cs<POLICY, STYLE, kQHead, FORM>(a, r, h, xa, xb, c, s, wts, l8, gmask);
  else if (kind == kKHead)
    process_head_cs<POLICY, STYLE, kKHead, FORM>(a, r, h, xa, xb, c, s, wts, l8, gmask);
  else if (kind == kVHead)
    process_head_cs<POLICY, STYLE, kVHead, FORM>(a, r, h, xa, xb, c, s, wts, l8, gmask);
  else if (h < nheads)
    process_head_cs<POLICY, STYLE, kAnyHead, FORM>(a, r, h, xa, xb, c, s, wts, l8, gmask);
}

// process_head for one quad whose first head is h0 (warp-uniform): the kind
// is decided once for the warp when all four heads exist; otherwise each
// group decides for its own head (h0 + g < nheads).
template <int POLICY, int STYLE, bool CS_SMEM, int FORM = kSumMixed, class W>
__device__ __forceinline__ void process_quad(const HeadParams& a, const RowCtx& r, int h0,
                                             int nheads, int g, uint4 xa, uint4 xb,
                                             const float* cs_row, const W& wts, int l8,
                                             unsigned gmask) {
  const int h = h0 + g;
  const int kind = h0 + 4 <= nheads ? quad_kind(a, h0) : kAnyHead;
  if (kind == kQHead)
    process_head<POLICY, STYLE, CS_SMEM, kQHead, FORM>(a, r, h, xa, xb, cs_row, wts, l8, gmask);
  else if (kind == kKHead)
    process_head<POLICY, STYLE, CS_SMEM, kKHead, FORM>(a, r, h, xa, xb, cs_row, wts, l8, gmask);
  else if (kind == kVHead)
    process_head<POLICY, STYLE, CS_SMEM, kVHead, FORM>(a, r, h, xa, xb, cs_row, wts, l8, gmask);
  else if (h < nheads)
    process_head<POLICY, STYLE, CS_SMEM, kAnyHead, FORM>(a, r, h, xa, xb, cs_row, wts, l8, gmask);
}

// Zero the whole tail (rows [last+1, P), all heads) of request b's last page in
// both caches: used for requests that append no token in this call.
template <int ES>
__device__ __forceinline__ void zero_request_tail(const HeadParams& a, const int32_t* page_table,
                                                  int max_pages, int b, int L, int lane) {
  const int P = a.page_size;
  const uint32_t pidx = a.pdiv.div(static_cast<uint32_t>(L - 1));
  const int last = L - 1 - static_cast<int>(pidx) * P;
  const int64_t page = __ldg(page_table + static_cast<int64_t>(b) * max_pages + pidx);
  const int64_t beg = static_cast<int64_t>(last + 1) * a.row_bytes;
  const int64_t end = static_cast<int64_t>(P) * a.row_bytes;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  char* kb = a.k_cache + page * a.k_page_bytes;
  char* vb = a.v_cache + page * a.v_page_bytes;
  for (int64_t off = beg + 16 * lane; off < end; off += 512) {
    st_v4(kb + off, z);
    st_v4(vb + off, z);
  }
}

}  // namespace fqr
