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
#include "fqr_device.cuh"
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

template <int FP8, int STYLE>
__global__ void __launch_bounds__(kThreads) mla_kernel(const MlaArgs a) {
  extern __shared__ int smem[];
  int* s_indptr = smem;
  int* s_seq = s_indptr + a.B + 1;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 3, l8 = lane & 7;
  const int64_t gwarp = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;

  grid_dependency_wait();
  grid_launch_dependents();
  const Meta m{a.q_indptr, a.seq_lens, a.positions, a.flags, a.T, a.B,
               static_cast<int64_t>(a.max_blocks) * a.block_size, a.cs_rows};
  if (stage_and_validate(m, s_indptr, s_seq)) return;

  const int64_t n_lat = a.T;
  const int64_t n_tasks = n_lat + static_cast<int64_t>(a.T) * a.qgroups;
  for (int64_t w = gwarp; w < n_tasks; w += nwarps) {
    const bool lat = w < n_lat;
    const int64_t qw = w - n_lat;
    const int t = lat ? static_cast<int>(w) : static_cast<int>(qw / a.qgroups);
    const int b = request_of_row(s_indptr, a.B, t);
    const int p_slot = t + s_seq[b] - s_indptr[b + 1];
    const int64_t pos = a.positions != nullptr ? a.positions[t] : static_cast<int64_t>(p_slot);
    const float* row = a.cs + pos * kRope;

    if (lat) {
      const int64_t blk =
          __ldg(a.block_table + static_cast<int64_t>(b) * a.max_blocks + p_slot / a.block_size);
      char* dst = a.latent + (blk * a.block_size + p_slot % a.block_size) * a.row_bytes;
      const uint16_t* kc = a.kv_c + static_cast<int64_t>(t) * a.kv_c_stride;
      const float sc = FP8 ? __ldg(a.kv_scale) : 1.0f;
      for (int c8 = lane; c8 < a.rank / 8; c8 += 32) {
        const uint4 v = ld_stream_v4(kc + 8 * c8);
        if (FP8) {
          float y[8];
          unpack8(v, y);
#pragma unroll
          for (int k = 0; k < 8; ++k) y[k] = __fdiv_rn(y[k], sc);
          st_v2(dst + 8 * c8, pack8_e4m3(y));
        } else {
          st_v4(dst + 16 * c8, v);
        }
      }
      if (lane < kRope / 8) {
        const uint16_t* kp = a.k_pe + static_cast<int64_t>(t) * a.k_pe_stride;
        float y[8], c[4], s[4];
        unpack4(ld_stream_v2(kp + 4 * lane), y);
        unpack4(ld_stream_v2(kp + kRope / 2 + 4 * lane), y + 4);
        mla_cos_sin<STYLE>(row, lane, c, s);
        mla_rotate<STYLE>(y, c, s);
        const int64_t e0 = a.rank + 4 * lane, e1 = a.rank + kRope / 2 + 4 * lane;
        if (FP8) {
#pragma unroll
          for (int k = 0; k < 8; ++k) y[k] = __fdiv_rn(y[k], sc);
          st_u32(dst + e0, pack4_e4m3(y));
          st_u32(dst + e1, pack4_e4m3(y + 4));
        } else {
          st_v2(dst + 2 * e0, pack4_bf16(y));
          st_v2(dst + 2 * e1, pack4_bf16(y + 4));
        }
      }
    } else {
      const int h = static_cast<int>(qw - static_cast<int64_t>(t) * a.qgroups) * 4 + g;
      if (h < a.Hq) {
        uint16_t* qp = a.q + static_cast<int64_t>(t) * a.q_tok + h * a.q_head + a.nope;
        float y[8], c[4], s[4];
        unpack4(ld_v2(qp + 4 * l8), y);
        unpack4(ld_v2(qp + kRope / 2 + 4 * l8), y + 4);
        mla_cos_sin<STYLE>(row, l8, c, s);
        mla_rotate<STYLE>(y, c, s);
        st_v2(qp + 4 * l8, pack4_bf16(y));
        st_v2(qp + kRope / 2 + 4 * l8, pack4_bf16(y + 4));
      }
    }
  }
}

using MlaKernel = void (*)(const MlaArgs);

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

  MlaKernel k = p.cache_fp8 ? (p.rope_style == 0 ? mla_kernel<1, 0> : mla_kernel<1, 1>)
                            : (p.rope_style == 0 ? mla_kernel<0, 0> : mla_kernel<0, 1>);
  const int64_t tasks = static_cast<int64_t>(p.T) * (1 + a.qgroups);
  const size_t smem = static_cast<size_t>(2 * p.B + 1) * sizeof(int);
  return launch_persistent(reinterpret_cast<const void*>(k), tasks, smem, stream,
                           [&](int grid) { return launch_pdl(k, grid, kThreads, smem, stream, a); });
}

}  // namespace fqr
