// pre_attn.cuh -- RoPE of one coordinate pair, and the RoPE + cache-append
// work that the absorb GEMM's launch carries in extra CTAs (mla_pre_attention).
//
// RoPE follows the RoFormer form (deepforge "DeepSeek-V2" page, §1: the
// decoupled RoPE key is stored beside the latent): pair (x_2k, x_2k+1) of a
// d_r-wide vector at absolute position p turns by the angle p * base^(-2k/d_r).
// The angle is formed and reduced to [-pi, pi] in fp64, so positions up to
// 128K keep their phase; the rotation itself is fp32.
//
// The standalone rope and append kernels and the fused pre-attention CTAs
// call the same functions, so the fused launch writes the same bits.
#pragma once

#include "common.cuh"

namespace mla {

// cos and sin of pair k's angle at position p.
__device__ __forceinline__ void rope_cos_sin(int k, int p, int d_rope, double base, float& c,
                                             float& s) {
  const double theta = pow(base, -2.0 * (double)k / (double)d_rope);
  const double ang = (double)p * theta;
  const double two_pi = 6.283185307179586476925286766559;
  const double red = ang - two_pi * rint(ang / two_pi);
  double sn, cs;
  sincos(red, &sn, &cs);
  c = (float)cs;
  s = (float)sn;
}

// (x0, x1) turned by the angle with cosine c and sine s.  Explicitly rounded
// operations, so every call site produces the same bits.
__device__ __forceinline__ void rope_rotate(float x0, float x1, float c, float s, float& y0,
                                            float& y1) {
  y0 = __fmaf_rn(x0, c, __fmul_rn(-x1, s));
  y1 = __fmaf_rn(x0, s, __fmul_rn(x1, c));
}

// Rotate pair k of the vector at x (position p, width d_rope) into y.  x and
// y may alias.
template <typename T>
__device__ __forceinline__ void rope_pair(const T* x, T* y, int k, int p, int d_rope,
                                          double base) {
  float c, s, y0, y1;
  rope_cos_sin(k, p, d_rope, base, c, s);
  rope_rotate(to_f32(x[2 * k]), to_f32(x[2 * k + 1]), c, s, y0, y1);
  y[2 * k] = from_f32<T>(y0);
  y[2 * k + 1] = from_f32<T>(y1);
}

// Pool row of new token t, or nullptr (raising MLA_ERR_BOUNDS) when its
// batch index, position or page id falls outside the page table or pool.
template <typename E>
__device__ __forceinline__ E* append_row(const int32_t* batch_idx, const int32_t* pos, int t,
                                         const int32_t* page_table, int max_pages, E* pool,
                                         int n_pages, int page_size, int D, bool report) {
  const int b = batch_idx[t];
  const int p = pos[t];
  const int lp = p / page_size;
  if (p < 0 || b < 0 || lp >= max_pages) {
    if (report) raise_flag(kFlagBounds);
    return nullptr;
  }
  const int page = page_table[(long long)b * max_pages + lp];
  if (page < 0 || page >= n_pages) {
    if (report) raise_flag(kFlagBounds);
    return nullptr;
  }
  return pool + ((long long)page * page_size + (p % page_size)) * D;
}

// The non-GEMM half of the pre-attention step for bf16 rows laid out as
// mla_project writes them for W_A0 = [W_Q; W_DKV; W_KR]:
//   y[t] = [q_1 .. q_H | c | k_rope_pre],  q_i = [q_nope (d_n) ; q_rope (d_r)].
// Work items, grid-strided:
//   [0, n_q)          RoPE pair (t, head, k) of q_rope -> qbuf[t][head][d_c + 2k ..]
//   [n_q, n_items)    pair e of token t's cache row: e < d_c/2 copies two latent
//                     numbers, otherwise RoPE pair e - d_c/2 of k_rope, written to
//                     the pool row and back into y (as the standalone in-place
//                     RoPE of k does).
struct PreAttnAux {
  __nv_bfloat16* y;
  long long ys_tok;       // elements per token row of y
  int H, d_nope, d_latent, d_rope;
  long long off_c;        // offset of c in a y row (= H * (d_nope + d_rope))
  __nv_bfloat16* qbuf;    // [T][H][d_latent + d_rope]
  const int32_t* batch_idx;
  const int32_t* pos;
  const int32_t* page_table;
  int max_pages;
  uint16_t* pool;
  int n_pages, page_size;
  double base;
  long long n_q, n_items;
};

__device__ __forceinline__ void pre_attention_aux(const PreAttnAux& a, long long i0,
                                                  long long stride) {
  const int half = a.d_rope / 2;
  const int dqk = a.d_nope + a.d_rope;
  const int D = a.d_latent + a.d_rope;
  const int row_pairs = D / 2;
  for (long long i = i0; i < a.n_items; i += stride) {
    if (i < a.n_q) {
      const int k = (int)(i % half);
      const int h = (int)((i / half) % a.H);
      const int t = (int)(i / ((long long)half * a.H));
      const __nv_bfloat16* x = a.y + t * a.ys_tok + (long long)h * dqk + a.d_nope;
      __nv_bfloat16* q = a.qbuf + ((long long)t * a.H + h) * D + a.d_latent;
      rope_pair(x, q, k, a.pos[t], a.d_rope, a.base);
    } else {
      const long long j = i - a.n_q;
      const int t = (int)(j / row_pairs);
      const int e = (int)(j % row_pairs);
      uint16_t* row = append_row(a.batch_idx, a.pos, t, a.page_table, a.max_pages, a.pool,
                                 a.n_pages, a.page_size, D, e == 0);
      if (row == nullptr) continue;
      __nv_bfloat16* yt = a.y + t * a.ys_tok + a.off_c;
      if (2 * e < a.d_latent) {
        const uint32_t v = *reinterpret_cast<const uint32_t*>(yt + 2 * e);
        *reinterpret_cast<uint32_t*>(row + 2 * e) = v;
      } else {
        const int k = e - a.d_latent / 2;
        __nv_bfloat16* kr = yt + a.d_latent;
        float c, sn, y0, y1;
        rope_cos_sin(k, a.pos[t], a.d_rope, a.base, c, sn);
        rope_rotate(to_f32(kr[2 * k]), to_f32(kr[2 * k + 1]), c, sn, y0, y1);
        const __nv_bfloat16 r0 = from_f32<__nv_bfloat16>(y0), r1 = from_f32<__nv_bfloat16>(y1);
        kr[2 * k] = r0;
        kr[2 * k + 1] = r1;
        row[a.d_latent + 2 * k] = __bfloat16_as_ushort(r0);
        row[a.d_latent + 2 * k + 1] = __bfloat16_as_ushort(r1);
      }
    }
  }
}

}  // namespace mla
