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
//   [0, n_rope)        (token t, head group g, pair k): one angle, applied to
//                      pair k of the q_rope of heads [8g, 8g + 8)
//                      (-> qbuf[t][head][d_c + 2k ..]); group 0 also turns
//                      pair k of k_rope (-> the pool row and back into y, as
//                      the standalone in-place RoPE of k does)
//   [n_rope, n_items)  (token t, 16-byte piece u) of the latent: copied to the
//                      pool row
// Consecutive items of a warp take consecutive k (or u), so every access of
// the warp is one contiguous run; a thread touches eight heads, not all of
// them, so the RoPE of many heads spreads over many threads.
constexpr int kRopeHeadsPerItem = 8;
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
  long long n_rope, n_items;
};

__device__ __forceinline__ void pre_attention_aux(const PreAttnAux& a, long long i0,
                                                  long long stride) {
  const int half = a.d_rope / 2;
  const int dqk = a.d_nope + a.d_rope;
  const int D = a.d_latent + a.d_rope;
  const int pieces = a.d_latent / 8;
  const int groups = (a.H + kRopeHeadsPerItem - 1) / kRopeHeadsPerItem;
  for (long long i = i0; i < a.n_items; i += stride) {
    if (i < a.n_rope) {
      const int t = (int)(i / ((long long)half * groups));
      const int rem = (int)(i % ((long long)half * groups));
      const int g = rem / half, k = rem % half;
      const int p = a.pos[t];
      float c, sn;
      rope_cos_sin(k, p, a.d_rope, a.base, c, sn);
      const __nv_bfloat16* xq = a.y + t * a.ys_tok + a.d_nope + 2 * k;
      __nv_bfloat16* yq = a.qbuf + (long long)t * a.H * D + a.d_latent + 2 * k;
      const int h0 = kRopeHeadsPerItem * g;
      const int h1 = min(a.H, h0 + kRopeHeadsPerItem);
      __nv_bfloat162 v[kRopeHeadsPerItem];
#pragma unroll
      for (int u = 0; u < kRopeHeadsPerItem; ++u)
        if (h0 + u < h1)
          v[u] = *reinterpret_cast<const __nv_bfloat162*>(xq + (long long)(h0 + u) * dqk);
#pragma unroll
      for (int u = 0; u < kRopeHeadsPerItem; ++u) {
        if (h0 + u >= h1) break;
        float y0, y1;
        rope_rotate(to_f32(v[u].x), to_f32(v[u].y), c, sn, y0, y1);
        __nv_bfloat162 o;
        o.x = from_f32<__nv_bfloat16>(y0);
        o.y = from_f32<__nv_bfloat16>(y1);
        *reinterpret_cast<__nv_bfloat162*>(yq + (long long)(h0 + u) * D) = o;
      }
      if (g != 0) continue;
      __nv_bfloat16* kr = a.y + t * a.ys_tok + a.off_c + a.d_latent + 2 * k;
      float y0, y1;
      rope_rotate(to_f32(kr[0]), to_f32(kr[1]), c, sn, y0, y1);
      const __nv_bfloat16 r0 = from_f32<__nv_bfloat16>(y0), r1 = from_f32<__nv_bfloat16>(y1);
      kr[0] = r0;
      kr[1] = r1;
      uint16_t* row = append_row(a.batch_idx, a.pos, t, a.page_table, a.max_pages, a.pool,
                                 a.n_pages, a.page_size, D, false);
      if (row != nullptr) {
        row[a.d_latent + 2 * k] = __bfloat16_as_ushort(r0);
        row[a.d_latent + 2 * k + 1] = __bfloat16_as_ushort(r1);
      }
    } else {
      const long long j = i - a.n_rope;
      const int t = (int)(j / pieces);
      const int u = (int)(j % pieces);
      uint16_t* row = append_row(a.batch_idx, a.pos, t, a.page_table, a.max_pages, a.pool,
                                 a.n_pages, a.page_size, D, u == 0);
      if (row == nullptr) continue;
      const uint4 v = *reinterpret_cast<const uint4*>(a.y + t * a.ys_tok + a.off_c + 8 * u);
      *reinterpret_cast<uint4*>(row + 8 * u) = v;
    }
  }
}

}  // namespace mla
