// simt.cuh -- CUDA-core kernels: the fp32 path of every step, plus the
// elementwise steps (RoPE, cache append, casts), the split planner and the
// log-sum-exp combine that the bf16 path shares.
#pragma once

#include "common.cuh"
#include "pre_attn.cuh"

namespace mla {

// ---------------------------------------------------------------------------
// Batched strided GEMM on CUDA cores (fp32 accumulate).
//   out[b*ob + n*on + m*om] (+)= sum_k A[b*ab + m*am + k*ak] * X[b*xb + n*xn + k*xk]
// 64x64 output tile per 256-thread block, 4x4 per thread, k-tiles of 16.
// ---------------------------------------------------------------------------
struct SimtGemmArgs {
  const void* A;
  const void* X;
  void* out;
  int M, N, K, batch;
  long long ab, am, ak, xb, xn, xk, ob, on, om;
  int atomic_out;  // fp32 output only: accumulate with atomicAdd
};

template <typename TI, typename TO>
__global__ void __launch_bounds__(256) simt_gemm_kernel(SimtGemmArgs g) {
  __shared__ float As[16][65];
  __shared__ float Xs[16][65];
  const TI* A = static_cast<const TI*>(g.A);
  const TI* X = static_cast<const TI*>(g.X);
  TO* out = static_cast<TO*>(g.out);
  const int b = blockIdx.z;
  const int m0 = blockIdx.x * 64, n0 = blockIdx.y * 64;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < g.K; k0 += 16) {
    for (int e = threadIdx.x; e < 16 * 64; e += 256) {
      int kk = e / 64, mm = e % 64;
      int k = k0 + kk;
      int m = m0 + mm, n = n0 + mm;
      As[kk][mm] = (k < g.K && m < g.M) ? to_f32(A[b * g.ab + m * g.am + k * g.ak]) : 0.f;
      Xs[kk][mm] = (k < g.K && n < g.N) ? to_f32(X[b * g.xb + n * g.xn + k * g.xk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], x[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][tx + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) x[j] = Xs[kk][ty + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], x[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int m = m0 + tx + 16 * i, n = n0 + ty + 16 * j;
      if (m < g.M && n < g.N) {
        long long o = b * g.ob + n * g.on + m * g.om;
        if constexpr (sizeof(TO) == 4) {
          if (g.atomic_out)
            atomicAdd(reinterpret_cast<float*>(out) + o, acc[i][j]);
          else
            out[o] = from_f32<TO>(acc[i][j]);
        } else {
          out[o] = from_f32<TO>(acc[i][j]);
        }
      }
    }
}

// ---------------------------------------------------------------------------
// RoPE: rotate consecutive pairs by pos * base^(-2k/d); angle in fp64.  One
// thread per (token, group of 32 heads, pair k), k fastest: the angle's cos
// and sin are formed once and turn pair k of all heads of the group.
// ---------------------------------------------------------------------------
constexpr int kRopeGroup = 32;

template <typename T>
__global__ void rope_kernel(const T* x, long long xs_tok, long long xs_head, int nh, T* y,
                            long long ys_tok, long long ys_head, const int32_t* pos, int Tn,
                            int d_rope, double base) {
  const int half = d_rope / 2;
  const int ng = (nh + kRopeGroup - 1) / kRopeGroup;
  long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  long long total = (long long)Tn * ng * half;
  if (idx >= total) return;
  const int k = (int)(idx % half);
  const int g = (int)((idx / half) % ng);
  const int t = (int)(idx / ((long long)half * ng));
  float c, s;
  rope_cos_sin(k, pos[t], d_rope, base, c, s);
  for (int i = 0; i < kRopeGroup; ++i) {
    const int h = g * kRopeGroup + i;
    if (h >= nh) break;
    const T* xp = x + t * xs_tok + h * xs_head;
    T* yp = y + t * ys_tok + h * ys_head;
    float y0, y1;
    rope_rotate(to_f32(xp[2 * k]), to_f32(xp[2 * k + 1]), c, s, y0, y1);
    yp[2 * k] = from_f32<T>(y0);
    yp[2 * k + 1] = from_f32<T>(y1);
  }
}

// ---------------------------------------------------------------------------
// Cache append: exact copy of each new token's latent and RoPE key into its
// page slot.  Element size E bytes (2 for bf16, 4 for fp32).
// ---------------------------------------------------------------------------
template <typename E>
__global__ void append_kernel(const E* c, long long cs_tok, const E* kr, long long ks_tok,
                              const int32_t* batch_idx, const int32_t* pos,
                              const int32_t* page_table, int max_pages, E* pool, int n_pages,
                              int page_size, int d_c, int d_r) {
  const int t = blockIdx.x;
  const int D = d_c + d_r;
  E* row = append_row(batch_idx, pos, t, page_table, max_pages, pool, n_pages, page_size, D,
                      threadIdx.x == 0);
  if (row == nullptr) return;
  for (int e = threadIdx.x; e < D; e += blockDim.x)
    row[e] = e < d_c ? c[t * cs_tok + e] : kr[t * ks_tok + (e - d_c)];
}

__global__ void cast_f32_bf16_kernel(const float* x, __nv_bfloat16* y, long long n) {
  long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i + 3 < n) {
    float4 v = *reinterpret_cast<const float4*>(x + i);
    uint2 o;
    o.x = pack_bf16x2(v.x, v.y);
    o.y = pack_bf16x2(v.z, v.w);
    *reinterpret_cast<uint2*>(y + i) = o;
  } else {
    for (; i < n; ++i) y[i] = __float2bfloat16_rn(x[i]);
  }
}

// ---------------------------------------------------------------------------
// Split planning.  Virtual sequence v = r*B + b is row block r of sequence
// b (R row blocks per sequence, row-block-major) and has nb_v =
// ceil(L_b / BLK) token blocks.  start[v] = sum_{u<v} nb_u and start[V] =
// total.  Worker k of G owns blocks [lo_k, lo_{k+1}) of the concatenation,
// lo_k = floor(k * total / G).  The piece of worker k in v writes partial
// slot k + v (unique: pieces form a monotone staircase).  Row-block-major
// order puts worker k of row block 0 and worker k + G/R of row block r on the
// same tokens of the same sequence at the same time (G a multiple of R), so
// the second read of a cache tile comes from L2.
// ---------------------------------------------------------------------------
// Block counts per virtual sequence and their exclusive prefix sums.  With
// `tail` (tokens of the sequence held elsewhere, after this cache's range) a
// sequence may hold any number of tokens here, none included, since its
// queries may sit in another cache; without it, it must hold the S_q query
// tokens.
__global__ void plan_kernel(const int32_t* seq_lens, const int32_t* tail, int B, int R, int S_q,
                            int max_tokens, int BLK, int32_t* start) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int V = B * R;
  for (int base = 0; base < V; base += blockDim.x) {
    const int v = base + threadIdx.x;
    int nb = 0;
    if (v < V) {
      const int L = seq_lens[v % B];
      const int tl = tail != nullptr ? tail[v % B] : 0;
      if (L < 0 || tl < 0 || L > max_tokens || (tail == nullptr && L < S_q)) {
        if (v < B) raise_flag(kFlagBounds);
      } else {
        nb = (L + BLK - 1) / BLK;
      }
    }
    // inclusive warp scan
    int x = nb;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[w] = x;
    __syncthreads();
    if (w == 0) {
      int s = lane < (int)(blockDim.x >> 5) ? warp_sums[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      warp_sums[lane] = s;  // inclusive prefix over warps
    }
    __syncthreads();
    const int excl = carry + (w > 0 ? warp_sums[w - 1] : 0) + x - nb;
    if (v < V) start[v] = excl;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = excl + nb;
    __syncthreads();
  }
  if (threadIdx.x == 0) start[V] = carry;
}

__device__ __forceinline__ int worker_lo(int k, int total, int G) {
  return (int)(((long long)k * total) / G);
}
// worker owning global block x (0 <= x < total)
__device__ __forceinline__ int worker_of(int x, int total, int G) {
  return (int)((((long long)x + 1) * G - 1) / total);
}
// first v with start[v+1] > x, i.e. the virtual sequence holding block x
__device__ __forceinline__ int seq_of_block(const int32_t* start, int V, int x) {
  int lo = 0, hi = V - 1;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (start[mid + 1] > x) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// ---------------------------------------------------------------------------
// SIMT split-KV decode: one warp per query row, 8 rows per block.  Grid
// (G workers, ceil(rows_per_v / 8)).  Writes normalised partial outputs and
// natural-log lse per piece into slot k + v.  R = 1 here (v = b).
// ---------------------------------------------------------------------------
template <typename T, int kMaxC>
__global__ void __launch_bounds__(256) decode_simt_kernel(
    const T* qbuf, const T* pool, int n_pages, const int32_t* page_table, int max_pages,
    const int32_t* seq_lens, const int32_t* tail, int B, int S_q, int H, int d_c, int d_r,
    int page_size, float scale, int G, int BLK, const int32_t* start, float* ws_lse,
    float* ws_o) {
  const int k = blockIdx.x;
  const int lane = threadIdx.x & 31;
  const int rows = S_q * H;
  const int r = blockIdx.y * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int total = start[B];
  if (total == 0) return;
  const int lo = worker_lo(k, total, G), hi = worker_lo(k + 1, total, G);
  if (lo >= hi) return;
  const int D = d_c + d_r;
  const int j = r / H;
  int v = seq_of_block(start, B, lo);
  for (; v < B && start[v] < hi; ++v) {
    const int x0 = max(lo, start[v]) - start[v];
    const int x1 = min(hi, start[v + 1]) - start[v];
    if (x1 <= x0) continue;
    const int L = seq_lens[v];
    // visible tokens t < limit; the query tokens are the last S_q of the
    // sequence, `tail` of which lie past this cache's range
    const int limit = L + (tail != nullptr ? tail[v] : 0) - S_q + j + 1;
    const int t0 = x0 * BLK, t1 = min(min(x1 * BLK, L), limit);
    const T* q = qbuf + ((long long)v * rows + r) * D;
    float m = -INFINITY, l = 0.f;
    float o[kMaxC];
#pragma unroll
    for (int u = 0; u < kMaxC; ++u) o[u] = 0.f;
    for (int t = t0; t < t1; ++t) {
      const int page = page_table[(long long)v * max_pages + t / page_size];
      if (page < 0 || page >= n_pages) {
        if (lane == 0) raise_flag(kFlagBounds);
        continue;
      }
      const T* row = pool + ((long long)page * page_size + t % page_size) * D;
      float s = 0.f;
      for (int e = lane; e < D; e += 32) s = fmaf(to_f32(q[e]), to_f32(row[e]), s);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      s *= scale;
      const float m_new = fmaxf(m, s);
      const float alpha = __expf(m - m_new);
      const float p = __expf(s - m_new);
      l = l * alpha + p;
#pragma unroll
      for (int u = 0; u < kMaxC; ++u) {
        const int c = lane + 32 * u;
        if (c < d_c) o[u] = o[u] * alpha + p * to_f32(row[c]);
      }
      m = m_new;
    }
    const long long slot = (long long)k + v;
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int u = 0; u < kMaxC; ++u) {
      const int c = lane + 32 * u;
      if (c < d_c) ws_o[(slot * rows + r) * d_c + c] = o[u] * inv;
    }
    if (lane == 0) ws_lse[slot * rows + r] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

// ---------------------------------------------------------------------------
// Log-sum-exp combine of the pieces of every virtual sequence.
//   o = sum_k w_k o_k / sum_k w_k, w_k = exp(lse_k - max lse), lse = max + ln sum w
// Grid (V, ceil(rows_per_v * wpr / 8)), 8 warps per CTA and wpr warps per
// row (1, 2, 4 or 8: more for rows that merge many pieces, a long sequence
// split over many workers).  The lanes of each warp read the row's piece
// LSEs 32 at a time and reduce them with shuffles; lane i keeps the weight
// of piece i of each group of 32 and hands it out with a shuffle.  Warp u
// of a row's wpr merges the pieces i with (i / 2) % wpr == u, two at a time,
// each lane owning four float4 columns (d_c <= 512, a multiple of 4), so
// every lane keeps eight loads in flight; the wpr partial sums meet in
// shared memory.  Virtual sequence v is row block v / B of sequence v % B
// (B = V / R): rows_per_v workspace rows, of which the ones past the
// sequence's rows_seq query rows are padding and skipped.
// ---------------------------------------------------------------------------
constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(
    const float* ws_lse, const float* ws_o, const int32_t* start, int V, int R, int G,
    int rows_per_v, int rows_seq, int d_c, int wpr, float* o_lat, float* lse) {
  __shared__ float4 part[7][128];   // partial sums of warps 1.. of a row group
  const int v = blockIdx.x;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = w % wpr;                               // this warp's share of the row
  const int r = (blockIdx.y * 8 + w) / wpr;
  const int nseq = V / R;
  const int row_in_seq = (v / nseq) * rows_per_v + r;
  const bool live_row = r < rows_per_v && row_in_seq < rows_seq;
  const int total = start[V];
  const long long out_row = (long long)(v % nseq) * rows_seq + row_in_seq;
  const bool any = start[v + 1] > start[v];
  const int k0 = any ? worker_of(start[v], total, G) : 0;
  const int n = (any && live_row) ? worker_of(start[v + 1] - 1, total, G) - k0 + 1 : 0;
  // lse of piece i of the row, -inf for a worker with an empty range (only
  // when G > total), which wrote no slot
  auto piece_lse = [&](int i) {
    const int k = k0 + i;
    return i < n && worker_lo(k + 1, total, G) > worker_lo(k, total, G)
               ? ws_lse[((long long)k + v) * rows_per_v + r] : -INFINITY;
  };
  float mx = -INFINITY;
  for (int i = lane; i < n; i += 32) mx = fmaxf(mx, piece_lse(i));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float z = 0.f;
  if (mx != -INFINITY)
    for (int i = lane; i < n; i += 32) z += __expf(piece_lse(i) - mx);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  if (live_row && u == 0 && lane == 0) lse[out_row] = mx == -INFINITY ? -INFINITY : mx + logf(z);
  float4 acc[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (mx != -INFINITY) {
    const float inv_z = 1.f / z;
    for (int g = 0; g < n; g += 32) {
      // lane i: weight of piece g + i (0 for a piece with nothing visible
      // or no slot written: its row is not read)
      const float w_mine = g + lane < n ? __expf(piece_lse(g + lane) - mx) * inv_z : 0.f;
      const int cnt = min(32, n - g);
      for (int i = 2 * u; i < cnt; i += 2 * wpr) {
        const float w0 = __shfl_sync(0xffffffffu, w_mine, i);
        const float w1 = __shfl_sync(0xffffffffu, w_mine, min(i + 1, 31));
        const float wb = i + 1 < cnt ? w1 : 0.f;
        const float* r0 = ws_o + (((long long)(k0 + g + i) + v) * rows_per_v + r) * d_c;
        const float* r1 = r0 + (long long)rows_per_v * d_c;   // the next slot
        float4 x0[4], x1[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c4 = 4 * lane + 128 * q;
          const bool in = c4 < d_c;
          x0[q] = in && w0 != 0.f ? *reinterpret_cast<const float4*>(r0 + c4)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
          x1[q] = in && wb != 0.f ? *reinterpret_cast<const float4*>(r1 + c4)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[q].x = fmaf(w0, x0[q].x, fmaf(wb, x1[q].x, acc[q].x));
          acc[q].y = fmaf(w0, x0[q].y, fmaf(wb, x1[q].y, acc[q].y));
          acc[q].z = fmaf(w0, x0[q].z, fmaf(wb, x1[q].z, acc[q].z));
          acc[q].w = fmaf(w0, x0[q].w, fmaf(wb, x1[q].w, acc[q].w));
        }
      }
    }
  }
  if (wpr > 1) {
    // warps 1.. of each row group leave their sums; warp 0 of the group adds
    if (u != 0) {
#pragma unroll
      for (int q = 0; q < 4; ++q) part[w - 1][32 * q + lane] = acc[q];
    }
    __syncthreads();
    if (u == 0) {
      for (int t = 1; t < wpr; ++t)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 y = part[w + t - 1][32 * q + lane];
          acc[q].x += y.x; acc[q].y += y.y; acc[q].z += y.z; acc[q].w += y.w;
        }
    }
  }
  if (!live_row || u != 0) return;
  float* dst = o_lat + out_row * d_c;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int c4 = 4 * lane + 128 * q;
    if (c4 < d_c) *reinterpret_cast<float4*>(dst + c4) = acc[q];
  }
}

// Warps per row of combine_kernel for a workload: enough that a row's
// pieces spread to about eight per warp.
inline int combine_warps_per_row(int V, int G) {
  const int pieces = (G + V - 1) / V + 1;   // pieces of a virtual sequence, about
  int wpr = 1;
  while (wpr < 8 && pieces > 8 * wpr) wpr *= 2;
  return wpr;
}

// Merge of partial attention results over disjoint token sets (the parts):
// one warp per row, parts with lse = -inf (nothing visible) contribute
// nothing, a row with no visible token anywhere gets o = 0, lse = -inf.
//   m = max_p lse_p,  z = sum_p e^(lse_p - m),
//   o = sum_p e^(lse_p - m) o_p / z,  lse = m + ln z.
__global__ void __launch_bounds__(256) combine_parts_kernel(const float* o_parts,
                                                            const float* lse_parts, int n_parts,
                                                            long long rows, int d_c, float* o,
                                                            float* lse) {
  const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  float mx = -INFINITY;
  for (int p = 0; p < n_parts; ++p) mx = fmaxf(mx, lse_parts[p * rows + r]);
  float* dst = o + r * d_c;
  if (mx == -INFINITY) {
    for (int c = lane; c < d_c; c += 32) dst[c] = 0.f;
    if (lane == 0) lse[r] = -INFINITY;
    return;
  }
  float z = 0.f;
  for (int p = 0; p < n_parts; ++p) z += __expf(lse_parts[p * rows + r] - mx);
  const float inv_z = 1.f / z;
  for (int c = lane; c < d_c; c += 32) {
    float acc = 0.f;
    for (int p = 0; p < n_parts; ++p) {
      const float w = __expf(lse_parts[p * rows + r] - mx) * inv_z;
      acc = fmaf(w, o_parts[((long long)p * rows + r) * d_c + c], acc);
    }
    dst[c] = acc;
  }
  if (lane == 0) lse[r] = mx + logf(z);
}

__global__ void wait_selftest_kernel(unsigned long long wait_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(smem_u32(&bar), 0)) {
      if (globaltimer() - t0 > wait_ns) {
        raise_flag(kFlagTimeout);
        break;
      }
    }
  }
}

}  // namespace mla
