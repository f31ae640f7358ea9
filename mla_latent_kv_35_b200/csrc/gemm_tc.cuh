// gemm_tc.cuh -- weight-streaming bf16 GEMM on the 5th-generation tensor
// cores (tcgen05, TMEM accumulator, TMA-fed 128-byte-swizzled operands).
//
//   out[b][n][m] (+)= sum_k W[b][m][k] * X[b][n][k]
//
// The weight matrix is the MMA's A operand (M = output features, 128 per
// CTA) and the few activation rows are the B operand (N = tokens, padded to
// a multiple of 16, at most 256 per CTA): at decode the token count is far
// below 128, so putting the weights on M keeps the MMA at full height.
// A may be K-major ([M][K], the usual [out, in] weight) or MN-major ([K][M],
// e.g. W_UK[i] read as its transpose).  X is always K-major.  Split-K over
// grid.y writes each split's fp32 partial to its own slice of the output
// (split s at out + s * os); an ordered sum of the slices follows, so the
// result does not depend on the order the splits finish in.
//
// Warp roles (128 threads): warp 0 lane 0 issues TMA loads into an
// S-stage ring; warp 1 allocates TMEM and its lane 0 issues the MMAs; after
// the last MMA all four warps read the accumulator (TMEM lane = output row)
// and store it.
//
// kMT = 2 gives a CTA two 128-row M tiles against the same token tile (two
// accumulators of BN columns, 512 TMEM columns at BN = 256): each token
// tile brought into shared memory serves twice the MMA work, which halves
// the operand traffic per FLOP when both M and N are large (prefill-sized
// GEMMs, whose operands are served from L2).
//
// Grid: x = token tile (fastest) x K split, y = M tile, z = batch entry.
// CTAs that run together share their weight tile, so each weight tile is
// read from HBM once and served to the token tiles from L2.
#pragma once

#include "common.cuh"
#include "pre_attn.cuh"

namespace mla {

enum GemmOut : int { kOutBf16 = 0, kOutF32 = 1, kOutF32Split = 2 };

struct GemmTcArgs {
  int M, N, K;           // per batch entry
  int vec_out;           // bf16 out with om == 1, on and ob multiples of 8, 16-byte aligned
  int n_tile;            // BN, multiple of 16, <= 256
  int n_tiles;           // ceil(N / BN)
  int k_chunks_per_split;
  int stages;
  void* out;
  long long ob, on, om;  // output strides in elements
  long long os;          // kOutF32Split: elements between the splits' slices
  int batch;             // GEMM batch entries
  int aux_z;             // grid.z slices [0, aux_z) run `aux`; GEMM entry b is slice aux_z + b
  PreAttnAux aux;
};

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 64;  // 64 bf16 = one 128-byte swizzle row

template <bool kAmn, int kOut, int kMT>
__global__ void __launch_bounds__(128, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                                                         const __grid_constant__ CUtensorMap tmX,
                                                         GemmTcArgs g) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[8];
  __shared__ __align__(8) uint64_t empty_bar[8];
  __shared__ __align__(8) uint64_t acc_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  if ((int)blockIdx.z < g.aux_z) {
    // extra CTAs of a fused pre-attention launch (scheduled first): RoPE and
    // cache append, independent of the GEMM CTAs (no barrier, no TMEM)
    const long long per_slice = (long long)gridDim.x * gridDim.y * blockDim.x;
    const long long cta = ((long long)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
    pre_attention_aux(g.aux, cta * blockDim.x + threadIdx.x, per_slice * (long long)g.aux_z);
    return;
  }

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * (kGemmBM * kMT);
  const int n_tile_idx = blockIdx.x % g.n_tiles;
  const int split = blockIdx.x / g.n_tiles;
  const int n0 = n_tile_idx * g.n_tile;
  const int b = blockIdx.z - g.aux_z;
  const int BN = g.n_tile;
  const int S = g.stages;
  const int k_chunks_total = (g.K + kGemmBK - 1) / kGemmBK;
  const int kc0 = split * g.k_chunks_per_split;
  const int kc1 = min(k_chunks_total, kc0 + g.k_chunks_per_split);
  const int nk = max(0, kc1 - kc0);

  const uint32_t a_tile = kGemmBM * kGemmBK * 2;   // 16 KB per M tile
  const uint32_t a_bytes = kMT * a_tile;
  const uint32_t x_bytes = BN * kGemmBK * 2;
  const uint32_t stage_bytes = a_bytes + x_bytes;
  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    mbar_init(smem_u32(&acc_bar), 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmX);
  }
  uint32_t tmem_cols = 32;
  while ((int)tmem_cols < BN * kMT) tmem_cols <<= 1;
  if (warp == 1) {
    tmem_alloc<1>(smem_u32(&tmem_base_sh), tmem_cols);
    tmem_relinquish<1>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_p = &abort_flag;

  if (warp == 0 && lane == 0 && nk > 0) {
    // ---------------- TMA producer ----------------
    int issued = 0;
    for (int i = 0; i < nk; ++i) {
      const int s = i % S;
      if (!mbar_wait(smem_u32(&empty_bar[s]), ((i / S) & 1) ^ 1, abort_p, 21, i)) break;
      const uint32_t fb = smem_u32(&full_bar[s]);
      const uint32_t sa = smem_base + s * stage_bytes;
      mbar_expect_tx(fb, stage_bytes);
      const int k = (kc0 + i) * kGemmBK;
#pragma unroll
      for (int mt = 0; mt < kMT; ++mt) {
        const int mr = m0 + mt * kGemmBM;
        if constexpr (kAmn) {
          tma_load_3d(sa + mt * a_tile, &tmA, mr, k, b, fb);
          tma_load_3d(sa + mt * a_tile + a_tile / 2, &tmA, mr + 64, k, b, fb);
        } else {
          tma_load_3d(sa + mt * a_tile, &tmA, k, mr, b, fb);
        }
      }
      tma_load_3d(sa + a_bytes, &tmX, k, n0, b, fb);
      ++issued;
    }
    if (*abort_p) {
      // let copies still in flight land before the CTA can exit
      for (int i = max(0, issued - S); i < issued; ++i)
        mbar_wait(smem_u32(&full_bar[i % S]), (i / S) & 1, nullptr);
    }
  } else if (warp == 1 && lane == 0 && nk > 0) {
    // ---------------- MMA issuer ----------------
    const uint32_t idesc = idesc_bf16_f32(kGemmBM, BN, kAmn, false);
    bool ok = true;
    for (int i = 0; i < nk; ++i) {
      const int s = i % S;
      if (!mbar_wait(smem_u32(&full_bar[s]), (i / S) & 1, abort_p, 22, i)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sa = smem_base + s * stage_bytes;
      const uint32_t sx = sa + a_bytes;
#pragma unroll
      for (int kk = 0; kk < kGemmBK / 16; ++kk) {
        const uint64_t xd = sw128_desc(sx + kk * 32, 16, 1024);
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt) {
          uint64_t ad;
          if constexpr (kAmn)
            ad = sw128_desc(sa + mt * a_tile + kk * 2048, 8192, 1024);  // 16 K-rows of 128 B
          else
            ad = sw128_desc(sa + mt * a_tile + kk * 32, 16, 1024);      // 16 K-elements = 32 B
          mma_bf16_ss<1>(tmem + mt * BN, ad, xd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
      }
      mma_commit_1(smem_u32(&empty_bar[s]));
    }
    if (ok) mma_commit_1(smem_u32(&acc_bar));
  }
  __syncwarp();

  // ---------------- epilogue: all 4 warps ----------------
  // TMEM loads are warp-collective: every thread takes the same branch
  const bool have =
      __syncthreads_and(nk > 0 && mbar_wait(smem_u32(&acc_bar), 0, abort_p, 23, 0)) != 0;
  if (have && kOut == kOutBf16 && g.vec_out) {
    // Rows m are TMEM lanes, one per thread, but the output has m
    // contiguous: each warp turns its 32 x 32 tiles around in shared memory
    // (the operand ring, idle once the last MMA has completed) and stores
    // 16-byte pieces of 8 consecutive m, 8 token rows per instruction.
    tc_fence_after();
    const uint32_t scratch = smem_base + warp * 2048;   // [32 tokens][32 m] bf16
    for (int mt = 0; mt < kMT; ++mt) {
      const int mw = m0 + mt * kGemmBM + warp * 32;       // this warp's first row
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + mt * BN + c0, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const __nv_bfloat16 v = __float2bfloat16_rn(__uint_as_float(r[i]));
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(scratch + i * 64 + lane * 2),
                       "h"(*reinterpret_cast<const uint16_t*>(&v))
                       : "memory");
        }
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int nl = q * 8 + (lane >> 2), ml = (lane & 3) * 8;
          uint4 v;
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                       : "r"(scratch + nl * 64 + ml * 2)
                       : "memory");
          const int n = n0 + c0 + nl, m = mw + ml;
          if (c0 + nl < BN && n < g.N && m < g.M)
            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) + (long long)b * g.ob +
                                      (long long)n * g.on + m) = v;
        }
        __syncwarp();
      }
    }
  } else if (have) {
    tc_fence_after();
    for (int mt = 0; mt < kMT; ++mt)
    for (int c0 = 0; c0 < BN; c0 += 32) {
      const int m = m0 + mt * kGemmBM + warp * 32 + lane;
      uint32_t r[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + mt * BN + c0, r);
      tmem_wait_ld();
      if (m < g.M) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int n = n0 + c0 + i;
          if (c0 + i < BN && n < g.N) {
            const long long o = (long long)b * g.ob + (long long)n * g.on + (long long)m * g.om;
            const float v = __uint_as_float(r[i]);
            if constexpr (kOut == kOutBf16)
              static_cast<__nv_bfloat16*>(g.out)[o] = __float2bfloat16_rn(v);
            else if constexpr (kOut == kOutF32)
              static_cast<float*>(g.out)[o] = v;
            else
              static_cast<float*>(g.out)[o + split * g.os] = v;
          }
        }
      }
    }
  } else if (nk == 0) {
    // empty K range: the product is zero
    for (int mt = 0; mt < kMT; ++mt) {
    const int m = m0 + mt * kGemmBM + warp * 32 + lane;
    if (m < g.M)
      for (int i = 0; i < BN; ++i) {
        const int n = n0 + i;
        if (n < g.N) {
          const long long o = (long long)b * g.ob + (long long)n * g.on + (long long)m * g.om;
          if constexpr (kOut == kOutBf16)
            static_cast<__nv_bfloat16*>(g.out)[o] = __float2bfloat16_rn(0.f);
          else if constexpr (kOut == kOutF32)
            static_cast<float*>(g.out)[o] = 0.f;
          else
            static_cast<float*>(g.out)[o + split * g.os] = 0.f;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc<1>(tmem, tmem_cols);
}

// out[i] = sum over s = 0 .. splits-1 of parts[s * n + i], in that order.
__global__ void sum_splits_kernel(const float* parts, int splits, long long n, float* out) {
  const long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i + 3 < n) {
    float4 acc = *reinterpret_cast<const float4*>(parts + i);
    for (int s = 1; s < splits; ++s) {
      const float4 v = *reinterpret_cast<const float4*>(parts + s * n + i);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    *reinterpret_cast<float4*>(out + i) = acc;
  } else {
    for (long long k = i; k < n; ++k) {
      float acc = parts[k];
      for (int s = 1; s < splits; ++s) acc += parts[s * n + k];
      out[k] = acc;
    }
  }
}

}  // namespace mla
