// fp8.cuh -- the 8-bit latent cache: row format and quantizer kernels.
//
// The pages' stretch goal (deepforge "DeepSeek-V2", §4 "Build it yourself":
// quantize the latent to 8 bits and measure the extra error a production
// cache pays).  Row of one token, 656 bytes:
//   [0, 512)    latent c / s_t in E4M3 (1 sign, 4 exponent bits with bias 7,
//               3 mantissa bits, largest finite value 448), round to nearest
//               even, saturating
//   [512, 640)  RoPE key k / s_t in IEEE half precision (64 x 2 bytes)
//   [640, 644)  s_t = max(max|c| / 448, max|k| / 65504) as fp32 (1 for an
//               all-zero row): one scale brings both parts into range
//   [644, 656)  zero
// s_t and the quotients are single-precision, correctly rounded divisions,
// so a quantizer on any machine that follows the same steps writes the same
// bytes.  The cache numbers a row stands for are s_t [c8 ; k16].
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace mla {

namespace fp8 {
constexpr int kDC = 512;
constexpr int kDR = 64;
constexpr int kRowBytes = 656;
constexpr int kOffRope = 512;
constexpr int kOffScale = 640;
constexpr float kMax = 448.0f;
constexpr float kHalfMax = 65504.0f;
}  // namespace fp8

// Two floats to two E4M3 bytes (lo -> lower address byte), nearest even,
// saturating at +-448.
__device__ __forceinline__ uint16_t e4m3x2_from_f32(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// One warp quantizes one row.  c: 512 bf16 latent values, kr: 64 bf16 RoPE
// values (raw bits), dst: the 656-byte row (16-byte aligned).
__device__ __forceinline__ void quantize_row_fp8(const uint16_t* c, const uint16_t* kr,
                                                 uint8_t* dst, int lane) {
  // lane owns latent values [16 lane, 16 lane + 16); lanes 0..7 also RoPE
  // values [8 lane, 8 lane + 8)
  uint32_t w[8];
  const uint4 a = *reinterpret_cast<const uint4*>(c + 16 * lane);
  const uint4 b = *reinterpret_cast<const uint4*>(c + 16 * lane + 8);
  w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
  w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  float v[16];
  float mc = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = bf16_lo(w[i]);
    v[2 * i + 1] = bf16_hi(w[i]);
    mc = fmaxf(mc, fmaxf(fabsf(v[2 * i]), fabsf(v[2 * i + 1])));
  }
  float kv[8];
  float mk = 0.f;
  if (lane < 8) {
    const uint4 k = *reinterpret_cast<const uint4*>(kr + 8 * lane);
    const uint32_t kw[4] = {k.x, k.y, k.z, k.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      kv[2 * i] = bf16_lo(kw[i]);
      kv[2 * i + 1] = bf16_hi(kw[i]);
      mk = fmaxf(mk, fmaxf(fabsf(kv[2 * i]), fabsf(kv[2 * i + 1])));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
    mk = fmaxf(mk, __shfl_xor_sync(0xffffffffu, mk, o));
  }
  // one scale for the row: both parts divided by it fit their formats
  float s = fmaxf(__fdiv_rn(mc, fp8::kMax), __fdiv_rn(mk, fp8::kHalfMax));
  if (!(s > 0.f)) s = 1.f;
  uint32_t q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint16_t lo = e4m3x2_from_f32(__fdiv_rn(v[4 * i], s), __fdiv_rn(v[4 * i + 1], s));
    const uint16_t hi = e4m3x2_from_f32(__fdiv_rn(v[4 * i + 2], s), __fdiv_rn(v[4 * i + 3], s));
    q[i] = (uint32_t)lo | ((uint32_t)hi << 16);
  }
  *reinterpret_cast<uint4*>(dst + 16 * lane) = make_uint4(q[0], q[1], q[2], q[3]);
  if (lane < 8) {
    uint32_t h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 hv = __floats2half2_rn(__fdiv_rn(kv[2 * i], s), __fdiv_rn(kv[2 * i + 1], s));
      h[i] = *reinterpret_cast<uint32_t*>(&hv);
    }
    *reinterpret_cast<uint4*>(dst + fp8::kOffRope + 16 * lane) = make_uint4(h[0], h[1], h[2], h[3]);
  } else if (lane == 8) {
    *reinterpret_cast<uint4*>(dst + fp8::kOffScale) = make_uint4(__float_as_uint(s), 0u, 0u, 0u);
  }
}

// Append: token t's [c ; kr] (bf16, row strides in elements) to the slot of
// (batch_idx[t], pos[t]) of the 8-bit pool.  One warp per token; a page id
// outside the pool skips the token and raises MLA_ERR_BOUNDS.
__global__ void __launch_bounds__(256) append_fp8_kernel(
    const uint16_t* c, long long cs_tok, const uint16_t* kr, long long ks_tok,
    const int32_t* batch_idx, const int32_t* pos, const int32_t* page_table, int max_pages,
    uint8_t* pool8, int n_pages, int page_size, int T) {
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const int p = pos[t];
  const int pi = p / page_size;
  int page = -1;
  if (p >= 0 && pi < max_pages) page = page_table[(long long)batch_idx[t] * max_pages + pi];
  if (page < 0 || page >= n_pages) {
    if (lane == 0) raise_flag(kFlagBounds);
    return;
  }
  uint8_t* dst = pool8 + ((size_t)page * page_size + p % page_size) * fp8::kRowBytes;
  quantize_row_fp8(c + t * cs_tok, kr + t * ks_tok, dst, lane);
}

// Whole-pool conversion: row r of the bf16 pool (576 values) to row r of the
// 8-bit pool.  One warp per row.
__global__ void __launch_bounds__(256) quantize_pool_fp8_kernel(const uint16_t* pool,
                                                                uint8_t* pool8, long long rows) {
  const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  const uint16_t* src = pool + r * (fp8::kDC + fp8::kDR);
  quantize_row_fp8(src, src + fp8::kDC, pool8 + r * fp8::kRowBytes, threadIdx.x & 31);
}

}  // namespace mla
