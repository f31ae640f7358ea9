// api.cu -- the extern "C" entry points of libmla_b200.so (see include/mla.h).
//
// Host-side validation, TMA descriptor encoding, split planning and kernel
// launches.  All device work is in the kernels included below; nothing here
// computes on the host.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/mla.h"
#include "common.cuh"
#include "decode_fp8.cuh"
#include "decode_tc.cuh"
#include "fp8.cuh"
#include "gemm_tc.cuh"
#include "prefill_tc.cuh"
#include "simt.cuh"

using namespace mla;

namespace {

std::atomic<uint64_t> g_launches{0};

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mla_status check_launch() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

#define MLA_TRY(expr)                   \
  do {                                  \
    mla_status _s = (expr);             \
    if (_s != MLA_OK) return _s;        \
  } while (0)

bool dims_ok(const mla_dims* d) {
  return d != nullptr && d->n_heads > 0 && d->d_nope > 0 && d->d_latent > 0 && d->d_rope >= 0 &&
         (d->d_rope % 2) == 0 && d->d_v > 0 && d->d_model > 0 && d->page_size > 0 &&
         (d->dtype == MLA_F32 || d->dtype == MLA_BF16) && std::isfinite(d->scale);
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// ---------------------------------------------------------------------------
// TMA descriptors (driver entry point fetched through the runtime)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 tensor of rank `rank` (<= 5), dims innermost first, byte strides of
// dims 1.., 128-byte swizzle, zero fill out of bounds.
bool make_tmap_typed(CUtensorMapDataType type, CUtensorMap* m, const void* ptr, int rank,
                     const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t d[5], s[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) s[i] = strides_bytes[i];
  CUresult r = fn(m, type, rank, const_cast<void*>(ptr), d, s, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_bf16(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box) {
  return make_tmap_typed(CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, m, ptr, rank, dims, strides_bytes, box);
}

bool make_tmap_f16(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims,
                   const uint64_t* strides_bytes, const uint32_t* box) {
  return make_tmap_typed(CU_TENSOR_MAP_DATA_TYPE_FLOAT16, m, ptr, rank, dims, strides_bytes, box);
}

// ---------------------------------------------------------------------------
// GEMM launchers
// ---------------------------------------------------------------------------
template <typename TI, typename TO>
mla_status launch_simt_gemm(const SimtGemmArgs& g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0 || g.batch <= 0) return MLA_OK;
  dim3 grid((g.M + 63) / 64, (g.N + 63) / 64, g.batch);
  simt_gemm_kernel<TI, TO><<<grid, 256, 0, st>>>(g);
  return check_launch();
}

// Wave-aware token tile width for two-M-tile GEMMs (see plan_tc_gemm).
#ifndef MLA_GEMM_WAVE_TILES
#define MLA_GEMM_WAVE_TILES 1
#endif

// Smallest K for two M tiles per CTA (see plan_tc_gemm).
#ifndef MLA_GEMM_MT2_MIN_K
#define MLA_GEMM_MT2_MIN_K 1024
#endif

struct TcGemmPlan {
  int n_tile, n_tiles, stages, splits, k_chunks_per_split, m_tiles_per_cta;
  size_t smem;
};

TcGemmPlan plan_tc_gemm(int M, int N, int K, int batch, bool allow_split) {
  TcGemmPlan p;
  int n16 = ((N + 15) / 16) * 16;
  p.n_tile = n16 < 256 ? n16 : 256;
  p.n_tiles = (N + p.n_tile - 1) / p.n_tile;
  // A grid with fewer CTAs than SMs takes narrower token tiles (down to 64
  // tokens), so that more SMs stream the weights (the W_UV GEMM of a decode
  // step: one M tile per head); the tiles of one weight tile meet in L2.
  if (!allow_split) {
    const long long mt = (M + kGemmBM - 1) / kGemmBM;
    while (p.n_tile >= 128 && mt * p.n_tiles * batch < sm_count()) {
      p.n_tile = ((p.n_tile / 2 + 15) / 16) * 16;
      p.n_tiles = (N + p.n_tile - 1) / p.n_tile;
    }
  }
  // two M tiles per CTA when M, N and K are large and the grid still has a
  // CTA for every SM (with a short K the store epilogue, which a lone CTA
  // on its SM does not overlap with MMAs, outweighs the halved operand
  // traffic)
  p.m_tiles_per_cta =
      (p.n_tile == 256 && M >= 2 * kGemmBM && K >= MLA_GEMM_MT2_MIN_K &&
       (long long)((M + 2 * kGemmBM - 1) / (2 * kGemmBM)) * p.n_tiles * batch >= sm_count())
          ? 2
          : 1;
  if (p.m_tiles_per_cta == 2 && MLA_GEMM_WAVE_TILES) {
    // One CTA per SM: the grid runs in ceil(CTAs / SMs) waves of CTAs whose
    // time grows with the token tile, plus a part that does not (the weight
    // tile's bytes).  Take the tile width (a multiple of 16 from 128 to 256)
    // that minimises waves x (width + 64), the widest on a tie (prefill W_O,
    // 5120 x 4096: 256 -> 3 waves of 320 CTAs, 192 -> 3 full waves of 440).
    const long long mt2 = (M + 2 * kGemmBM - 1) / (2 * kGemmBM);
    long long best = -1;
    int best_n = p.n_tile;
    for (int n = 256; n >= 128; n -= 16) {
      const long long c = mt2 * ((N + n - 1) / n) * batch;
      const long long cost = ((c + sm_count() - 1) / sm_count()) * (n + 64);
      if (best < 0 || cost < best) {
        best = cost;
        best_n = n;
      }
    }
    p.n_tile = best_n;
    p.n_tiles = (N + p.n_tile - 1) / p.n_tile;
  }
  const size_t stage_bytes =
      (size_t)p.m_tiles_per_cta * kGemmBM * kGemmBK * 2 + (size_t)p.n_tile * kGemmBK * 2;
  const int k_chunks = (K + kGemmBK - 1) / kGemmBK;
  p.splits = 1;
  const int bm = kGemmBM * p.m_tiles_per_cta;
  const long long ctas = (long long)((M + bm - 1) / bm) * p.n_tiles * batch;
  if (allow_split && p.m_tiles_per_cta == 1) {
    // as many splits as keep the grid within two CTAs per SM (one wave: a
    // partial second wave would double the time of its SMs)
    const long long target = 2LL * sm_count();
    while (ctas * (p.splits + 1) <= target && k_chunks / (p.splits + 1) >= 4) ++p.splits;
  }
  p.k_chunks_per_split = (k_chunks + p.splits - 1) / p.splits;
  // Ring depth: the weights stream from HBM, so a CTA keeps as many of its
  // k-chunks in flight as shared memory allows: up to ~200 KB when the grid
  // has at most one CTA per SM, ~96 KB (two CTAs per SM) otherwise, and
  // never more stages than the CTA has chunks (a short K leaves room for
  // more CTAs per SM instead).
  // (two M tiles take all 512 TMEM columns: one CTA per SM)
  const size_t budget =
      (p.m_tiles_per_cta == 2 || ctas * p.splits <= sm_count()) ? 200 * 1024 : 96 * 1024;
  int st = (int)(budget / stage_bytes);
  st = st < 2 ? 2 : (st > 8 ? 8 : st);
  if (st > p.k_chunks_per_split) st = p.k_chunks_per_split < 2 ? 2 : p.k_chunks_per_split;
  p.stages = st;
  p.smem = stage_bytes * p.stages + 1024;
  return p;
}

// A: [batch][M][K] K-major (a_mn = false) or [batch][K][M] (a_mn = true);
// X: [batch][N][K] with row stride xs_n and batch stride xs_b (elements).
// out element (b, n, m) at ob*b + on*n + om*m.
// kOutF32Split: the partial of split s goes to out + s * M * N (elements),
// laid out by (ob, on, om) within the slice; *splits_out receives the split
// count (the caller sums the slices).
mla_status launch_tc_gemm(const void* A, bool a_mn, long long as_b, const void* X, long long xs_n,
                          long long xs_b, int M, int N, int K, int batch, void* out, long long ob,
                          long long on, long long om, int out_kind, cudaStream_t st,
                          const PreAttnAux* aux = nullptr, int* splits_out = nullptr) {
  if (M <= 0 || N <= 0 || batch <= 0) return MLA_OK;
  if (!aligned16(A) || !aligned16(X) || (K % 8) != 0 || (xs_n % 8) != 0 || (xs_b % 8) != 0 ||
      (as_b % 8) != 0)
    return MLA_ERR_INVALID_ARG;
  if (a_mn && (M % 8) != 0) return MLA_ERR_INVALID_ARG;
  TcGemmPlan p = plan_tc_gemm(M, N, K, batch, out_kind == kOutF32Split);
  if (splits_out) *splits_out = p.splits;
  CUtensorMap tA, tX;
  {
    uint64_t dims[3], strides[2];
    uint32_t box[3];
    if (a_mn) {
      dims[0] = M; dims[1] = K; dims[2] = batch;
      strides[0] = (uint64_t)M * 2; strides[1] = (uint64_t)as_b * 2;
      box[0] = 64; box[1] = kGemmBK; box[2] = 1;
    } else {
      dims[0] = K; dims[1] = M; dims[2] = batch;
      strides[0] = (uint64_t)K * 2; strides[1] = (uint64_t)as_b * 2;
      box[0] = kGemmBK; box[1] = kGemmBM; box[2] = 1;
    }
    if (batch == 1) strides[1] = strides[0] * dims[1];
    if (!make_tmap_bf16(&tA, A, 3, dims, strides, box)) return MLA_ERR_CUDA;
  }
  {
    uint64_t dims[3] = {(uint64_t)K, (uint64_t)N, (uint64_t)batch};
    uint64_t strides[2] = {(uint64_t)xs_n * 2, (uint64_t)xs_b * 2};
    if (batch == 1) strides[1] = strides[0] * dims[1];
    uint32_t box[3] = {(uint32_t)kGemmBK, (uint32_t)p.n_tile, 1};
    if (!make_tmap_bf16(&tX, X, 3, dims, strides, box)) return MLA_ERR_CUDA;
  }
  GemmTcArgs g;
  g.M = M; g.N = N; g.K = K;
  g.n_tile = p.n_tile; g.n_tiles = p.n_tiles;
  g.k_chunks_per_split = p.k_chunks_per_split;
  g.stages = p.stages;
  g.out = out; g.ob = ob; g.on = on; g.om = om;
  // The 16-byte stores cover 8 consecutive m from a multiple of 8: whole
  // pieces only when M is a multiple of 8 too.
  g.vec_out = (out_kind == kOutBf16 && om == 1 && (on % 8) == 0 && (ob % 8) == 0 &&
               (M % 8) == 0 && aligned16(out))
                  ? 1
                  : 0;
  g.os = (long long)M * N;
  g.batch = batch;
  g.aux = PreAttnAux{};
  int aux_z = 0;
  if (aux != nullptr && aux->n_items > 0) {
    // enough extra z-slices for about 2 work items per thread
    g.aux = *aux;
    const long long per_slice =
        (long long)((M + kGemmBM * p.m_tiles_per_cta - 1) / (kGemmBM * p.m_tiles_per_cta)) *
        p.n_tiles * p.splits * 128;
    aux_z = (int)std::min<long long>(4096, (aux->n_items + 2 * per_slice - 1) / (2 * per_slice));
  }
  g.aux_z = aux_z;
  const int bm = kGemmBM * p.m_tiles_per_cta;
  dim3 grid(p.n_tiles * p.splits, (M + bm - 1) / bm, batch + aux_z);
#define MLA_GEMM_LAUNCH(AMN, OUT)                                                              \
  do {                                                                                         \
    auto kfn = p.m_tiles_per_cta == 2 ? gemm_tc_kernel<AMN, OUT, 2> : gemm_tc_kernel<AMN, OUT, 1>; \
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem) != \
        cudaSuccess)                                                                           \
      return MLA_ERR_CUDA;                                                                     \
    kfn<<<grid, 128, p.smem, st>>>(tA, tX, g);                                                 \
  } while (0)
  if (a_mn) {
    if (out_kind == kOutBf16) MLA_GEMM_LAUNCH(true, kOutBf16);
    else if (out_kind == kOutF32) MLA_GEMM_LAUNCH(true, kOutF32);
    else MLA_GEMM_LAUNCH(true, kOutF32Split);
  } else {
    if (out_kind == kOutBf16) MLA_GEMM_LAUNCH(false, kOutBf16);
    else if (out_kind == kOutF32) MLA_GEMM_LAUNCH(false, kOutF32);
    else MLA_GEMM_LAUNCH(false, kOutF32Split);
  }
#undef MLA_GEMM_LAUNCH
  return check_launch();
}

// ---------------------------------------------------------------------------
// decode planning
// ---------------------------------------------------------------------------
// cache tokens per work block: the tensor-core kernel's block (four pages),
// and the CUDA-core kernel's
constexpr int kBlockTokensSimt = 128;

// The tensor-core kernel covers every bf16 shape with DeepSeek-V2's cache
// row (512 + 64) and 64-token pages; query blocks of fewer than 128 rows
// (S_q * H < 128, or the last block of a sequence) are padded to the MMA's
// 128 rows, whose extra rows are computed and dropped.
bool use_tc_decode(const mla_dims* d, int S_q) {
  (void)S_q;
  return kDecodeTcReady && d->dtype == MLA_BF16 && d->d_latent == 512 && d->d_rope == 64 &&
         d->page_size == 64;
}

struct DecodeLayout {
  int R, rows_per_v, V, G;
  size_t off_start, off_lse, off_o, total;
};

DecodeLayout decode_layout(const mla_dims* d, int B, int S_q, int num_workers) {
  DecodeLayout L;
  const bool tc = use_tc_decode(d, S_q);
  // R blocks of rows_per_v workspace rows per sequence (the last block of
  // the tensor-core path may be partly padding)
  L.R = tc ? (S_q * d->n_heads + 127) / 128 : 1;
  L.rows_per_v = tc ? 128 : S_q * d->n_heads;
  L.V = B * L.R;
  const int sms = sm_count();
  L.G = num_workers > 0 ? num_workers : (tc ? sms / 2 : 2 * sms);
  const size_t n_slots = (size_t)L.G + L.V;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  L.off_start = 0;
  L.off_lse = up(sizeof(int32_t) * (L.V + 1));
  L.off_o = L.off_lse + up(sizeof(float) * n_slots * L.rows_per_v);
  L.total = L.off_o + up(sizeof(float) * n_slots * L.rows_per_v * d->d_latent);
  return L;
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported shape for the selected kernels";
    case MLA_ERR_CUDA: return "CUDA runtime error";
    case MLA_ERR_TIMEOUT: return "device wait timed out";
    case MLA_ERR_BOUNDS: return "device index out of bounds";
  }
  return "unknown status";
}

uint64_t mla_launch_count(void) { return g_launches.load(); }

mla_status mla_get_device_status(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return MLA_ERR_CUDA;
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return MLA_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (v & kFlagTimeout) return MLA_ERR_TIMEOUT;
  if (v & kFlagBounds) return MLA_ERR_BOUNDS;
  return MLA_OK;
}

mla_status mla_get_wait_diag(uint32_t* out4) {
  if (out4 == nullptr) return MLA_ERR_INVALID_ARG;
  unsigned v[4] = {0, 0, 0, 0}, z[4] = {0, 0, 0, 0};
  if (cudaMemcpyFromSymbol(v, g_wait_diag, sizeof(v)) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_wait_diag, z, sizeof(z)) != cudaSuccess) return MLA_ERR_CUDA;
  for (int i = 0; i < 4; ++i) out4[i] = v[i];
  return MLA_OK;
}

mla_status mla_selftest_wait_timeout(unsigned long long wait_ns, void* stream) {
  wait_selftest_kernel<<<1, 32, 0, as_stream(stream)>>>(wait_ns);
  return check_launch();
}

mla_status mla_project(const mla_dims* dims, const void* x, const void* w, void* y, int rows,
                       int in_f, int out_f, void* stream) {
  if (!dims_ok(dims) || rows < 0 || in_f < 1 || out_f < 1) return MLA_ERR_INVALID_ARG;
  if (rows == 0) return MLA_OK;
  if (!x || !w || !y) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  if (dims->dtype == MLA_F32) {
    SimtGemmArgs g{w, x, y, out_f, rows, in_f, 1, 0, in_f, 1, 0, in_f, 1, 0, out_f, 1, 0};
    return launch_simt_gemm<float, float>(g, st);
  }
  return launch_tc_gemm(w, false, 0, x, in_f, 0, out_f, rows, in_f, 1, y, 0, out_f, 1, kOutBf16,
                        st);
}

mla_status mla_absorb_q(const mla_dims* dims, const void* q, int q_stride_tok, const void* w_uk,
                        void* qbuf, int T, void* stream) {
  if (!dims_ok(dims) || T < 0) return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (!q || !w_uk || !qbuf) return MLA_ERR_INVALID_ARG;
  const int H = dims->n_heads, dn = dims->d_nope, dc = dims->d_latent, dr = dims->d_rope;
  const int dqk = dn + dr, D = dc + dr;
  if (q_stride_tok < H * dqk) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  if (dims->dtype == MLA_F32) {
    SimtGemmArgs g{w_uk, q, qbuf, dc, T, dn, H,
                   (long long)dn * dc, 1, dc,
                   dqk, q_stride_tok, 1,
                   D, (long long)H * D, 1, 0};
    return launch_simt_gemm<float, float>(g, st);
  }
  if ((dn % 16) != 0 || (dc % 128) != 0 || (q_stride_tok % 8) != 0 || (dqk % 8) != 0)
    return MLA_ERR_UNSUPPORTED;
  // A = W_UK[i] read as [K = d_nope][M = d_latent] (MN-major); X = q_nope of head i.
  return launch_tc_gemm(w_uk, true, (long long)dn * dc, q, q_stride_tok, dqk, dc, T, dn, H, qbuf,
                        D, (long long)H * D, 1, kOutBf16, st);
}

mla_status mla_rope(const mla_dims* dims, const void* x, int xs_tok, int xs_head, int n_heads_x,
                    void* y, int ys_tok, int ys_head, const int32_t* pos, int T, void* stream) {
  if (!dims_ok(dims) || T < 0 || n_heads_x < 0) return MLA_ERR_INVALID_ARG;
  if (T == 0 || n_heads_x == 0 || dims->d_rope == 0) return MLA_OK;
  if (!x || !y || !pos) return MLA_ERR_INVALID_ARG;
  const long long n =
      (long long)T * ((n_heads_x + kRopeGroup - 1) / kRopeGroup) * (dims->d_rope / 2);
  const int blk = 256;
  const long long grid = (n + blk - 1) / blk;
  cudaStream_t st = as_stream(stream);
  if (dims->dtype == MLA_F32)
    rope_kernel<float><<<(unsigned)grid, blk, 0, st>>>(
        static_cast<const float*>(x), xs_tok, xs_head, n_heads_x, static_cast<float*>(y), ys_tok,
        ys_head, pos, T, dims->d_rope, (double)dims->rope_base);
  else
    rope_kernel<__nv_bfloat16><<<(unsigned)grid, blk, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), xs_tok, xs_head, n_heads_x,
        static_cast<__nv_bfloat16*>(y), ys_tok, ys_head, pos, T, dims->d_rope,
        (double)dims->rope_base);
  return check_launch();
}

mla_status mla_cache_append(const mla_dims* dims, const void* c, int cs_tok, const void* kr,
                            int ks_tok, const int32_t* batch_idx, const int32_t* pos,
                            const int32_t* page_table, int max_pages, void* pool, int n_pages,
                            int T, void* stream) {
  if (!dims_ok(dims) || T < 0 || max_pages < 1 || n_pages < 1) return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (!c || !batch_idx || !pos || !page_table || !pool || (dims->d_rope > 0 && !kr))
    return MLA_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  if (dims->dtype == MLA_F32)
    append_kernel<uint32_t><<<T, 128, 0, st>>>(
        static_cast<const uint32_t*>(c), cs_tok, static_cast<const uint32_t*>(kr), ks_tok,
        batch_idx, pos, page_table, max_pages, static_cast<uint32_t*>(pool), n_pages,
        dims->page_size, dims->d_latent, dims->d_rope);
  else
    append_kernel<uint16_t><<<T, 128, 0, st>>>(
        static_cast<const uint16_t*>(c), cs_tok, static_cast<const uint16_t*>(kr), ks_tok,
        batch_idx, pos, page_table, max_pages, static_cast<uint16_t*>(pool), n_pages,
        dims->page_size, dims->d_latent, dims->d_rope);
  return check_launch();
}

static bool fp8_dims_ok(const mla_dims* d) {
  return d->dtype == MLA_BF16 && d->d_latent == fp8::kDC && d->d_rope == fp8::kDR;
}

mla_status mla_cache_append_fp8(const mla_dims* dims, const void* c, int cs_tok, const void* kr,
                                int ks_tok, const int32_t* batch_idx, const int32_t* pos,
                                const int32_t* page_table, int max_pages, void* pool8,
                                int n_pages, int T, void* stream) {
  if (!dims_ok(dims) || T < 0 || max_pages < 1 || n_pages < 1) return MLA_ERR_INVALID_ARG;
  if (!fp8_dims_ok(dims)) return MLA_ERR_UNSUPPORTED;
  if (T == 0) return MLA_OK;
  if (!c || !kr || !batch_idx || !pos || !page_table || !pool8) return MLA_ERR_INVALID_ARG;
  if (!aligned16(c) || !aligned16(kr) || !aligned16(pool8) || (cs_tok % 8) != 0 ||
      (ks_tok % 8) != 0)
    return MLA_ERR_INVALID_ARG;
  append_fp8_kernel<<<(T + 7) / 8, 256, 0, as_stream(stream)>>>(
      static_cast<const uint16_t*>(c), cs_tok, static_cast<const uint16_t*>(kr), ks_tok,
      batch_idx, pos, page_table, max_pages, static_cast<uint8_t*>(pool8), n_pages,
      dims->page_size, T);
  return check_launch();
}

mla_status mla_cache_quantize_fp8(const mla_dims* dims, const void* pool, void* pool8,
                                  int n_pages, void* stream) {
  if (!dims_ok(dims) || n_pages < 0) return MLA_ERR_INVALID_ARG;
  if (!fp8_dims_ok(dims)) return MLA_ERR_UNSUPPORTED;
  if (n_pages == 0) return MLA_OK;
  if (!pool || !pool8 || !aligned16(pool) || !aligned16(pool8)) return MLA_ERR_INVALID_ARG;
  const long long rows = (long long)n_pages * dims->page_size;
  quantize_pool_fp8_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, as_stream(stream)>>>(
      static_cast<const uint16_t*>(pool), static_cast<uint8_t*>(pool8), rows);
  return check_launch();
}

mla_status mla_pre_attention(const mla_dims* dims, void* y, int y_stride_tok, const void* w_uk,
                             void* qbuf, const int32_t* batch_idx, const int32_t* pos,
                             const int32_t* page_table, int max_pages, void* pool, int n_pages,
                             int T, void* stream) {
  if (!dims_ok(dims) || T < 0 || max_pages < 1 || n_pages < 1) return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (!y || !w_uk || !qbuf || !batch_idx || !pos || !page_table || !pool)
    return MLA_ERR_INVALID_ARG;
  const int H = dims->n_heads, dn = dims->d_nope, dc = dims->d_latent, dr = dims->d_rope;
  const int dqk = dn + dr;
  const long long off_c = (long long)H * dqk;
  if ((long long)y_stride_tok < off_c + dc + dr) return MLA_ERR_INVALID_ARG;
  const int D = dc + dr;
  if (dims->dtype == MLA_F32) {
    // the same four steps as separate launches
    char* yb = static_cast<char*>(y);
    const int es = 4;
    MLA_TRY(mla_rope(dims, yb + (long long)dn * es, y_stride_tok, dqk, H,
                     static_cast<char*>(qbuf) + (long long)dc * es, H * D, D, pos, T, stream));
    void* kr = yb + (off_c + dc) * es;
    MLA_TRY(mla_rope(dims, kr, y_stride_tok, 0, 1, kr, y_stride_tok, 0, pos, T, stream));
    MLA_TRY(mla_cache_append(dims, yb + off_c * es, y_stride_tok, kr, y_stride_tok, batch_idx,
                             pos, page_table, max_pages, pool, n_pages, T, stream));
    return mla_absorb_q(dims, y, y_stride_tok, w_uk, qbuf, T, stream);
  }
  // 16-byte pieces of the latent and 4-byte RoPE pairs in y, qbuf and the pool
  if ((y_stride_tok % 8) != 0 || (dc % 8) != 0 || (dr % 8) != 0 || (off_c % 8) != 0 ||
      (reinterpret_cast<uintptr_t>(y) & 15u) != 0 || (reinterpret_cast<uintptr_t>(pool) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(qbuf) & 3u) != 0)
    return MLA_ERR_UNSUPPORTED;
  if ((dn % 16) != 0 || (dc % 128) != 0 || (y_stride_tok % 8) != 0 || (dqk % 8) != 0)
    return MLA_ERR_UNSUPPORTED;
  PreAttnAux aux{};
  aux.y = static_cast<__nv_bfloat16*>(y);
  aux.ys_tok = y_stride_tok;
  aux.H = H; aux.d_nope = dn; aux.d_latent = dc; aux.d_rope = dr;
  aux.off_c = off_c;
  aux.qbuf = static_cast<__nv_bfloat16*>(qbuf);
  aux.batch_idx = batch_idx; aux.pos = pos; aux.page_table = page_table;
  aux.max_pages = max_pages;
  aux.pool = static_cast<uint16_t*>(pool);
  aux.n_pages = n_pages; aux.page_size = dims->page_size;
  aux.base = (double)dims->rope_base;
  aux.n_rope = (long long)T * (dr / 2) * ((H + kRopeHeadsPerItem - 1) / kRopeHeadsPerItem);
  aux.n_items = aux.n_rope + (long long)T * (dc / 8);
  // A1 on the GEMM CTAs, A2 and A3 on extra CTAs of the same launch
  return launch_tc_gemm(w_uk, true, (long long)dn * dc, y, y_stride_tok, dqk, dc, T, dn, H, qbuf,
                        D, (long long)H * D, 1, kOutBf16, as_stream(stream), &aux);
}

mla_status mla_decode_config(const mla_dims* dims, int S_q, int num_workers, int* kernel,
                             int* block_tokens, int* workers) {
  if (!dims_ok(dims) || S_q < 1 || S_q > 2 || num_workers < 0) return MLA_ERR_INVALID_ARG;
  const DecodeLayout L = decode_layout(dims, 1, S_q, num_workers);
  if (kernel) *kernel = use_tc_decode(dims, S_q) ? MLA_DECODE_KERNEL_TC : MLA_DECODE_KERNEL_SIMT;
  if (block_tokens) *block_tokens = use_tc_decode(dims, S_q) ? dtc::kBlk : kBlockTokensSimt;
  if (workers) *workers = L.G;
  return MLA_OK;
}

size_t mla_decode_workspace_size(const mla_dims* dims, int B, int S_q, int num_workers) {
  if (!dims_ok(dims) || B < 0 || S_q < 1 || num_workers < 0) return 0;
  return decode_layout(dims, B, S_q, num_workers).total;
}

static mla_status decode_impl(const mla_dims* dims, const void* qbuf, const void* pool, int n_pages,
                              const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                              const int32_t* tail, int B, int S_q, int num_workers,
                              void* workspace, size_t ws_bytes, float* o_lat, float* lse,
                              void* stream) {
  if (!dims_ok(dims) || B < 0 || S_q < 1 || S_q > 2 || num_workers < 0 || n_pages < 1 ||
      max_pages < 1)
    return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if (!qbuf || !pool || !page_table || !seq_lens || !workspace || !o_lat || !lse)
    return MLA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MLA_ERR_INVALID_ARG;
  if ((dims->d_latent % 4) != 0 || dims->d_latent > 512) return MLA_ERR_UNSUPPORTED;
  const DecodeLayout L = decode_layout(dims, B, S_q, num_workers);
  if (ws_bytes < L.total) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  char* ws = static_cast<char*>(workspace);
  int32_t* start = reinterpret_cast<int32_t*>(ws + L.off_start);
  float* ws_lse = reinterpret_cast<float*>(ws + L.off_lse);
  float* ws_o = reinterpret_cast<float*>(ws + L.off_o);
  const int max_tokens = max_pages * dims->page_size;
  const bool tc = use_tc_decode(dims, S_q);
  plan_kernel<<<1, 1024, 0, st>>>(seq_lens, tail, B, L.R, S_q, max_tokens,
                                  tc ? dtc::kBlk : kBlockTokensSimt, start);
  MLA_TRY(check_launch());
  const int H = dims->n_heads, dc = dims->d_latent, dr = dims->d_rope;
  if (tc) {
    if (!aligned16(qbuf) || !aligned16(pool)) return MLA_ERR_INVALID_ARG;
    MLA_TRY(launch_decode_tc_impl(make_tmap_bf16, qbuf, pool, n_pages, page_table, max_pages,
                                  seq_lens, tail, B, S_q, H, dims->scale, L.G, start, ws_lse,
                                  ws_o, st));
    g_launches.fetch_add(1, std::memory_order_relaxed);
  } else {
    dim3 grid(L.G, (L.rows_per_v + 7) / 8);
    const int kc = (dc + 31) / 32;
#define MLA_SIMT_DECODE(T, KC)                                                                 \
  decode_simt_kernel<T, KC><<<grid, 256, 0, st>>>(                                             \
      static_cast<const T*>(qbuf), static_cast<const T*>(pool), n_pages, page_table, max_pages, \
      seq_lens, tail, B, S_q, H, dc, dr, dims->page_size, dims->scale, L.G, kBlockTokensSimt,   \
      start, ws_lse, ws_o)
    if (dims->dtype == MLA_F32) {
      if (kc <= 2) MLA_SIMT_DECODE(float, 2);
      else if (kc <= 4) MLA_SIMT_DECODE(float, 4);
      else if (kc <= 8) MLA_SIMT_DECODE(float, 8);
      else MLA_SIMT_DECODE(float, 16);
    } else {
      if (kc <= 2) MLA_SIMT_DECODE(__nv_bfloat16, 2);
      else if (kc <= 4) MLA_SIMT_DECODE(__nv_bfloat16, 4);
      else if (kc <= 8) MLA_SIMT_DECODE(__nv_bfloat16, 8);
      else MLA_SIMT_DECODE(__nv_bfloat16, 16);
    }
#undef MLA_SIMT_DECODE
    MLA_TRY(check_launch());
  }
  const int wpr = combine_warps_per_row(L.V, L.G);
  dim3 cgrid(L.V, (L.rows_per_v * wpr + 7) / 8);
  combine_kernel<<<cgrid, kCombineThreads, 0, st>>>(ws_lse, ws_o, start, L.V, L.R, L.G,
                                                    L.rows_per_v, S_q * H, dc, wpr, o_lat, lse);
  return check_launch();
}

mla_status mla_decode(const mla_dims* dims, const void* qbuf, const void* pool, int n_pages,
                      const int32_t* page_table, int max_pages, const int32_t* seq_lens, int B,
                      int S_q, int num_workers, void* workspace, size_t ws_bytes, float* o_lat,
                      float* lse, void* stream) {
  return decode_impl(dims, qbuf, pool, n_pages, page_table, max_pages, seq_lens, nullptr, B, S_q,
                     num_workers, workspace, ws_bytes, o_lat, lse, stream);
}

// Workspace of mla_decode_fp8: mla_decode's layout (same split planning),
// then the half copy of the query, [B][S_q][H][576].
static size_t fp8_q16_offset(const mla_dims* dims, int B, int S_q, int num_workers) {
  return decode_layout(dims, B, S_q, num_workers).total;
}

size_t mla_decode_fp8_workspace_size(const mla_dims* dims, int B, int S_q, int num_workers) {
  if (!dims_ok(dims) || B < 0 || S_q < 1 || num_workers < 0 || !fp8_dims_ok(dims)) return 0;
  return fp8_q16_offset(dims, B, S_q, num_workers) +
         (((size_t)B * S_q * dims->n_heads * 576 * 2 + 255) & ~(size_t)255);
}

mla_status mla_decode_fp8(const mla_dims* dims, const void* qbuf, const void* pool8,
                          int n_pages, const int32_t* page_table, int max_pages,
                          const int32_t* seq_lens, int B, int S_q, int num_workers,
                          void* workspace, size_t ws_bytes, float* o_lat, float* lse,
                          void* stream) {
  if (!dims_ok(dims) || B < 0 || S_q < 1 || S_q > 2 || num_workers < 0 || n_pages < 1 ||
      max_pages < 1)
    return MLA_ERR_INVALID_ARG;
  if (!fp8_dims_ok(dims) || dims->page_size != 64) return MLA_ERR_UNSUPPORTED;
  if (B == 0) return MLA_OK;
  if (!qbuf || !pool8 || !page_table || !seq_lens || !workspace || !o_lat || !lse)
    return MLA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || !aligned16(qbuf) ||
      !aligned16(pool8))
    return MLA_ERR_INVALID_ARG;
  if (ws_bytes < mla_decode_fp8_workspace_size(dims, B, S_q, num_workers))
    return MLA_ERR_INVALID_ARG;
  const DecodeLayout L = decode_layout(dims, B, S_q, num_workers);
  cudaStream_t st = as_stream(stream);
  char* ws = static_cast<char*>(workspace);
  int32_t* start = reinterpret_cast<int32_t*>(ws + L.off_start);
  float* ws_lse = reinterpret_cast<float*>(ws + L.off_lse);
  float* ws_o = reinterpret_cast<float*>(ws + L.off_o);
  uint16_t* q16 = reinterpret_cast<uint16_t*>(ws + fp8_q16_offset(dims, B, S_q, num_workers));
  const long long nq = (long long)B * S_q * dims->n_heads * 576;
  bf16_to_f16_kernel<<<(unsigned)((nq / 8 + 255) / 256 + 1), 256, 0, st>>>(
      static_cast<const uint16_t*>(qbuf), q16, nq);
  MLA_TRY(check_launch());
  plan_kernel<<<1, 1024, 0, st>>>(seq_lens, nullptr, B, L.R, S_q, max_pages * dims->page_size,
                                  dfp::kBlk, start);
  MLA_TRY(check_launch());
  MLA_TRY(launch_decode_fp8_impl(make_tmap_f16, q16, pool8, n_pages, page_table, max_pages,
                                 seq_lens, nullptr, B, S_q, dims->n_heads, dims->scale, L.G,
                                 start, ws_lse, ws_o, st));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  const int wpr = combine_warps_per_row(L.V, L.G);
  dim3 cgrid(L.V, (L.rows_per_v * wpr + 7) / 8);
  combine_kernel<<<cgrid, kCombineThreads, 0, st>>>(ws_lse, ws_o, start, L.V, L.R, L.G,
                                                    L.rows_per_v, S_q * dims->n_heads,
                                                    dims->d_latent, wpr, o_lat, lse);
  return check_launch();
}

mla_status mla_decode_partial(const mla_dims* dims, const void* qbuf, const void* pool,
                              int n_pages, const int32_t* page_table, int max_pages,
                              const int32_t* seq_lens, const int32_t* seq_tail, int B, int S_q,
                              int num_workers, void* workspace, size_t ws_bytes, float* o_lat,
                              float* lse, void* stream) {
  if (!seq_tail && B > 0) return MLA_ERR_INVALID_ARG;
  return decode_impl(dims, qbuf, pool, n_pages, page_table, max_pages, seq_lens, seq_tail, B, S_q,
                     num_workers, workspace, ws_bytes, o_lat, lse, stream);
}

mla_status mla_combine_parts(const mla_dims* dims, const float* o_parts, const float* lse_parts,
                             int n_parts, int rows, float* o_lat, float* lse, void* stream) {
  if (!dims_ok(dims) || n_parts < 1 || rows < 0) return MLA_ERR_INVALID_ARG;
  if (rows == 0) return MLA_OK;
  if (!o_parts || !lse_parts || !o_lat || !lse) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  combine_parts_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
      o_parts, lse_parts, n_parts, rows, dims->d_latent, o_lat, lse);
  return check_launch();
}

// Split count of the W_O GEMM for T tokens (its fp32 partials live in the
// scratch).
static int w_o_splits(const mla_dims* d, int T) {
  return plan_tc_gemm(d->d_model, T, d->n_heads * d->d_v, 1, true).splits;
}

size_t mla_out_proj_scratch_size(const mla_dims* dims, int T) {
  if (!dims_ok(dims) || T < 0) return 0;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t H = dims->n_heads;
  if (dims->dtype == MLA_F32) return up((size_t)T * H * dims->d_v * 4);
  return up((size_t)T * H * dims->d_latent * 2) + up((size_t)T * H * dims->d_v * 2) +
         up((size_t)w_o_splits(dims, T) * T * dims->d_model * 4);
}

mla_status mla_out_proj(const mla_dims* dims, const float* o_lat, const void* w_uv,
                        const void* w_o, void* scratch, size_t scratch_bytes, float* out, int T,
                        void* stream) {
  if (!dims_ok(dims) || T < 0) return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (!o_lat || !w_uv || !w_o || !scratch || !out) return MLA_ERR_INVALID_ARG;
  if (scratch_bytes < mla_out_proj_scratch_size(dims, T)) return MLA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(scratch) & 255u) != 0) return MLA_ERR_INVALID_ARG;
  const int H = dims->n_heads, dc = dims->d_latent, dv = dims->d_v, dm = dims->d_model;
  cudaStream_t st = as_stream(stream);
  if (dims->dtype == MLA_F32) {
    float* o = static_cast<float*>(scratch);
    SimtGemmArgs g1{w_uv, o_lat, o, dv, T, dc, H,
                    (long long)dv * dc, dc, 1,
                    dc, (long long)H * dc, 1,
                    dv, (long long)H * dv, 1, 0};
    MLA_TRY((launch_simt_gemm<float, float>(g1, st)));
    SimtGemmArgs g2{w_o, o, out, dm, T, H * dv, 1, 0, (long long)H * dv, 1, 0, (long long)H * dv,
                    1, 0, dm, 1, 0};
    return launch_simt_gemm<float, float>(g2, st);
  }
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  __nv_bfloat16* olb = static_cast<__nv_bfloat16*>(scratch);
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(scratch) +
                                                      up((size_t)T * H * dc * 2));
  const long long n = (long long)T * H * dc;
  cast_f32_bf16_kernel<<<(unsigned)((n / 4 + 255) / 256 + 1), 256, 0, st>>>(o_lat, olb, n);
  MLA_TRY(check_launch());
  // o[t, i, :] = W_UV[i] o_lat[t, i, :]
  MLA_TRY(launch_tc_gemm(w_uv, false, (long long)dv * dc, olb, (long long)H * dc, dc, dv, T, dc, H,
                         o, dv, (long long)H * dv, 1, kOutBf16, st));
  // out[t, :] = W_O o[t, :]: split-K partials into the scratch, then their
  // ordered sum (deterministic: no atomics)
  float* parts = reinterpret_cast<float*>(reinterpret_cast<char*>(o) + up((size_t)T * H * dv * 2));
  int splits = 1;
  MLA_TRY(launch_tc_gemm(w_o, false, 0, o, (long long)H * dv, 0, dm, T, H * dv, 1, parts, 0, dm, 1,
                         kOutF32Split, st, nullptr, &splits));
  const long long n_out = (long long)T * dm;
  sum_splits_kernel<<<(unsigned)((n_out / 4 + 255) / 256 + 1), 256, 0, st>>>(parts, splits, n_out,
                                                                             out);
  return check_launch();
}

// ---------------------------------------------------------------------------
// chunked prefill (non-absorbed)
// ---------------------------------------------------------------------------
static bool prefill_dims_ok(const mla_dims* d) {
  return d->dtype == MLA_BF16 && d->d_nope == pfa::kDN && d->d_rope == pfa::kDR &&
         d->d_v == pfa::kDV && d->d_latent == pfa::kDC;
}

mla_status mla_prefill_rebuild_kv(const mla_dims* dims, const void* pool, int n_pages,
                                  const int32_t* page_row, int L, const void* w_uk,
                                  const void* w_uv, void* ctx, void* k_nope, void* v,
                                  void* stream) {
  if (!dims_ok(dims) || L < 0 || n_pages < 1) return MLA_ERR_INVALID_ARG;
  if (!prefill_dims_ok(dims)) return MLA_ERR_UNSUPPORTED;
  if (L == 0) return MLA_OK;
  if (!pool || !page_row || !w_uk || !w_uv || !ctx || !k_nope || !v) return MLA_ERR_INVALID_ARG;
  if (!aligned16(pool) || !aligned16(ctx) || !aligned16(k_nope) || !aligned16(v) ||
      !aligned16(w_uk) || !aligned16(w_uv))
    return MLA_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  const int H = dims->n_heads, D = pfa::kD;
  const int row_vecs = D * 2 / 16;
  const long long n = (long long)L * row_vecs;
  gather_rows_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
      static_cast<const uint4*>(pool), n_pages, dims->page_size, page_row, L, row_vecs,
      static_cast<uint4*>(ctx));
  MLA_TRY(check_launch());
  // k_nope[t][i*128 + n] = sum_c w_uk[i*128 + n][c] ctx[t][c]: A = w_uk as
  // [H*128][512] (K-major), X = the first 512 columns of ctx rows
  MLA_TRY(launch_tc_gemm(w_uk, false, 0, ctx, D, 0, H * pfa::kDN, L, pfa::kDC, 1, k_nope, 0,
                         (long long)H * pfa::kDN, 1, kOutBf16, st));
  return launch_tc_gemm(w_uv, false, 0, ctx, D, 0, H * pfa::kDV, L, pfa::kDC, 1, v, 0,
                        (long long)H * pfa::kDV, 1, kOutBf16, st);
}

mla_status mla_prefill_attention(const mla_dims* dims, const void* q, int q_stride_tok,
                                 const void* ctx, const void* k_nope, const void* v, int T,
                                 int L, void* o, float* lse, void* stream) {
  if (!dims_ok(dims) || T < 0 || L < T) return MLA_ERR_INVALID_ARG;
  if (!prefill_dims_ok(dims)) return MLA_ERR_UNSUPPORTED;
  if (T == 0) return MLA_OK;
  const int H = dims->n_heads;
  if (!q || !ctx || !k_nope || !v || !o || !lse) return MLA_ERR_INVALID_ARG;
  if (q_stride_tok < H * pfa::kDQK || (q_stride_tok % 8) != 0 || !aligned16(q) ||
      !aligned16(ctx) || !aligned16(k_nope) || !aligned16(v) || !aligned16(o))
    return MLA_ERR_INVALID_ARG;
  const mla_status s = launch_prefill_attn_impl(make_tmap_bf16, q, q_stride_tok, ctx, k_nope, v,
                                                T, L, H, dims->scale,
                                                static_cast<__nv_bfloat16*>(o), lse,
                                                as_stream(stream));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return s;
}

}  // extern "C"

// ===========================================================================
// Allocation-free decode: the workspace is a fixed array in this library's
// device memory instead of caller-provided scratch (see mla_decode_noalloc in
// include/mla.h for who needs this and the sharing rules).
// ===========================================================================
static __device__ __align__(256) unsigned char g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name only stands in for the symbol, so the address is looked
// up once per device (with that device current) and cached.
mla_status noalloc_scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return MLA_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" size_t mla_decode_noalloc_scratch_bytes(void) {
  return (size_t)MLA_NOALLOC_SCRATCH_BYTES;
}

extern "C" mla_status mla_decode_noalloc(const mla_dims* dims, const void* qbuf,
                                         const void* pool, int n_pages,
                                         const int32_t* page_table, int max_pages,
                                         const int32_t* seq_lens, int B, int S_q,
                                         int num_workers, float* o_lat, float* lse,
                                         void* stream) {
  if (!dims_ok(dims) || B < 0 || S_q < 1 || S_q > 2 || num_workers < 0)
    return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  const size_t need = mla_decode_workspace_size(dims, B, S_q, num_workers);
  if (need == 0 || need > (size_t)MLA_NOALLOC_SCRATCH_BYTES) return MLA_ERR_UNSUPPORTED;
  void* ws = nullptr;
  MLA_TRY(noalloc_scratch_address(&ws));
  return mla_decode(dims, qbuf, pool, n_pages, page_table, max_pages, seq_lens, B, S_q,
                    num_workers, ws, (size_t)MLA_NOALLOC_SCRATCH_BYTES, o_lat, lse, stream);
}
