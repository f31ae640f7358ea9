// decode_fp8.cuh -- split-KV decode on the 8-bit latent cache (fp8.cuh rows).
//
// Same attention as decode_tc.cuh (deepforge "DeepSeek-V2", §1 "Store a
// latent, rebuild the keys and values"; the 8-bit cache is the stretch goal
// of §4 "Build it yourself"), over rows that store the latent in E4M3 with a
// per-token scale s_t and the RoPE key in half precision.  The cache numbers a
// row stands for are [s_t c8_t ; k_rope_t].
//
// Work decomposition: as in decode_tc.cuh -- a CTA pair owns 128 query rows
// and runs pair MMAs (M = 128 rows, N = 256 tokens for QK, N = 256 latent
// columns for PV) over 256-token blocks, with the QK and PV tiles in two
// rings and one thread issuing MMAs from both streams as their operands land.
// The differences:
//   * The tensor cores compute in IEEE half precision (kind::f16 with f16
//     operands) on the stored numbers: Q is a half copy of the bf16 query
//     (exact), the E4M3 codes become halves exactly, and the RoPE part is
//     already stored divided by the row scale s_t.  So QK gives s_t-free dot
//     products, scaled by s_t in fp32 in the softmax; the value product takes
//     the weights 64 p_t s_t rounded to half (the 64 keeps them in half's
//     normal range and is divided out at the end).
//   * Eight converter warps fill both rings from the 8-bit pool: each reads
//     16 bytes (16 E4M3 codes) of a row, converts them to half pairs and
//     stores 32 bytes into the 128-byte-swizzled operand layout; the RoPE
//     part is copied.  Warps 4-7 build the QK stages, warps 8-11 the PV
//     stages: two pairs per ring take its stages in turn, and the two warps
//     of a pair split a stage.  Rows past the sequence are written as zeros.  In the peer
//     CTA, warp 1 lane 0 relays landed PV stages and warp 2 lane 0 landed QK
//     stages to the leader's barriers.
//   * Four softmax warps, one TMEM lane quadrant each, all 128 columns of a
//     lane (two pages).  They stage each block's 256 row scales in shared
//     memory one block ahead.
// The 8-bit rows halve the bytes read per token (656 instead of 1152).
//
// Shared memory: Q 72 KB + P 32 KB + QK ring 64 KB + PV ring 48 KB.
// Every wait is bounded (MLA_WAIT_NS) as in decode_tc.cuh, with the same
// drain on the way out.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"
#include "decode_tc.cuh"
#include "fp8.cuh"
#include "simt.cuh"

namespace mla {

// Blocks ahead of the converters whose pages are prefetched into L2 (0: none).
#ifndef MLA_FP8_PREFETCH_BLOCKS
#define MLA_FP8_PREFETCH_BLOCKS 2
#endif

namespace dfp {
constexpr int kRow = fp8::kRowBytes;     // 656 bytes per token
constexpr int kPage = 64;
constexpr int kBlk = 256;
constexpr int kPageBytes = kPage * kRow;
constexpr int kChunk = 8192;             // 64 rows x 64 columns half
constexpr int kQkStageBytes = 4 * kChunk;  // 2 chunks x 2 pages
constexpr int kQkStages = 2;
constexpr int kQkStagesPerBlock = 5;     // latent chunks {0,1} .. {6,7}, then the RoPE chunk
constexpr int kPvStageBytes = 2 * kChunk;
constexpr int kPvStages = 3;
constexpr int kPvStagesPerBlock = 8;
constexpr int kQBytes = 9 * kChunk;
constexpr int kPBytes = 4 * kChunk;
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffP = kOffQ + kQBytes;
constexpr uint32_t kOffQk = kOffP + kPBytes;
constexpr uint32_t kOffPv = kOffQk + kQkStages * kQkStageBytes;
constexpr uint32_t kSmemBytes = kOffPv + kPvStages * kPvStageBytes + 1024;
constexpr int kThreads = 512;
constexpr int kConvWarp0 = 4;
constexpr int kSoftmaxWarp0 = 12;
constexpr int kSoftmaxThreads = 128;
constexpr int kRegsLaunch = 128;
constexpr int kRegsControl = 64;
constexpr int kRegsConvert = 96;
constexpr int kRegsSoftmax = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;
constexpr uint32_t kTmemS = 256;
constexpr float kRescaleLog2 = 8.0f;
}  // namespace dfp

// Instruction descriptor, kind::f16 with f16 A/B and f32 D (A/B format 0).
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Two E4M3 bytes (lower byte -> lower half) to two halves.
__device__ __forceinline__ uint32_t f16x2_from_e4m3x2(uint16_t v) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(v));
  return r;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// 16 E4M3 values (one 16-byte piece of a row) as 8 half pairs (exact).
__device__ __forceinline__ void e4m3x16_to_f16(const uint4 raw, uint32_t (&o)[8]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    o[2 * q] = f16x2_from_e4m3x2((uint16_t)(w[q] & 0xFFFFu));
    o[2 * q + 1] = f16x2_from_e4m3x2((uint16_t)(w[q] >> 16));
  }
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// One warp: 128 latent columns (8 pieces of 16) of 32 tokens [32 half, +32)
// of one page, their E4M3 codes as halves (exact; the row scale is applied to
// the fp32 scores and to the softmax weights instead) in [2 chunks][64
// slots][128 B] at dst + chunk * chunk_stride (128-byte swizzle by slot).
// Rows t >= valid become zeros.
__device__ __forceinline__ void convert_page_cols(const uint8_t* page, int col_byte0, int valid,
                                                  uint32_t dst, uint32_t chunk_stride, int lane,
                                                  int half) {
  // All eight 16-byte loads of a lane are issued before the first
  // conversion: the rows come from HBM or L2, and a chain of dependent
  // rounds would leave the stage waiting several latencies.
  const int u = lane & 7, tq = lane >> 3;
  const int cc = u >> 2, unit = 2 * (u & 3);
  uint4 raw[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = 32 * half + 4 * i + tq;
    raw[i] = t < valid
                 ? __ldg(reinterpret_cast<const uint4*>(page + (size_t)t * dfp::kRow + col_byte0 +
                                                        16 * u))
                 : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = 32 * half + 4 * i + tq;
    const uint32_t row = dst + cc * chunk_stride + t * 128;
    const uint32_t a0 = row + (((unit) ^ (t & 7)) << 4);
    const uint32_t a1 = row + (((unit + 1) ^ (t & 7)) << 4);
    uint32_t o[8];
    e4m3x16_to_f16(raw[i], o);   // zero bytes convert to +0
    st_shared_v4(a0, o[0], o[1], o[2], o[3]);
    st_shared_v4(a1, o[4], o[5], o[6], o[7]);
  }
}

// One warp: the RoPE part (64 halves of k / s = one 128-byte row) of 64
// tokens of one page, copied into [64 slots][128 B] at dst (swizzled); rows
// t >= valid become zeros.
__device__ __forceinline__ void copy_page_rope(const uint8_t* page, int valid, uint32_t dst,
                                               int lane) {
  const int u = lane & 7, tq = lane >> 3;
  uint4 v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int t = 4 * i + tq;
    v[i] = t < valid ? __ldg(reinterpret_cast<const uint4*>(page + (size_t)t * dfp::kRow +
                                                            fp8::kOffRope + 16 * u))
                     : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int t = 4 * i + tq;
    st_shared_v4(dst + t * 128 + ((u ^ (t & 7)) << 4), v[i].x, v[i].y, v[i].z, v[i].w);
  }
}

struct DecodeFp8Params {
  const uint8_t* pool8;   // [n_pages][64][656]
  const int32_t* page_table;
  const int32_t* seq_lens;
  const int32_t* tail;
  const int32_t* start;
  float* ws_lse;
  float* ws_o;
  int n_pages, max_pages, B, S_q, H, R, G;
  float scale_log2;
};

__device__ __forceinline__ int page_of_fp8(const DecodeFp8Params& P, int b, int L, int x, int p,
                                           int& valid) {
  const int first = x * dfp::kBlk + p * dfp::kPage;
  valid = 0;
  if (first >= L) return -1;
  const int pg = P.page_table[(long long)b * P.max_pages + first / dfp::kPage];
  if (pg < 0 || pg >= P.n_pages) {
    raise_flag(kFlagBounds);
    return -1;
  }
  valid = min(L - first, dfp::kPage);
  return pg;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(dfp::kThreads, 1)
    decode_fp8_kernel(const __grid_constant__ CUtensorMap tmQ, const DecodeFp8Params P) {
  using namespace dfp;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t qk_full[kQkStages], qk_empty[kQkStages], qk_local[kQkStages];
  __shared__ __align__(8) uint64_t pv_full[kPvStages], pv_empty[kPvStages], pv_local[kPvStages];
  __shared__ __align__(8) uint64_t q_full, q_empty, o_empty, p_full, pv_done, mma_drain;
  __shared__ __align__(8) uint64_t s_full[2];
  __shared__ float red_max[2][2][64];
  __shared__ float red_sum[2][64];
  __shared__ __align__(16) float sc_buf[3][kBlk];  // row scales of a block's 256 tokens
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int worker = blockIdx.x >> 1;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base + kOffQ, sP = base + kOffP;
  const uint32_t sQk = base + kOffQk, sPv = base + kOffPv;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    // full: the MMA's view (leader: own converter warp + the peer's relay);
    // local: the peer's own converter warp, watched by its relay lane
    for (int s = 0; s < kQkStages; ++s) {
      mbar_init(smem_u32(&qk_full[s]), rank == 0 ? 3u : 1u);
      mbar_init(smem_u32(&qk_local[s]), 2);
      mbar_init(smem_u32(&qk_empty[s]), 1);
    }
    for (int s = 0; s < kPvStages; ++s) {
      mbar_init(smem_u32(&pv_full[s]), rank == 0 ? 3u : 1u);
      mbar_init(smem_u32(&pv_local[s]), 2);
      mbar_init(smem_u32(&pv_empty[s]), 1);
    }
    mbar_init(smem_u32(&q_full), 1);
    mbar_init(smem_u32(&q_empty), 1);
    mbar_init(smem_u32(&o_empty), 8);       // 4 softmax warps x 2 CTAs
    mbar_init(smem_u32(&p_full), 8);
    mbar_init(smem_u32(&pv_done), 1);
    mbar_init(smem_u32(&mma_drain), 1);
    mbar_init(smem_u32(&s_full[0]), 1);
    mbar_init(smem_u32(&s_full[1]), 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
  }
  if (warp == 1) {
    tmem_alloc<2>(smem_u32(&tmem_base_sh), kTmemCols);
    tmem_relinquish<2>();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_p = &abort_flag;

  const int V = P.B * P.R;
  const int total = P.start[V];
  const int lo = total > 0 ? worker_lo(worker, total, P.G) : 0;
  const int hi = total > 0 ? worker_lo(worker + 1, total, P.G) : 0;
  const int rows_seq = P.S_q * P.H;

  static_assert(128 * kRegsControl + 256 * kRegsConvert + 128 * kRegsSoftmax <=
                        kRegsLaunch * kThreads &&
                    kRegsLaunch * kThreads <= 65536,
                "register split exceeds the launch allocation");
  if (warp < kConvWarp0) {
    setmaxnreg_dec<kRegsControl>();
    if (warp == 0 && lane == 0) {
      // ==========  Q slices (one TMA load per piece)  ==========
      const uint32_t lead_qfull = mapa_shared(smem_u32(&q_full), 0);
      uint32_t q_issued = 0;
      PieceIter pi;
      pi.init(P.start, V, lo, hi);
      int v, x0, x1, piece = 0;
      while (pi.next(v, x0, x1)) {
        const int b = v % P.B, rb = v / P.B;
        if (piece > 0 && !mbar_wait(smem_u32(&q_empty), (piece - 1) & 1, abort_p, 2, piece)) break;
        if (rank == 0) mbar_expect_tx(smem_u32(&q_full), 2 * kQBytes);
        const int row0 = b * rows_seq + rb * 128 + 64 * (int)rank;
        for (int c = 0; c < 9; ++c)
          tma_load_2d_pair(sQ + c * kChunk, &tmQ, c * 64, row0, lead_qfull);
        ++q_issued;
        ++piece;
      }
      if (*abort_p && rank == 0 && q_issued > 0)
        mbar_wait_bounded(smem_u32(&q_full), (q_issued - 1) & 1, kDrainNs);
    } else if ((warp == 1 || warp == 2) && lane == 0 && rank == 1) {
      // ======  peer relays: landed stages to the leader's barriers  ======
      // (warp 1: PV stages, warp 2: QK stages)
      const bool pv = (warp == 1);
      const int per_block = pv ? kPvStagesPerBlock : kQkStagesPerBlock;
      const int nst = pv ? kPvStages : kQkStages;
      uint64_t* local = pv ? pv_local : qk_local;
      uint64_t* full = pv ? pv_full : qk_full;
      const uint32_t lead0 = mapa_shared(smem_u32(&full[0]), 0);
      PieceIter pi;
      pi.init(P.start, V, lo, hi);
      int v, x0, x1;
      uint32_t it = 0;
      bool ok = true;
      while (ok && pi.next(v, x0, x1))
        for (int x = x0; x < x1 && ok; ++x)
          for (int k = 0; k < per_block; ++k, ++it) {
            const int s = it % nst;
            if (!mbar_wait(smem_u32(&local[s]), (it / nst) & 1, abort_p, pv ? 14 : 15, it)) {
              ok = false;
              break;
            }
            fence_proxy_async_smem();
            mbar_arrive_cluster(lead0 + s * 8);
          }
    } else if (warp == 1 && lane == 0 && rank == 0) {
      // =================  MMA issuer (leader CTA)  =================
      // The two-stream scheduler of decode_tc.cuh, on half operands.  The
      // QK stages are [chunk][page][64 slots][128 B]: the 16 slot groups of
      // one chunk are 1 KB apart.
      const uint32_t idesc_qk = idesc_f16_f32(128, 256, false, false);
      const uint32_t idesc_pv = idesc_f16_f32(128, 256, false, true);
      const uint64_t q_desc = sw128_desc(sQ, 16, 1024);
      const uint64_t p_desc = sw128_desc(sP, 16, 1024);
      const uint64_t qk_desc = sw128_desc(sQk, 16, 1024);
      const uint64_t pv_desc = sw128_desc(sPv, kChunk, 1024);
      PieceIter qi, vi;
      qi.init(P.start, V, lo, hi);
      vi.init(P.start, V, lo, hi);
      int qv, qx0 = 0, qx1 = 0, vv, vx0 = 0, vx1 = 0;
      bool q_more = qi.next(qv, qx0, qx1), v_more = vi.next(vv, vx0, vx1);
      int qx = qx0, q_piece = 0, jq = 0, kq = 0;
      bool q_in = false;
      int vx = vx0, v_piece = 0, jp = 0, tp = 0;
      bool p_in = false;
      uint32_t itq = 0, itv = 0;
      bool ok = true;
      uint64_t t_stall = 0;
      uint32_t spins = 0;
      while (ok && (q_more || v_more)) {
        bool progressed = false;
        if (q_more && jq <= jp + (p_in ? 1 : 0) + 1) {
          bool ready = true;
          if (!q_in) {
            ready = mbar_try_wait(smem_u32(&q_full), q_piece & 1);
            if (ready) q_in = true;
          }
          const int s = itq % kQkStages;
          if (ready && mbar_try_wait(smem_u32(&qk_full[s]), (itq / kQkStages) & 1)) {
            fence_proxy_async_smem();
            tc_fence_after();
            const uint32_t sd = tmem + kTmemS + 128 * (jq & 1);
            const uint64_t b0 = qk_desc + (uint64_t)s * (kQkStageBytes >> 4);
            const int ncc = (kq == kQkStagesPerBlock - 1) ? 1 : 2;
            for (int cc = 0; cc < ncc; ++cc) {
              const int c = 2 * kq + cc;
              const uint64_t a0 = q_desc + (uint64_t)((c * kChunk) >> 4);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss<2>(sd, a0 + (uint64_t)((kk * 32) >> 4),
                               b0 + (uint64_t)((cc * 2 * kChunk + kk * 32) >> 4), idesc_qk,
                               (c | kk) ? 1u : 0u);
            }
            mma_commit_2_mc(smem_u32(&qk_empty[s]), 3);
            ++itq;
            progressed = true;
            if (++kq == kQkStagesPerBlock) {
              kq = 0;
              mma_commit_2_mc(smem_u32(&s_full[jq & 1]), 3);
              ++jq;
              if (++qx == qx1) {
                mma_commit_2_mc(smem_u32(&q_empty), 3);
                q_more = qi.next(qv, qx0, qx1);
                qx = qx0;
                ++q_piece;
                q_in = false;
              }
            }
          }
        }
        if (v_more && jp < jq) {
          if (!p_in) {
            p_in = mbar_try_wait(smem_u32(&p_full), jp & 1) &&
                   (vx != vx0 || v_piece == 0 ||
                    mbar_try_wait(smem_u32(&o_empty), (v_piece - 1) & 1));
            if (p_in) tc_fence_after();
          }
          const int s = itv % kPvStages;
          if (p_in && mbar_try_wait(smem_u32(&pv_full[s]), (itv / kPvStages) & 1)) {
            fence_proxy_async_smem();
            tc_fence_after();
            const int p = tp >> 1, n = tp & 1;
            const bool first = (vx == vx0);
            const uint64_t a0 = p_desc + (uint64_t)((p * kChunk) >> 4);
            const uint64_t b0 = pv_desc + (uint64_t)s * (kPvStageBytes >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t acc = (first && p == 0 && kk == 0) ? 0u : 1u;
              mma_bf16_ss<2>(tmem + kTmemO + 128 * n, a0 + (uint64_t)((kk * 32) >> 4),
                             b0 + (uint64_t)((kk * 2048) >> 4), idesc_pv, acc);
            }
            mma_commit_2_mc(smem_u32(&pv_empty[s]), 3);
            ++itv;
            progressed = true;
            if (++tp == kPvStagesPerBlock) {
              tp = 0;
              mma_commit_2_mc(smem_u32(&pv_done), 3);
              ++jp;
              p_in = false;
              if (++vx == vx1) {
                v_more = vi.next(vv, vx0, vx1);
                vx = vx0;
                ++v_piece;
              }
            }
          }
        }
        if (progressed) {
          spins = 0;
        } else if ((++spins & 63u) == 0) {
          const uint64_t now = globaltimer();
          if (spins == 64) t_stall = now;
          if (*abort_p) {
            ok = false;
          } else if (now - t_stall > MLA_WAIT_NS) {
            raise_flag(kFlagTimeout);
            record_timeout(3, (uint32_t)jq, (uint32_t)jp);
            *abort_p = 1;
            ok = false;
          }
        }
      }
      if (!ok) {
        mma_commit_2_mc(smem_u32(&mma_drain), 1);
        mbar_wait_bounded(smem_u32(&mma_drain), 0, kDrainNs);
      }
    }
  } else if (warp < kSoftmaxWarp0) {
    setmaxnreg_dec<kRegsConvert>();
    // ==========  converters: 8-bit rows -> half operand tiles  ==========
    // eight converter warps: four per ring, two pairs taking the ring's
    // stages in turn; the two warps of a pair split a stage (QK: one page
    // each; PV: 32 of the page's 64 tokens each)
    const int cv = warp - kConvWarp0;
    const bool qk = cv < 4;
    const int mine = (cv >> 1) & 1;
    const int half = cv & 1;
    const int per_block = qk ? kQkStagesPerBlock : kPvStagesPerBlock;
    const int nst = qk ? kQkStages : kPvStages;
    uint64_t* empty = qk ? qk_empty : pv_empty;
    // the leader's converters complete the MMA's barrier directly; the
    // peer's complete a local one that its relay forwards
    uint64_t* done = (rank == 0) ? (qk ? qk_full : pv_full) : (qk ? qk_local : pv_local);
    PieceIter pi;
    pi.init(P.start, V, lo, hi);
    int v, x0, x1;
    uint32_t it = 0;
    bool ok = true;
    while (ok && pi.next(v, x0, x1)) {
      const int b = v % P.B;
      const int L = P.seq_lens[b];
      for (int x = x0; x < x1 && ok; ++x)
        for (int k = 0; k < per_block; ++k, ++it) {
          if ((int)(it & 1) != mine) continue;
          const int s = it % nst;
          const bool got = mbar_wait(smem_u32(&empty[s]), ((it / nst) & 1) ^ 1, abort_p, 11, it);
          if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
          if (qk) {
            // The converters wait out each load's latency.  An 8-bit page is
            // one contiguous range, so the first QK stage of a block asks
            // for this CTA's two pages of block x + MLA_FP8_PREFETCH_BLOCKS
            // to be brought into L2 (the peer asks for the other two; PV
            // reads all four).
            if (MLA_FP8_PREFETCH_BLOCKS > 0 && k == 0 && lane == 0 &&
                x + MLA_FP8_PREFETCH_BLOCKS < x1) {
              int vf;
              const int pf = page_of_fp8(P, b, L, x + MLA_FP8_PREFETCH_BLOCKS,
                                         2 * (int)rank + half, vf);
              if (pf >= 0)
                prefetch_l2_bulk(P.pool8 + (size_t)pf * kPageBytes, (uint32_t)kPageBytes);
            }
            const uint32_t dst = sQk + s * kQkStageBytes;
            // this warp's page of the stage: page 2r + half
            int valid;
            const int pg = page_of_fp8(P, b, L, x, 2 * (int)rank + half, valid);
            const uint8_t* page = P.pool8 + (size_t)(pg < 0 ? 0 : pg) * kPageBytes;
            if (k < kQkStagesPerBlock - 1) {
              // latent chunks 2k, 2k+1: row bytes [128k, 128k + 128)
              convert_page_cols(page, 128 * k, valid, dst + half * kChunk, 2 * kChunk, lane, 0);
              convert_page_cols(page, 128 * k, valid, dst + half * kChunk, 2 * kChunk, lane, 1);
            } else {
              copy_page_rope(page, valid, dst + half * kChunk, lane);
            }
          } else {
            // page p = k / 2, latent half n = k % 2: columns [256n + 128r, +128)
            const int p = k >> 1, n = k & 1;
            int valid;
            const int pg = page_of_fp8(P, b, L, x, p, valid);
            const uint8_t* page = P.pool8 + (size_t)(pg < 0 ? 0 : pg) * kPageBytes;
            convert_page_cols(page, 256 * n + 128 * (int)rank, valid,
                              sPv + s * kPvStageBytes, kChunk, lane, half);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&done[s]));
        }
    }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    // =================  softmax + epilogue (both CTAs)  =================
    const int quad = warp - kSoftmaxWarp0;
    const int tl = 32 * quad + lane;
    const int h = tl & 63, hh = tl >> 6;     // row, token half (pages 2hh, 2hh+1)
    const uint32_t lane_addr = (uint32_t)(32 * quad) << 16;
    const uint32_t lead_pfull = mapa_shared(smem_u32(&p_full), 0);
    const uint32_t lead_oempty = mapa_shared(smem_u32(&o_empty), 0);
    PieceIter pi;
    pi.init(P.start, V, lo, hi);
    int v, x0, x1;
    int j = 0;
    bool dead = false;
    while (!dead && pi.next(v, x0, x1)) {
      const int b = v % P.B, rb = v / P.B;
      const int L = P.seq_lens[b];
      const int grow = rb * 128 + 64 * (int)rank + h;
      const int tail = P.tail != nullptr ? P.tail[b] : 0;
      const int limit = min(L, L + tail - P.S_q + grow / P.H + 1);
      float m = -INFINITY, l = 0.f;
      bool o_started = false;
      // row scales of block xb's tokens tl and tl + 128 into sc_buf[buf]
      auto load_scales = [&](int xb, int buf) {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int u = tl + 128 * k;
          int valid;
          const int pg = page_of_fp8(P, b, L, xb, u >> 6, valid);
          const int t = u & 63;
          sc_buf[buf][u] = t < valid ? __ldg(reinterpret_cast<const float*>(
                                           P.pool8 + (size_t)pg * kPageBytes + (size_t)t * kRow +
                                           fp8::kOffScale))
                                     : 0.f;
        }
      };
      for (int x = x0; x < x1; ++x, ++j) {
        if (x == x0) {
          load_scales(x, j % 3);
          named_bar_sync(1, kSoftmaxThreads);
        }
        const bool got = mbar_wait(smem_u32(&s_full[j & 1]), (j >> 1) & 1, abort_p, 7, j);
        float mx = -INFINITY;
        const float* sc = sc_buf[j % 3] + 128 * hh;   // scales of this lane's 128 tokens
        // columns [64 ch, 64 ch + 64) of this lane are page 2 hh + ch
        const int cbase = limit - (x * kBlk + 2 * hh * kPage);   // visible: col < cbase
        const uint32_t sa = tmem + lane_addr + kTmemS + 128 * (j & 1);
        if (__all_sync(0xffffffffu, got)) {
          tc_fence_after();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t r[32];
            tmem_ld32(sa + 32 * q4, r);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (32 * q4 + c < cbase) mx = fmaxf(mx, __uint_as_float(r[c]) * sc[32 * q4 + c]);
          }
        }
        // the next block's scales, read after the barrier below
        if (x + 1 < x1) load_scales(x + 1, (j + 1) % 3);
        red_max[j & 1][hh][h] = mx;
        if (named_bar_or(1, kSoftmaxThreads, !got || *abort_p)) { dead = true; break; }
        mx = fmaxf(mx, red_max[j & 1][hh ^ 1][h]);
        const float m_blk = mx * P.scale_log2;
        const bool need = m_blk > m + kRescaleLog2 || (m == -INFINITY && m_blk > -INFINITY);
        const float alpha = !need ? 1.f : (m == -INFINITY ? 0.f : ex2_approx(m - m_blk));
        const float m_use = need ? m_blk : m;
        uint32_t pk[64];
        float lsum = 0.f;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t r[32];
          tmem_ld32(sa + 32 * q4, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c0 = 32 * q4 + 2 * e;
            const float s0 = sc[c0], s1 = sc[c0 + 1];
            const float p0 = c0 < cbase ? ex2_approx(fmaf(__uint_as_float(r[2 * e]) * s0,
                                                          P.scale_log2, -m_use))
                                        : 0.f;
            const float p1 = c0 + 1 < cbase ? ex2_approx(fmaf(__uint_as_float(r[2 * e + 1]) * s1,
                                                              P.scale_log2, -m_use))
                                            : 0.f;
            lsum += p0 + p1;
            // the value product's weights: 64 p s, the 64 keeping them in
            // half's normal range (divided out in the epilogue)
            pk[16 * q4 + e] = pack_f16x2(64.f * p0 * s0, 64.f * p1 * s1);
          }
        }
        bool ok = true;
        if (j > 0) ok = mbar_wait(smem_u32(&pv_done), (j - 1) & 1, abort_p, 8, j);
        if (__all_sync(0xffffffffu, ok)) {
          if (o_started && __any_sync(0xffffffffu, need)) {
            tc_fence_after();
            for (int cc = 0; cc < 8; ++cc) {
              uint32_t r[32];
              const uint32_t oa = tmem + lane_addr + kTmemO + 32 * cc;
              tmem_ld32(oa, r);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i)
                r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
              tmem_st32(oa, r);
            }
            tmem_wait_st();
          }
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            const uint32_t prow = sP + (2 * hh + ch) * kChunk + h * 128;
#pragma unroll
            for (int u = 0; u < 8; ++u)
              st_shared_v4(prow + ((u ^ (h & 7)) << 4), pk[32 * ch + 4 * u],
                           pk[32 * ch + 4 * u + 1], pk[32 * ch + 4 * u + 2],
                           pk[32 * ch + 4 * u + 3]);
          }
        }
        l = need ? l * alpha + lsum : l + lsum;
        m = m_use;
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(lead_pfull);
        o_started = true;
      }
      if (dead) break;
      const int jl = j - 1;
      const bool got = mbar_wait(smem_u32(&pv_done), jl & 1, abort_p, 10, jl);
      red_sum[hh][h] = l;
      if (named_bar_or(1, kSoftmaxThreads, !got || *abort_p)) { dead = true; break; }
      tc_fence_after();
      const float lt = red_sum[0][h] + red_sum[1][h];
      const float inv = lt > 0.f ? 1.f / (64.f * lt) : 0.f;
      const long long slot = (long long)worker + v;
      const long long row = slot * 128 + 64 * (int)rank + h;
      for (int n = 0; n < 2; ++n) {
        float* dst = P.ws_o + row * 512 + 256 * n + 128 * hh;
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_addr + kTmemO + 128 * n + 32 * cc, r);
          tmem_wait_ld();
          float4* d4 = reinterpret_cast<float4*>(dst + 32 * cc);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            d4[i] = make_float4(__uint_as_float(r[4 * i]) * inv,
                                __uint_as_float(r[4 * i + 1]) * inv,
                                __uint_as_float(r[4 * i + 2]) * inv,
                                __uint_as_float(r[4 * i + 3]) * inv);
        }
      }
      if (hh == 0)
        P.ws_lse[row] = lt > 0.f ? (m + log2f(lt)) * 0.69314718055994531f : -INFINITY;
      named_bar_sync(1, kSoftmaxThreads);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(lead_oempty);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) tmem_dealloc<2>(tmem, kTmemCols);
}

// bf16 -> half, elementwise (the query's exact half copy).
__global__ void bf16_to_f16_kernel(const uint16_t* x, uint16_t* y, long long n) {
  long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (i + 7 < n) {
    const uint4 v = *reinterpret_cast<const uint4*>(x + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) o[k] = pack_f16x2(bf16_lo(w[k]), bf16_hi(w[k]));
    *reinterpret_cast<uint4*>(y + i) = make_uint4(o[0], o[1], o[2], o[3]);
  } else {
    for (; i < n; ++i) {
      __half hv = __float2half_rn(__uint_as_float((uint32_t)x[i] << 16));
      y[i] = *reinterpret_cast<uint16_t*>(&hv);
    }
  }
}

inline mla_status launch_decode_fp8_impl(
    bool (*make_tmap_f16)(CUtensorMap*, const void*, int, const uint64_t*, const uint64_t*,
                          const uint32_t*),
    const void* q16, const void* pool8, int n_pages, const int32_t* page_table, int max_pages,
    const int32_t* seq_lens, const int32_t* tail, int B, int S_q, int H, float scale, int G,
    const int32_t* start, float* ws_lse, float* ws_o, cudaStream_t st) {
  using namespace dfp;
  CUtensorMap tQ;
  {
    const uint64_t dims[2] = {576, (uint64_t)B * S_q * H};
    const uint64_t strides[1] = {576 * 2};
    const uint32_t box[2] = {64, 64};
    if (!make_tmap_f16(&tQ, q16, 2, dims, strides, box)) return MLA_ERR_CUDA;
  }
  DecodeFp8Params p;
  p.pool8 = static_cast<const uint8_t*>(pool8);
  p.page_table = page_table;
  p.seq_lens = seq_lens;
  p.tail = tail;
  p.start = start;
  p.ws_lse = ws_lse;
  p.ws_o = ws_o;
  p.n_pages = n_pages;
  p.max_pages = max_pages;
  p.B = B;
  p.S_q = S_q;
  p.H = H;
  p.R = (S_q * H + 127) / 128;
  p.G = G;
  p.scale_log2 = scale * 1.4426950408889634f;
  if (cudaFuncSetAttribute(decode_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBytes) != cudaSuccess)
    return MLA_ERR_CUDA;
  decode_fp8_kernel<<<2 * G, kThreads, kSmemBytes, st>>>(tQ, p);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
