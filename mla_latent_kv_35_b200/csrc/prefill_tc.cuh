// prefill_tc.cuh -- chunked prefill without absorption: causal attention of
// T new queries of one sequence over its L cached tokens with the keys and
// values rebuilt per head (tcgen05 pair MMAs, TMEM accumulators, TMA).
//
// What it computes (deepforge "DeepSeek-V2", §1 "Store a latent, rebuild the
// keys and values"): head h's key of cached token t is
// k_{h,t} = [W_UK[h] c_t ; k_rope_t] (128 + 64 numbers) and its value is
// v_{h,t} = W_UV[h] c_t (128).  When many queries share a tile, rebuilding
// k and v once per (head, token) and reusing them across all queries costs
// less than attending in the 576-wide latent space per query, which is why
// a prefill chunk takes this form while decode stays absorbed.  Query i of
// the chunk sits at position L - T + i and sees tokens t <= L - T + i.
//
// Two kernels:
//   * gather_rows_kernel copies the sequence's cache rows, page by page, to
//     a contiguous [L][576] buffer (the B operand of the rebuild GEMMs and
//     the source of the shared RoPE keys).
//   * prefill_attn_kernel: flash attention over the rebuilt k and v.
//
// prefill_attn_kernel work decomposition
//   * A cluster of two CTAs owns 256 query rows of one head: CTA r holds rows
//     [128r, 128r + 128) of the tile (Q: 128 rows x 192 columns, 48 KB).
//   * Blocks of 128 keys.  QK: pair MMAs (cta_group::2, M = 256, N = 128,
//     K = 192); CTA r supplies keys [64r, 64r + 64) of the block (k_nope from
//     the rebuilt keys, k_rope from the gathered rows), so each SM streams
//     half of every key block.  S lands in TMEM with lane = row, the 128
//     keys in 128 columns.
//   * PV: pair MMAs (M = 256, N = 128 value columns, K = 128 keys).  A is P
//     in TMEM (bf16 pairs over the first 64 columns of S, in place; in a
//     pair MMA output lane l of CTA r reads its A row from TMEM lane l of CTA
//     r).  CTA r supplies value columns [64r, 64r + 64) of all 128 keys
//     (MN-major B).
//   * TMEM: O at columns [0, 128) and three S/P buffers at [128, 512): QK
//     runs up to three blocks ahead of the softmax; QK(j + 3) reuses the
//     buffer of P(j) once PV(j) has completed.
//   * Shared memory: Q 48 KB + five 24 KB key stages + three 16 KB value
//     stages = 216 KB.  In each CTA lane 0 of warp 0 loads Q and its key
//     halves, lane 0 of warp 2 its value halves; the leader arms every full
//     barrier with both CTAs' bytes.  A key stage is released by a commit
//     after the QK of its block, a value stage after the PV.
//   * Softmax: eight warps per CTA.  Warps w and w + 4 share TMEM lane
//     quadrant w and take 64 of the 128 keys each, so a thread holds one
//     row's scores of one key half; the two halves' maxima meet in shared
//     memory, each warp pair on a named barrier of its own.  Blocks off the
//     causal diagonal take a path without masks; maxima and row sums run in
//     independent chains, scores go through the packed fp32 FMA, and a share
//     of the exponentials is evaluated on the FMA pipe (exp2_poly2).  The
//     running max is rescaled lazily (O in TMEM is rescaled only when a row's
//     max grows by more than 2^8, after PV(j - 1)).
//   * Two threads of the leader issue the MMAs: lane 0 of warp 1 the QK
//     stream, lane 0 of warp 3 the PV stream, so that neither stream's
//     barrier waits hold up the other's MMAs.
//   * Epilogue: O / l in bf16 to o[t][h][0..128) and the natural-log LSE to
//     lse[t][h] for the rows t < T.
//
// Out-of-range rows and keys.  Query rows past T and keys past L load as
// zeros (TMA out-of-bounds fill): their scores are finite, the keys are
// causally hidden from every row t < T, and rows past T are not stored.
//
// Every mbarrier wait is bounded (MLA_WAIT_NS); on expiry the kernel raises
// MLA_ERR_TIMEOUT in the device status and every role leaves its loop; the
// leader's producer waits (bounded) for the copies it armed and the issuer
// for a last commit of its own before the pair frees its TMEM.
#pragma once

#include "common.cuh"
#include "decode_tc.cuh"

namespace mla {

namespace pfa {
constexpr int kDN = 128;             // d_nope
constexpr int kDR = 64;              // d_rope
constexpr int kDQK = kDN + kDR;      // 192
constexpr int kDV = 128;             // d_v
constexpr int kDC = 512;             // latent width
constexpr int kD = 576;              // cached numbers per token
constexpr int kRows = 128;           // query rows per CTA
constexpr int kBlk = 128;            // keys per block
constexpr int kChunkQ = kRows * 128;         // 128 rows x 64 columns bf16 (16 KB)
constexpr int kQBytes = 3 * kChunkQ;         // 48 KB
constexpr int kChunkK = (kBlk / 2) * 128;    // 64 keys x 64 columns (8 KB)
constexpr int kKBytes = 3 * kChunkK;         // this CTA's key half (24 KB)
constexpr int kVBytes = kBlk * 128;          // 128 keys x 64 value columns (16 KB)
#ifndef MLA_PREFILL_KSTAGES
#define MLA_PREFILL_KSTAGES 5
#endif
#ifndef MLA_PREFILL_VSTAGES
#define MLA_PREFILL_VSTAGES 3
#endif
constexpr int kKStages = MLA_PREFILL_KSTAGES;   // 24 KB key stages
constexpr int kVStages = MLA_PREFILL_VSTAGES;   // 16 KB value stages
constexpr int kSBufs = 3;            // S/P buffers in TMEM
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kQBytes;
constexpr uint32_t kOffV = kOffK + kKStages * kKBytes;
constexpr uint32_t kSmemBytes = kOffV + kVStages * kVBytes + 1024;  // + alignment
constexpr int kThreads = 384;
constexpr int kSoftmaxWarp0 = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;
constexpr uint32_t kTmemS = 128;     // S_b / P_b at [128 + 128b, +128), b < 3
constexpr float kRescaleLog2 = 8.0f;
}  // namespace pfa

// One pair of exponentials in MLA_EXP2_POLY_EVERY goes to exp2_poly2 (0: none).
#ifndef MLA_EXP2_POLY_EVERY
#define MLA_EXP2_POLY_EVERY 4
#endif


struct PrefillParams {
  __nv_bfloat16* o;   // [T][H][128]
  float* lse;         // [T][H]
  int T, L, H;
  float scale_log2;   // softmax scale * log2(e)
};

// ---------------------------------------------------------------------------
// ctx[t][:] = pool row of token t (page page_row[t / page], slot t % page).
// One thread per 16 bytes.  A page id outside the pool raises
// MLA_ERR_BOUNDS and leaves the row zero.
// ---------------------------------------------------------------------------
__global__ void gather_rows_kernel(const uint4* pool, int n_pages, int page_size,
                                   const int32_t* page_row, int L, int row_vecs, uint4* ctx) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)L * row_vecs) return;
  const int t = (int)(i / row_vecs), u = (int)(i % row_vecs);
  const int pg = page_row[t / page_size];
  if (pg < 0 || pg >= n_pages) {
    if (u == 0) raise_flag(kFlagBounds);
    ctx[i] = make_uint4(0, 0, 0, 0);
    return;
  }
  ctx[i] = pool[((long long)pg * page_size + t % page_size) * row_vecs + u];
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pfa::kThreads, 1)
    prefill_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmKR,
                        const __grid_constant__ CUtensorMap tmV, const PrefillParams P) {
  using namespace pfa;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t k_full[kKStages], k_empty[kKStages];
  __shared__ __align__(8) uint64_t v_full[kVStages], v_empty[kVStages];
  __shared__ __align__(8) uint64_t q_full, s_full[kSBufs], s_free[kSBufs], p_full[kSBufs];
  __shared__ __align__(8) uint64_t o_final, drain_qk, drain_pv;
  __shared__ float red_max[2][2][kRows];   // [block & 1][key half][row]
  __shared__ float red_l[2][kRows];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int h = blockIdx.y;
  const int n_pt = (P.T + 2 * kRows - 1) / (2 * kRows);
  const int pt = n_pt - 1 - (int)(blockIdx.x >> 1);     // longest tiles first
  const int r0 = pt * 2 * kRows;                        // first query row of the pair
  const int L0 = P.L - P.T;                             // position of query row 0
  // keys the pair needs: t < min(L, L0 + r0 + 256)
  const int kend = min(P.L, L0 + r0 + 2 * kRows);
  const int nblk = (kend + kBlk - 1) / kBlk;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base + kOffQ, sK = base + kOffK, sV = base + kOffV;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    // full barriers: the leader's arrive.expect_tx with both CTAs' bytes;
    // empty barriers: an MMA commit multicast to both CTAs
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(smem_u32(&k_full[s]), 1);
      mbar_init(smem_u32(&k_empty[s]), 1);    // after QK of the stage's block
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(smem_u32(&v_full[s]), 1);
      mbar_init(smem_u32(&v_empty[s]), 1);    // after PV of the stage's block
    }
    mbar_init(smem_u32(&q_full), 1);
    for (int b = 0; b < kSBufs; ++b) {
      mbar_init(smem_u32(&s_full[b]), 1);     // QK commit
      mbar_init(smem_u32(&s_free[b]), 1);     // PV commit: P_b consumed, O updated
      mbar_init(smem_u32(&p_full[b]), 16);    // 8 softmax warps x 2 CTAs
    }
    mbar_init(smem_u32(&o_final), 1);         // after the last PV (one phase)
    mbar_init(smem_u32(&drain_qk), 1);
    mbar_init(smem_u32(&drain_pv), 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmKR);
    tma_prefetch_desc(&tmV);
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

  if (warp < kSoftmaxWarp0) {
    if (warp == 0 && lane == 0) {
      // ============  Q and K producer (both CTAs)  ============
      const uint32_t lead_q = mapa_shared(smem_u32(&q_full), 0);
      const uint32_t lead_k0 = mapa_shared(smem_u32(&k_full[0]), 0);
      if (rank == 0) mbar_expect_tx(smem_u32(&q_full), 2 * kQBytes);
      const int qrow = r0 + kRows * (int)rank;
      for (int c = 0; c < 3; ++c) tma_load_3d_pair(sQ + c * kChunkQ, &tmQ, 64 * c, h, qrow, lead_q);
      int issued = 0;
      for (int j = 0; j < nblk; ++j) {
        const int s = j % kKStages;
        if (!mbar_wait(smem_u32(&k_empty[s]), ((j / kKStages) & 1) ^ 1, abort_p, 31, j)) break;
        const int key0 = j * kBlk + (kBlk / 2) * (int)rank;
        const uint32_t dk = sK + s * kKBytes;
        const uint32_t fb = lead_k0 + 8 * s;
        if (rank == 0) mbar_expect_tx(smem_u32(&k_full[s]), 2 * kKBytes);
        tma_load_3d_pair(dk, &tmK, 0, h, key0, fb);
        tma_load_3d_pair(dk + kChunkK, &tmK, 64, h, key0, fb);
        tma_load_2d_pair(dk + 2 * kChunkK, &tmKR, kDC, key0, fb);
        ++issued;
      }
      if (*abort_p && rank == 0) {
        // Leaving early: wait (bounded) for the stages already armed, so that
        // no copy lands in this pair's shared memory after it exits.
        mbar_wait_bounded(smem_u32(&q_full), 0, kDrainNs);
        for (int i = max(0, issued - kKStages); i < issued; ++i)
          mbar_wait_bounded(smem_u32(&k_full[i % kKStages]), (i / kKStages) & 1, kDrainNs);
      }
    } else if (warp == 2 && lane == 0) {
      // ===============  V producer (both CTAs)  ===============
      const uint32_t lead_v0 = mapa_shared(smem_u32(&v_full[0]), 0);
      int issued = 0;
      for (int j = 0; j < nblk; ++j) {
        const int s = j % kVStages;
        if (!mbar_wait(smem_u32(&v_empty[s]), ((j / kVStages) & 1) ^ 1, abort_p, 30, j)) break;
        if (rank == 0) mbar_expect_tx(smem_u32(&v_full[s]), 2 * kVBytes);
        tma_load_3d_pair(sV + s * kVBytes, &tmV, 64 * (int)rank, h, j * kBlk, lead_v0 + 8 * s);
        ++issued;
      }
      if (*abort_p && rank == 0)
        for (int i = max(0, issued - kVStages); i < issued; ++i)
          mbar_wait_bounded(smem_u32(&v_full[i % kVStages]), (i / kVStages) & 1, kDrainNs);
    } else if (warp == 1 && lane == 0 && rank == 0) {
      // ==============  QK issuer (leader)  ==============
      // QK(j) into S/P buffer j % 3 once PV(j - 3) has consumed the P there.
      const uint32_t idesc_qk = idesc_bf16_f32(256, kBlk, false, false);
      const uint64_t q_desc = sw128_desc(sQ, 16, 1024);
      const uint64_t k_desc = sw128_desc(sK, 16, 1024);
      bool ok = mbar_wait(smem_u32(&q_full), 0, abort_p, 32, 0);
      for (int j = 0; j < nblk && ok; ++j) {
        const int b = j % kSBufs, s = j % kKStages;
        if (j >= kSBufs &&
            !mbar_wait(smem_u32(&s_free[b]), (j / kSBufs - 1) & 1, abort_p, 36, j)) {
          ok = false;
          break;
        }
        if (!mbar_wait(smem_u32(&k_full[s]), (j / kKStages) & 1, abort_p, 33, j)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sd = tmem + kTmemS + 128 * b;
        const uint64_t b0 = k_desc + (uint64_t)((s * kKBytes) >> 4);
#pragma unroll
        for (int c = 0; c < 3; ++c)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss<2>(sd, q_desc + (uint64_t)((c * kChunkQ + kk * 32) >> 4),
                           b0 + (uint64_t)((c * kChunkK + kk * 32) >> 4), idesc_qk,
                           (c | kk) ? 1u : 0u);
        mma_commit_2_mc(smem_u32(&k_empty[s]), 3);
        mma_commit_2_mc(smem_u32(&s_full[b]), 3);
      }
      if (!ok) {
        mma_commit_2_mc(smem_u32(&drain_qk), 1);
        mbar_wait_bounded(smem_u32(&drain_qk), 0, kDrainNs);
      }
    } else if (warp == 3 && lane == 0 && rank == 0) {
      // ==============  PV issuer (leader)  ==============
      // PV(j) once P(j) is in TMEM (both CTAs) and V(j) has landed; its
      // commit on s_free[j % 3] releases the buffer for QK(j + 3) and tells
      // the softmax that O holds PV(j).
      const uint32_t idesc_pv = idesc_bf16_f32(256, kDV, false, true);
      const uint64_t v_desc = sw128_desc(sV, kVBytes, 1024);
      bool ok = true;
      for (int j = 0; j < nblk; ++j) {
        const int b = j % kSBufs, s = j % kVStages;
        if (!mbar_wait(smem_u32(&p_full[b]), (j / kSBufs) & 1, abort_p, 34, j) ||
            !mbar_wait(smem_u32(&v_full[s]), (j / kVStages) & 1, abort_p, 35, j)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t pa = tmem + kTmemS + 128 * b;
        const uint64_t b0 = v_desc + (uint64_t)((s * kVBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk)
          mma_bf16_ts<2>(tmem + kTmemO, pa + 8 * kk, b0 + (uint64_t)((kk * 2048) >> 4), idesc_pv,
                         (j | kk) ? 1u : 0u);
        mma_commit_2_mc(smem_u32(&v_empty[s]), 3);
        mma_commit_2_mc(smem_u32(&s_free[b]), 3);
        if (j == nblk - 1) mma_commit_2_mc(smem_u32(&o_final), 3);
      }
      if (!ok) {
        mma_commit_2_mc(smem_u32(&drain_pv), 1);
        mbar_wait_bounded(smem_u32(&drain_pv), 0, kDrainNs);
      }
    }
  } else {
    // ===============  softmax + epilogue (both CTAs)  ===============
    const int sw = warp - kSoftmaxWarp0;
    const int quad = sw & 3, ch = sw >> 2;     // TMEM lane quadrant, key half
    const int row = 32 * quad + lane;          // row of this CTA = TMEM lane
    const uint32_t lane_addr = (uint32_t)(32 * quad) << 16;
    const uint32_t lead_p = mapa_shared(smem_u32(&p_full[0]), 0);
    const int qi = r0 + kRows * (int)rank + row;   // query row in the chunk
    const int pos = L0 + qi;                        // its position: sees keys t <= pos
    float m = -INFINITY, l = 0.f;
    bool dead = false;
    for (int j = 0; j < nblk; ++j) {
      const int b = j % kSBufs;
      const bool got = mbar_wait(smem_u32(&s_full[b]), (j / kSBufs) & 1, abort_p, 37, j);
      const uint32_t sa = tmem + lane_addr + kTmemS + 128 * b + 64 * ch;
      const int cmax = pos - (j * kBlk + 64 * ch) + 1;   // columns c < cmax are visible
      uint32_t ra[32], rb[32];
      float mx = -INFINITY;
      // a warp whose 32 rows see all 64 of its columns (every block off the
      // causal diagonal) takes the mask-free path
      const bool full = __all_sync(0xffffffffu, cmax >= 64);
      if (__all_sync(0xffffffffu, got)) {
        tc_fence_after();
        tmem_ld32(sa, ra);
        tmem_ld32(sa + 32, rb);
        tmem_wait_ld();
        // maximum over eight independent chains
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = -INFINITY;
        if (full) {
#pragma unroll
          for (int c = 0; c < 32; c += 8)
#pragma unroll
            for (int i = 0; i < 8; ++i)
              acc[i] = fmaxf(acc[i], fmaxf(__uint_as_float(ra[c + i]), __uint_as_float(rb[c + i])));
        } else {
#pragma unroll
          for (int c = 0; c < 32; c += 8)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              if (c + i < cmax) acc[i] = fmaxf(acc[i], __uint_as_float(ra[c + i]));
              if (c + i + 32 < cmax) acc[i] = fmaxf(acc[i], __uint_as_float(rb[c + i]));
            }
        }
        mx = fmaxf(fmaxf(fmaxf(acc[0], acc[1]), fmaxf(acc[2], acc[3])),
                   fmaxf(fmaxf(acc[4], acc[5]), fmaxf(acc[6], acc[7])));
      }
      red_max[j & 1][ch][row] = mx;
      // both warps of these rows have read S (P overwrites it below) and the
      // other key half's maximum is visible
      tc_fence_before();
      if (named_bar_or(2 + quad, 64, !got || *abort_p)) { dead = true; break; }
      tc_fence_after();
      mx = fmaxf(mx, red_max[j & 1][ch ^ 1][row]);
      const float m_blk = mx * P.scale_log2;
      const bool need = m_blk > m + kRescaleLog2 || (m == -INFINITY && m_blk > -INFINITY);
      const float alpha = !need ? 1.f : (m == -INFINITY ? 0.f : ex2_approx(m - m_blk));
      const float m_use = need ? m_blk : m;
      // p = 2^(s * scale * log2(e) - m): pairs of scores through the packed
      // fp32 FMA, row sums over four independent packed accumulators
      uint32_t pk[32];
      const float2 sc2 = make_float2(P.scale_log2, P.scale_log2);
      const float2 nm2 = make_float2(-m_use, -m_use);
      float2 ls[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) ls[i] = make_float2(0.f, 0.f);
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const uint32_t s0 = e < 16 ? ra[2 * e] : rb[2 * e - 32];
        const uint32_t s1 = e < 16 ? ra[2 * e + 1] : rb[2 * e - 31];
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(s0), __uint_as_float(s1)), sc2, nm2);
        float p0, p1;
        if (MLA_EXP2_POLY_EVERY > 0 &&
            e % (MLA_EXP2_POLY_EVERY > 0 ? MLA_EXP2_POLY_EVERY : 1) == MLA_EXP2_POLY_EVERY - 1) {
          const float2 pp = exp2_poly2(x);
          p0 = pp.x;
          p1 = pp.y;
        } else {
          p0 = ex2_approx(x.x);
          p1 = ex2_approx(x.y);
        }
        if (!full) {
          p0 = 2 * e < cmax ? p0 : 0.f;
          p1 = 2 * e + 1 < cmax ? p1 : 0.f;
        }
        ls[e & 3] = __fadd2_rn(ls[e & 3], make_float2(p0, p1));
        pk[e] = pack_bf16x2(p0, p1);
      }
      const float2 l01 = __fadd2_rn(__fadd2_rn(ls[0], ls[1]), __fadd2_rn(ls[2], ls[3]));
      const float lsum = l01.x + l01.y;
      // O is rescaled only when some row of this warp moved its max, after
      // PV(j - 1), whose commit is phase (j - 1) / 3 of s_free[(j - 1) % 3].
      // Parity wait: S(j) implies PV(j - 3), the barrier's previous phase,
      // is done, and PV(j + 2), its next, needs P(j + 2): one phase at most
      // is outstanding.
      bool ok = true;
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&s_free[(j - 1) % kSBufs]),
                                               ((j - 1) / kSBufs) & 1, abort_p, 38, j));
        if (ok) {
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t o[32];
            const uint32_t oa = tmem + lane_addr + kTmemO + 64 * ch + 32 * cc;
            tmem_ld32(oa, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(oa, o);
          }
        }
      }
      // P(j) over the first 64 columns of S(j): keys [64ch, 64ch + 64) as
      // bf16 pairs in columns [32ch, 32ch + 32).  A warp whose wait gave up
      // hands over nothing; the abort flag it raised stops every softmax
      // thread together at the next barrier.
      if (ok) {
        tmem_st32(tmem + lane_addr + kTmemS + 128 * b + 32 * ch, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(lead_p + 8 * b);
      }
      l = need ? l * alpha + lsum : l + lsum;
      m = m_use;
    }
    if (!dead) {
      // O is final once the last PV is done: o_final completes exactly once.
      const bool got = mbar_wait(smem_u32(&o_final), 0, abort_p, 39, nblk);
      red_l[ch][row] = l;
      if (!named_bar_or(2 + quad, 64, !got || *abort_p)) {
        tc_fence_after();
        const float lt = red_l[0][row] + red_l[1][row];
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        uint32_t ob[32];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_addr + kTmemO + 64 * ch + 32 * cc, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            ob[16 * cc + i] =
                pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
        }
        if (qi < P.T) {
          uint4* dst = reinterpret_cast<uint4*>(P.o + ((long long)qi * P.H + h) * kDV + 64 * ch);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_uint4(ob[4 * i], ob[4 * i + 1], ob[4 * i + 2], ob[4 * i + 3]);
          if (ch == 0)
            P.lse[(long long)qi * P.H + h] =
                lt > 0.f ? (m + log2f(lt)) * 0.69314718055994531f : -INFINITY;
        }
      }
    }
  }

  // =====================  teardown  =====================
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) tmem_dealloc<2>(tmem, kTmemCols);
}

// Host launcher.  q: [T][q_stride] with head h's 192 numbers at h * 192;
// ctx: [L][576]; k_nope, v: [L][H][128]; all bf16, 16-byte aligned.
inline mla_status launch_prefill_attn_impl(
    bool (*make_tmap)(CUtensorMap*, const void*, int, const uint64_t*, const uint64_t*,
                      const uint32_t*),
    const void* q, int q_stride, const void* ctx, const void* k_nope, const void* v, int T,
    int L, int H, float scale, __nv_bfloat16* o, float* lse, cudaStream_t st) {
  using namespace pfa;
  CUtensorMap tQ, tK, tKR, tV;
  {
    const uint64_t dims[3] = {(uint64_t)kDQK, (uint64_t)H, (uint64_t)T};
    const uint64_t strides[2] = {(uint64_t)kDQK * 2, (uint64_t)q_stride * 2};
    const uint32_t box[3] = {64, 1, (uint32_t)kRows};
    if (!make_tmap(&tQ, q, 3, dims, strides, box)) return MLA_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {(uint64_t)kDN, (uint64_t)H, (uint64_t)L};
    const uint64_t strides[2] = {(uint64_t)kDN * 2, (uint64_t)H * kDN * 2};
    const uint32_t box[3] = {64, 1, (uint32_t)(kBlk / 2)};
    if (!make_tmap(&tK, k_nope, 3, dims, strides, box)) return MLA_ERR_CUDA;
  }
  {
    const uint64_t dims[2] = {(uint64_t)kD, (uint64_t)L};
    const uint64_t strides[1] = {(uint64_t)kD * 2};
    const uint32_t box[2] = {64, (uint32_t)(kBlk / 2)};
    if (!make_tmap(&tKR, ctx, 2, dims, strides, box)) return MLA_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {(uint64_t)kDV, (uint64_t)H, (uint64_t)L};
    const uint64_t strides[2] = {(uint64_t)kDV * 2, (uint64_t)H * kDV * 2};
    const uint32_t box[3] = {64, 1, (uint32_t)kBlk};
    if (!make_tmap(&tV, v, 3, dims, strides, box)) return MLA_ERR_CUDA;
  }
  PrefillParams p;
  p.o = o;
  p.lse = lse;
  p.T = T;
  p.L = L;
  p.H = H;
  p.scale_log2 = scale * 1.4426950408889634f;
  if (cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBytes) != cudaSuccess)
    return MLA_ERR_CUDA;
  const int n_pt = (T + 2 * kRows - 1) / (2 * kRows);
  dim3 grid(2 * n_pt, H);
  prefill_attn_kernel<<<grid, kThreads, kSmemBytes, st>>>(tQ, tK, tKR, tV, p);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
