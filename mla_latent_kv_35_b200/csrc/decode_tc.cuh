// decode_tc.cuh -- split-KV flash-decode on the paged latent cache with the
// 5th-generation tensor cores (tcgen05 pair MMAs, TMEM accumulators, TMA).
//
// What it computes (deepforge "DeepSeek-V2", §1 "Store a latent, rebuild the
// keys and values" and "The bottleneck at inference time"): with W_UK folded
// into the query, every head's score against cached token t is
// q_abs . [c_t ; k_rope_t] over the 576 cached numbers, and the latent output
// is sum_t softmax(s)_t c_t.  The cache row is read once and serves both as
// the key (all 576 columns) and as the value (the first 512).
//
// Work decomposition
//   * A cluster of two CTAs (one per SM of a TPC) owns 128 query rows
//     (S_q*H rows of one sequence, 128 at a time) and a contiguous run of
//     128-token blocks.  CTA r holds rows [64r, 64r+64): its Q slice (72 KB)
//     stays in shared memory for the whole piece.
//   * QK: one pair MMA (cta_group::2, M = 128 rows, N = 128 tokens, K = 576).
//     CTA r supplies the B half of page r of the block.  Each SM gets its 64
//     rows x 128 tokens in TMEM folded onto 128 lanes x 64 columns: lane l<64
//     holds row l, tokens 0..63; lane l>=64 holds row l-64, tokens 64..127.
//   * PV: two pair MMAs per 16-token step (N = 256 latent columns each,
//     M = 128 rows, K = 128 tokens per block).  CTA r supplies latent columns
//     [256n + 128r, +128) of all 128 tokens (MN-major B read straight from
//     the cache tile) and its own 64 rows of P (bf16, K-major).  O therefore
//     takes 256 TMEM columns per SM; S is double buffered in 2 x 64 more.
//   * Each 128-thread softmax warpgroup reads its SM's S, exchanges row
//     maxima between the two lanes that share a row, keeps a lazily rescaled
//     running max (O is only rescaled in TMEM when the max grows by more than
//     2^8), writes P to shared memory and signals the MMA warp of the leader.
//   * Pieces (sequence, block range) of a worker write normalised partial
//     outputs and natural-log LSE into slot worker + v of the workspace; the
//     combine kernel merges them.
//
// Partial pages: a page with `valid` < 64 tokens is loaded through a 3-D
// tensor map [pages][64 slots][576] starting at slot valid-64, so the rows
// before the page are out of bounds and arrive as zeros; pages past the end
// are loaded entirely out of bounds.  Unused cache slots are never read.
//
// Every mbarrier wait is bounded (MLA_WAIT_NS); on expiry the kernel raises
// MLA_ERR_TIMEOUT in the device status, every role leaves its loop, the pair
// meets at a final cluster barrier and frees its TMEM.
#pragma once

#include "common.cuh"
#include "simt.cuh"

namespace mla {

constexpr bool kDecodeTcReady = true;

namespace dtc {
constexpr int kDC = 512;           // latent width
constexpr int kD = 576;            // cached numbers per token
constexpr int kPage = 64;          // tokens per page
constexpr int kBlk = 128;          // tokens per block (two pages)
constexpr int kStages = 7;         // ring stages of 16 KB
constexpr int kStageBytes = 16384;
constexpr int kQBytes = 9 * 8192;  // 64 rows x 576 cols bf16
constexpr int kPBytes = 16384;     // 64 rows x 128 tokens bf16
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffP = kOffQ + kQBytes;
constexpr uint32_t kOffRing = kOffP + 2 * kPBytes;
constexpr uint32_t kSmemBytes = kOffRing + kStages * kStageBytes + 1024;  // + alignment
constexpr int kThreads = 256;
constexpr int kSoftmaxWarp0 = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;     // O_n at columns [128n, 128n + 128)
constexpr uint32_t kTmemS = 256;   // S_b at columns [256 + 64b, +64)
constexpr float kRescaleLog2 = 8.0f;
}  // namespace dtc

struct DecodeTcParams {
  const int32_t* page_table;
  const int32_t* seq_lens;
  const int32_t* start;   // [V + 1] block prefix sums from plan_kernel
  float* ws_lse;          // [slots][128]
  float* ws_o;            // [slots][128][512]
  int n_pages, max_pages, B, S_q, H, R, G;
  float scale_log2;       // softmax scale * log2(e)
};

__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx_cluster(uint32_t bar_cluster, uint32_t bytes) {
  asm volatile(
      "mbarrier.arrive.expect_tx.release.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(
          bar_cluster),
      "r"(bytes)
      : "memory");
}

// Piece iteration shared by all roles: worker k's blocks [lo, hi) split by
// virtual sequence.
struct PieceIter {
  const int32_t* start;
  int V, lo, hi, v;
  __device__ void init(const int32_t* s, int V_, int lo_, int hi_) {
    start = s; V = V_; lo = lo_; hi = hi_;
    v = (lo < hi) ? seq_of_block(start, V, lo) : V;
  }
  // next piece with at least one block; returns false when done
  __device__ bool next(int& pv, int& x0, int& x1) {
    while (v < V && start[v] < hi) {
      const int a = max(lo, start[v]) - start[v];
      const int b = min(hi, start[v + 1]) - start[v];
      const int cur = v++;
      if (b > a) { pv = cur; x0 = a; x1 = b; return true; }
    }
    return false;
  }
};

// Page of token block x, half p (0/1) of sequence b: returns the pool page
// (or -1 when the page lies past the context) and the slot shift for a
// partial page (rows before it load as zeros).
__device__ __forceinline__ void page_of(const DecodeTcParams& P, int b, int L, int x, int p,
                                        int& page, int& slot0) {
  const int first = x * dtc::kBlk + p * dtc::kPage;
  const int valid = min(L - first, dtc::kPage);
  if (valid <= 0) {
    page = 0;
    slot0 = dtc::kPage;  // entirely out of bounds -> zeros
    return;
  }
  int pg = P.page_table[(long long)b * P.max_pages + first / dtc::kPage];
  if (pg < 0 || pg >= P.n_pages) {
    raise_flag(kFlagBounds);
    page = 0;
    slot0 = dtc::kPage;
    return;
  }
  page = pg;
  slot0 = valid - dtc::kPage;  // 0 for a full page, negative for a partial one
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(dtc::kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmKV, const DecodeTcParams P) {
  using namespace dtc;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ __align__(8) uint64_t q_full, q_empty, o_empty;
  __shared__ __align__(8) uint64_t s_full[2], p_full[2], pv_done[2];
  __shared__ float red_max[2][2][64];
  __shared__ float red_sum[2][64];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int worker = blockIdx.x >> 1;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base + kOffQ, sP = base + kOffP, sRing = base + kOffRing;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 2);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    mbar_init(smem_u32(&q_full), 2);
    mbar_init(smem_u32(&q_empty), 1);
    mbar_init(smem_u32(&o_empty), 8);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&s_full[b]), 1);
      mbar_init(smem_u32(&p_full[b]), 8);
      mbar_init(smem_u32(&pv_done[b]), 1);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmKV);
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

  if (warp == 0 && lane == 0) {
    // =====================  TMA producer (both CTAs)  =====================
    const uint32_t leader_full0 = mapa_shared(smem_u32(&full_bar[0]), 0);
    const uint32_t leader_qfull = mapa_shared(smem_u32(&q_full), 0);
    uint32_t it = 0;  // ring position
    PieceIter pi;
    pi.init(P.start, V, lo, hi);
    int v, x0, x1, piece = 0;
    bool ok = true;
    // schedule: per block j: QK(j) stages; PV(j-1) stages after QK(j)
    int pv_pend_b = -1, pv_pend_L = 0, pv_pend_x = 0;  // pending PV block
    auto load_stage = [&](int page, int slot0, int cc0, int nchunks) -> bool {
      const int s = it % kStages;
      if (!mbar_wait(smem_u32(&empty_bar[s]), ((it / kStages) & 1) ^ 1, abort_p, 1, it)) return false;
      const uint32_t fb = leader_full0 + s * 8;
      mbar_expect_tx_cluster(fb, nchunks * 8192);
      const uint32_t dst = sRing + s * kStageBytes;
      for (int c = 0; c < nchunks; ++c)
        tma_load_3d_pair(dst + c * 8192, &tmKV, (cc0 + c) * 64, slot0, page, fb);
      ++it;
      return true;
    };
    auto load_pv = [&](int b, int L, int x) -> bool {
      for (int n = 0; n < 2; ++n)
        for (int p = 0; p < 2; ++p) {
          int page, slot0;
          page_of(P, b, L, x, p, page, slot0);
          if (!load_stage(page, slot0, 4 * n + 2 * (int)rank, 2)) return false;
        }
      return true;
    };
    while (ok && pi.next(v, x0, x1)) {
      const int b = v / P.R, rb = v % P.R;
      const int L = P.seq_lens[b];
      // Q slice of this piece (needs the previous piece's QK MMAs finished)
      if (piece > 0 && !mbar_wait(smem_u32(&q_empty), (piece - 1) & 1, abort_p, 2, piece)) { ok = false; break; }
      mbar_expect_tx_cluster(leader_qfull, kQBytes);
      const int row0 = b * rows_seq + rb * 128 + 64 * (int)rank;
      for (int c = 0; c < 9; ++c) tma_load_2d_pair(sQ + c * 8192, &tmQ, c * 64, row0, leader_qfull);
      for (int x = x0; x < x1 && ok; ++x) {
        int page, slot0;
        page_of(P, b, L, x, (int)rank, page, slot0);
        for (int c = 0; c < 4 && ok; ++c) ok = load_stage(page, slot0, 2 * c, 2);
        if (ok) ok = load_stage(page, slot0, 8, 1);
        if (ok && pv_pend_b >= 0) ok = load_pv(pv_pend_b, pv_pend_L, pv_pend_x);
        pv_pend_b = b; pv_pend_L = L; pv_pend_x = x;
      }
      ++piece;
    }
    if (ok && pv_pend_b >= 0) ok = load_pv(pv_pend_b, pv_pend_L, pv_pend_x);
    if (!ok) {
      // give copies already issued time to land before the CTA can exit
      const uint64_t t0 = globaltimer();
      while (globaltimer() - t0 < 50000ull) {
      }
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // =====================  MMA issuer (leader CTA)  =====================
    const uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
    const uint32_t idesc_pv = idesc_bf16_f32(128, 256, false, true);
    uint32_t it = 0;
    int j = 0;  // global block counter of this worker
    PieceIter pi;
    pi.init(P.start, V, lo, hi);
    int v, x0, x1, piece = 0;
    bool ok = true;
    int pend = -1;            // global index of the block whose PV is pending
    bool pend_first = false;  // that block is the first of its piece
    int pend_piece = 0;
    auto consume = [&](int& s) -> bool {
      s = it % kStages;
      if (!mbar_wait(smem_u32(&full_bar[s]), (it / kStages) & 1, abort_p, 3, it)) return false;
      tc_fence_after();
      ++it;
      return true;
    };
    auto issue_pv = [&](int jb, bool first, int pc) -> bool {
      if (!mbar_wait(smem_u32(&p_full[jb & 1]), (jb >> 1) & 1, abort_p, 4, jb)) return false;
      if (first && pc > 0 && !mbar_wait(smem_u32(&o_empty), (pc - 1) & 1, abort_p, 5, pc)) return false;
      tc_fence_after();
      const uint32_t pbuf = sP + (jb & 1) * kPBytes;
      for (int n = 0; n < 2; ++n)
        for (int p = 0; p < 2; ++p) {
          int s;
          if (!consume(s)) return false;
          const uint32_t st = sRing + s * kStageBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = sw128_desc(pbuf + p * 8192 + kk * 32, 16, 1024);
            const uint64_t bd = sw128_desc(st + kk * 2048, 8192, 1024);
            const uint32_t acc = (first && p == 0 && kk == 0) ? 0u : 1u;
            mma_bf16_ss<2>(tmem + kTmemO + 128 * n, ad, bd, idesc_pv, acc);
          }
          mma_commit_2_mc(smem_u32(&empty_bar[s]), 3);
        }
      mma_commit_2_mc(smem_u32(&pv_done[jb & 1]), 3);
      return true;
    };
    while (ok && pi.next(v, x0, x1)) {
      if (!mbar_wait(smem_u32(&q_full), piece & 1, abort_p, 6, piece)) { ok = false; break; }
      tc_fence_after();
      for (int x = x0; x < x1 && ok; ++x, ++j) {
        // QK(j) into S[j & 1]
        const uint32_t sd = tmem + kTmemS + 64 * (j & 1);
        for (int c = 0; c < 5 && ok; ++c) {
          int s;
          if (!consume(s)) { ok = false; break; }
          const uint32_t st = sRing + s * kStageBytes;
          const int nk = (c < 4) ? 8 : 4;
          for (int kk = 0; kk < nk; ++kk) {
            const int col = c * 2 + kk / 4;  // 64-column chunk of the 576
            const uint64_t ad = sw128_desc(sQ + col * 8192 + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = sw128_desc(st + (kk / 4) * 8192 + (kk & 3) * 32, 16, 1024);
            mma_bf16_ss<2>(sd, ad, bd, idesc_qk, (c | kk) ? 1u : 0u);
          }
          mma_commit_2_mc(smem_u32(&empty_bar[s]), 3);
        }
        if (!ok) break;
        mma_commit_2_mc(smem_u32(&s_full[j & 1]), 3);
        if (x == x1 - 1) mma_commit_2_mc(smem_u32(&q_empty), 3);
        if (pend >= 0 && !issue_pv(pend, pend_first, pend_piece)) { ok = false; break; }
        pend = j; pend_first = (x == x0); pend_piece = piece;
      }
      ++piece;
    }
    if (ok && pend >= 0) issue_pv(pend, pend_first, pend_piece);
  } else if (warp >= kSoftmaxWarp0) {
    // =====================  softmax + epilogue (both CTAs)  =====================
    const int tid = threadIdx.x - kSoftmaxWarp0 * 32;  // = TMEM lane
    const int h = tid & 63, half = tid >> 6;
    const uint32_t lane_addr = (uint32_t)(32 * (warp - kSoftmaxWarp0)) << 16;
    const uint32_t leader_pfull0 = mapa_shared(smem_u32(&p_full[0]), 0);
    const uint32_t leader_oempty = mapa_shared(smem_u32(&o_empty), 0);
    PieceIter pi;
    pi.init(P.start, V, lo, hi);
    int v, x0, x1;
    int j = 0;
    bool dead = false;
    while (!dead && pi.next(v, x0, x1)) {
      const int b = v / P.R, rb = v % P.R;
      const int L = P.seq_lens[b];
      const int grow = rb * 128 + 64 * (int)rank + h;      // row within the sequence
      const int limit = L - P.S_q + grow / P.H + 1;         // visible tokens t < limit
      float m = -INFINITY, l = 0.f;
      bool o_started = false;
      for (int x = x0; x < x1; ++x, ++j) {
        bool fail = !mbar_wait(smem_u32(&s_full[j & 1]), (j >> 1) & 1, abort_p, 7, j);
        if (named_bar_or(1, 128, fail || *abort_p)) { dead = true; break; }
        tc_fence_after();
        uint32_t s_raw[64];
        {
          uint32_t (&a)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s_raw[0]);
          uint32_t (&c)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s_raw[32]);
          const uint32_t sa = tmem + lane_addr + kTmemS + 64 * (j & 1);
          tmem_ld32(sa, a);
          tmem_ld32(sa + 32, c);
          tmem_wait_ld();
        }
        // token t of this lane's page: first + c - shift, valid if c >= shift
        const int first = x * kBlk + half * kPage;
        const int valid = min(L - first, kPage);
        const int shift = valid > 0 ? kPage - valid : kPage;
        const int cmax = limit - first + shift;  // columns c < cmax are visible
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= shift && c < cmax) mx = fmaxf(mx, __uint_as_float(s_raw[c]));
        red_max[j & 1][half][h] = mx;
        named_bar_sync(1, 128);
        mx = fmaxf(mx, red_max[j & 1][half ^ 1][h]);
        const float m_blk = mx * P.scale_log2;
        // Lazy rescale: a row moves its running max only when the block max
        // exceeds it by more than 2^kRescaleLog2.  The decision is per row,
        // but TMEM loads/stores are warp-collective, so a warp rescales when
        // any of its rows needs it, with alpha = 1 for the other rows.
        const bool need = m_blk > m + kRescaleLog2 || (m == -INFINITY && m_blk > -INFINITY);
        const float alpha = !need ? 1.f : (m == -INFINITY ? 0.f : exp2f(m - m_blk));
        if (o_started && __any_sync(0xffffffffu, need)) {
          // O holds PV up to block j-1: wait for it, then rescale in TMEM
          const bool ok = mbar_wait(smem_u32(&pv_done[(j - 1) & 1]), ((j - 1) >> 1) & 1,
                                    abort_p, 8, j);
          if (__all_sync(0xffffffffu, ok)) {
            tc_fence_after();
            for (int n = 0; n < 2; ++n)
              for (int cc = 0; cc < 4; ++cc) {
                uint32_t r[32];
                const uint32_t oa = tmem + lane_addr + kTmemO + 128 * n + 32 * cc;
                tmem_ld32(oa, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                tmem_st32(oa, r);
              }
            tmem_wait_st();
          }
        }
        if (need) {
          l *= alpha;
          m = m_blk;
        }
        // P buffer (j & 1) was last read by PV(j - 2)
        if (j >= 2) mbar_wait(smem_u32(&pv_done[j & 1]), ((j - 2) >> 1) & 1, abort_p, 9, j);
        float lsum = 0.f;
        const uint32_t prow = sP + (j & 1) * kPBytes + half * 8192 + h * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c0 = u * 8 + e * 2;
            float p0 = (c0 >= shift && c0 < cmax)
                           ? exp2f(fmaf(__uint_as_float(s_raw[c0]), P.scale_log2, -m)) : 0.f;
            float p1 = (c0 + 1 >= shift && c0 + 1 < cmax)
                           ? exp2f(fmaf(__uint_as_float(s_raw[c0 + 1]), P.scale_log2, -m)) : 0.f;
            lsum += p0 + p1;
            pk[e] = pack_bf16x2(p0, p1);
          }
          const uint32_t addr = prow + ((u ^ (h & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[0]),
                       "r"(pk[1]), "r"(pk[2]), "r"(pk[3])
                       : "memory");
        }
        l += lsum;
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(leader_pfull0 + (j & 1) * 8);
        o_started = true;
      }
      if (dead) break;
      // ---------------- epilogue of the piece ----------------
      const int jl = j - 1;
      bool fail = !mbar_wait(smem_u32(&pv_done[jl & 1]), (jl >> 1) & 1, abort_p, 10, jl);
      if (named_bar_or(1, 128, fail || *abort_p)) { dead = true; break; }
      tc_fence_after();
      red_sum[half][h] = l;
      named_bar_sync(1, 128);
      const float lt = l + red_sum[half ^ 1][h];
      named_bar_sync(1, 128);  // red_sum reused by the next piece
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const long long slot = (long long)worker + v;
      const long long row = slot * 128 + 64 * (int)rank + h;
      float* dst = P.ws_o + row * kDC;
      for (int n = 0; n < 2; ++n)
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_addr + kTmemO + 128 * n + 32 * cc, r);
          tmem_wait_ld();
          float4* d4 = reinterpret_cast<float4*>(dst + 256 * n + 128 * half + 32 * cc);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            d4[i] = make_float4(__uint_as_float(r[4 * i]) * inv, __uint_as_float(r[4 * i + 1]) * inv,
                                __uint_as_float(r[4 * i + 2]) * inv,
                                __uint_as_float(r[4 * i + 3]) * inv);
        }
      if (half == 0)
        P.ws_lse[row] = lt > 0.f ? (m + log2f(lt)) * 0.69314718055994531f : -INFINITY;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_oempty);
    }
  }

  // =====================  teardown  =====================
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) tmem_dealloc<2>(tmem, kTmemCols);
}

// Host launcher: TMA descriptors for the query rows and the page pool.
inline mla_status launch_decode_tc_impl(
    bool (*make_tmap)(CUtensorMap*, const void*, int, const uint64_t*, const uint64_t*,
                      const uint32_t*),
    const void* qbuf, const void* pool, int n_pages, const int32_t* page_table, int max_pages,
    const int32_t* seq_lens, int B, int S_q, int H, float scale, int G, const int32_t* start,
    float* ws_lse, float* ws_o, cudaStream_t st) {
  using namespace dtc;
  CUtensorMap tQ, tKV;
  {
    const uint64_t dims[2] = {(uint64_t)kD, (uint64_t)B * S_q * H};
    const uint64_t strides[1] = {(uint64_t)kD * 2};
    const uint32_t box[2] = {64, 64};
    if (!make_tmap(&tQ, qbuf, 2, dims, strides, box)) return MLA_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {(uint64_t)kD, (uint64_t)kPage, (uint64_t)n_pages};
    const uint64_t strides[2] = {(uint64_t)kD * 2, (uint64_t)kD * 2 * kPage};
    const uint32_t box[3] = {64, 64, 1};
    if (!make_tmap(&tKV, pool, 3, dims, strides, box)) return MLA_ERR_CUDA;
  }
  DecodeTcParams p;
  p.page_table = page_table;
  p.seq_lens = seq_lens;
  p.start = start;
  p.ws_lse = ws_lse;
  p.ws_o = ws_o;
  p.n_pages = n_pages;
  p.max_pages = max_pages;
  p.B = B;
  p.S_q = S_q;
  p.H = H;
  p.R = (S_q * H) / 128;
  p.G = G;
  p.scale_log2 = scale * 1.4426950408889634f;
  if (cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBytes) != cudaSuccess)
    return MLA_ERR_CUDA;
  decode_tc_kernel<<<2 * G, kThreads, kSmemBytes, st>>>(tQ, tKV, p);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
