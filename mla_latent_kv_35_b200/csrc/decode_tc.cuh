// decode_tc.cuh -- split-KV flash-decode on the paged latent cache with the
// 5th-generation tensor cores (tcgen05 pair MMAs, TMEM accumulators, TMA).
//
// What it computes (deepforge "DeepSeek-V2", §1 "Store a latent, rebuild the
// keys and values" and "The bottleneck at inference time"): with W_UK folded
// into the query, every head's score against cached token t is
// q_abs . [c_t ; k_rope_t] over the 576 cached numbers, and the latent output
// is sum_t softmax(s)_t c_t.  The cache row serves both as the key (all 576
// columns) and as the value (the first 512).
//
// Work decomposition
//   * A cluster of two CTAs (one per SM of a TPC) owns 128 query rows
//     (S_q*H rows of one sequence, 128 at a time) and a contiguous run of
//     128-token blocks.  CTA r holds rows [64r, 64r+64): its Q slice (72 KB,
//     one TMA load per piece) stays in shared memory for the whole piece.
//   * QK: pair MMAs (cta_group::2, M = 128 rows, N = 128 tokens, K = 576).
//     CTA r supplies the B half of page r of the block.  Each SM gets its 64
//     rows x 128 tokens in TMEM folded onto 128 lanes x 64 columns: lane l<64
//     holds row l, tokens 0..63; lane l>=64 holds row l-64, tokens 64..127.
//   * PV: two pair MMAs per 16-token step (N = 256 latent columns each,
//     M = 128 rows, K = 128 tokens per block).  CTA r supplies latent columns
//     [256n + 128r, +128) of all 128 tokens (MN-major B read straight from
//     the cache tile) and its own 64 rows of P (bf16, K-major).  O therefore
//     takes 256 TMEM columns per SM; S is double buffered in 2 x 64 more.
//   * Loads.  Warp 0 lane 0 of each CTA streams its own page of the block
//     for QK through a 3-stage ring.  Each stage is one 24 KB TMA box (64
//     columns x 64 slots x 3 chunks) of a 4-D view of the pool: (64 columns,
//     64 slots, 9 chunks, pages), strides (1152 B, 128 B, 73728 B).  Only the
//     leader arms the stage barrier, for the bytes of both CTAs; the peer's
//     box completes on the leader's barrier.
//   * PV tiles come through a second ring of two 32 KB stages, one page's
//     latent half each.  Warps 2 and 3 fill them with 16-byte cp.async into
//     the 128-byte-swizzled layout, so this traffic bypasses the bulk-copy
//     engine the QK boxes keep busy.  In the peer CTA, warp 1 lane 0 relays
//     each landed stage to the leader's barrier.
//   * Each 128-thread softmax warpgroup reads its SM's S and exchanges row
//     maxima between the two lanes that share a row.  It keeps a lazily
//     rescaled running max: O is rescaled in TMEM only when the max grows by
//     more than 2^8, and warp-uniformly, since tcgen05.ld/st are collective.
//     It then writes P to shared memory and signals the leader's MMA warp.
//   * Pieces (sequence, block range) of a worker write normalised partial
//     outputs and natural-log LSE into slot worker + v of the workspace; the
//     combine kernel merges them.
//
// Shared memory: Q 72 KB + P 16 KB + QK ring 72 KB + PV ring 64 KB.  Each
// ring holds one block.  The QK MMA shape the pair split gives, 64 x 128 x 16
// per SM, costs about as much per instruction as a full-size one.  So the
// MMA sequence and the one block of ring depth bound this kernel, not HBM.
//
// Partial pages: a page with `valid` < 64 tokens starts its boxes at slot
// valid - 64.  The rows before the page are out of bounds and arrive as
// zeros, and the cp.async loader shifts its rows the same way.  Pages past
// the end load entirely out of bounds (slot 64).  Unused cache slots are
// never read.
//
// Every mbarrier wait is bounded (MLA_WAIT_NS); on expiry the kernel raises
// MLA_ERR_TIMEOUT in the device status and every role leaves its loop.  On
// the way out the leader's producer waits (bounded) for the boxes it armed
// and its MMA thread for a last commit, the loader warps for their own
// cp.async; then the pair meets at a final cluster barrier and frees its
// TMEM.
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
constexpr int kChunk = 8192;       // 64 tokens x 64 columns bf16, one swizzled operand tile
constexpr int kQkChunks = 3;       // chunks per QK stage (one TMA box)
constexpr int kQkStages = 3;       // QK ring: 3 stages x 3 chunks = this CTA's page of one block
constexpr int kQkStageBytes = kQkChunks * kChunk;
constexpr int kPvStages = 2;       // PV ring: one page's latent half (4 chunks) per stage
constexpr int kPvStageBytes = 4 * kChunk;
constexpr int kQBytes = 9 * kChunk;  // 64 rows x 576 cols bf16
constexpr int kPBytes = 2 * kChunk;  // 64 rows x 128 tokens bf16
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffP = kOffQ + kQBytes;
constexpr uint32_t kOffQk = kOffP + kPBytes;
constexpr uint32_t kOffPv = kOffQk + kQkStages * kQkStageBytes;
constexpr uint32_t kSmemBytes = kOffPv + kPvStages * kPvStageBytes + 1024;  // + alignment
constexpr int kThreads = 256;
constexpr int kSoftmaxWarp0 = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;     // O_n at columns [128n, 128n + 128)
constexpr uint32_t kTmemS = 256;   // S_b at columns [256 + 64b, +64)
constexpr float kRescaleLog2 = 8.0f;
}  // namespace dtc

struct DecodeTcParams {
  const uint8_t* pool;    // [n_pages][64][576] bf16
  const int32_t* page_table;
  const int32_t* seq_lens;
  const int32_t* tail;    // [B] tokens past this cache's range, or nullptr
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

// Page of token block x, half p (0/1) of sequence b: the pool page and the
// first slot to load.  A partial page starts at a negative slot (the rows
// before the page load as zeros); a page past the context, or a page id
// outside the pool (raising MLA_ERR_BOUNDS), loads entirely out of bounds.
__device__ __forceinline__ void page_of(const DecodeTcParams& P, int b, int L, int x, int p,
                                        int& page, int& slot0) {
  const int first = x * dtc::kBlk + p * dtc::kPage;
  const int valid = min(L - first, dtc::kPage);
  if (valid <= 0) {
    page = 0;
    slot0 = dtc::kPage;
    return;
  }
  const int pg = P.page_table[(long long)b * P.max_pages + first / dtc::kPage];
  if (pg < 0 || pg >= P.n_pages) {
    raise_flag(kFlagBounds);
    page = 0;
    slot0 = dtc::kPage;
    return;
  }
  page = pg;
  slot0 = valid - dtc::kPage;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(dtc::kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmQK,
                     const DecodeTcParams P) {
  using namespace dtc;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t qk_full[kQkStages], qk_empty[kQkStages];
  __shared__ __align__(8) uint64_t pv_full[kPvStages], pv_empty[kPvStages];
  __shared__ __align__(8) uint64_t q_full, q_empty, o_empty, p_full, pv_done, mma_drain;
  __shared__ __align__(8) uint64_t s_full[2];
  __shared__ float red_max[2][2][64];
  __shared__ float red_sum[2][64];
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
    for (int s = 0; s < kQkStages; ++s) {
      // full barriers: the leader's producer arrives once with the bytes of
      // both CTAs; the peer's copies only complete transactions on it
      mbar_init(smem_u32(&qk_full[s]), 1);
      mbar_init(smem_u32(&qk_empty[s]), 1);  // MMA commit (multicast)
    }
    for (int s = 0; s < kPvStages; ++s) {
      // 32 cp.async lanes of one loader warp (+ the peer's relay on the leader)
      mbar_init(smem_u32(&pv_full[s]), rank == 0 ? 33u : 32u);
      mbar_init(smem_u32(&pv_empty[s]), 1);
    }
    mbar_init(smem_u32(&q_full), 1);
    mbar_init(smem_u32(&q_empty), 1);
    mbar_init(smem_u32(&o_empty), 8);        // 4 softmax warps x 2 CTAs
    mbar_init(smem_u32(&p_full), 8);
    mbar_init(smem_u32(&pv_done), 1);
    mbar_init(smem_u32(&mma_drain), 1);
    mbar_init(smem_u32(&s_full[0]), 1);
    mbar_init(smem_u32(&s_full[1]), 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmQK);
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
    // =================  QK producer: Q slices and QK chunks  =================
    const uint32_t lead_full0 = mapa_shared(smem_u32(&qk_full[0]), 0);
    const uint32_t lead_qfull = mapa_shared(smem_u32(&q_full), 0);
    uint32_t it = 0;
    PieceIter pi;
    pi.init(P.start, V, lo, hi);
    int v, x0, x1, piece = 0;
    uint32_t q_issued = 0;
    bool ok = true;
    while (ok && pi.next(v, x0, x1)) {
      const int b = v / P.R, rb = v % P.R;
      const int L = P.seq_lens[b];
      // the Q slice is free once the previous piece's QK MMAs completed
      if (piece > 0 && !mbar_wait(smem_u32(&q_empty), (piece - 1) & 1, abort_p, 2, piece)) {
        ok = false;
        break;
      }
      if (rank == 0) mbar_expect_tx(smem_u32(&q_full), 2 * kQBytes);
      const int row0 = b * rows_seq + rb * 128 + 64 * (int)rank;
      for (int c = 0; c < 9; ++c)
        tma_load_2d_pair(sQ + c * kChunk, &tmQ, c * 64, row0, lead_qfull);
      ++q_issued;
      for (int x = x0; x < x1 && ok; ++x) {
        int page, slot0;
        page_of(P, b, L, x, (int)rank, page, slot0);
        // one box = chunks [3k, 3k+3) of the page (64 slots x 64 columns each)
        for (int k = 0; k < 9 / kQkChunks; ++k, ++it) {
          const int s = it % kQkStages;
          if (!mbar_wait(smem_u32(&qk_empty[s]), ((it / kQkStages) & 1) ^ 1, abort_p, 1, it)) {
            ok = false;
            break;
          }
          const uint32_t fb = lead_full0 + s * 8;
          if (rank == 0) mbar_expect_tx(smem_u32(&qk_full[s]), 2 * kQkStageBytes);
          tma_load_4d_pair(sQk + s * kQkStageBytes, &tmQK, 0, slot0, kQkChunks * k, page, fb);
        }
      }
      ++piece;
    }
    if (!ok && rank == 0) {
      // Leaving early: wait (bounded) until the boxes already issued have
      // landed, so that no copy writes into this pair's shared memory after
      // it exits.  Only the leader's barriers count bytes; they count both
      // CTAs' boxes of a stage, and the peer waits for the leader at the
      // final cluster barrier.  A stage the peer never issued cannot
      // complete, so each wait is bounded on its own.
      for (uint32_t i = it > (uint32_t)kQkStages ? it - kQkStages : 0u; i < it; ++i)
        mbar_wait_bounded(smem_u32(&qk_full[i % kQkStages]), (i / kQkStages) & 1, kDrainNs);
      if (q_issued > 0) mbar_wait_bounded(smem_u32(&q_full), (q_issued - 1) & 1, kDrainNs);
    }
  } else if (warp == 2 || warp == 3) {
    // ======  PV loader warps (cp.async): this CTA's latent half of page p  ======
    // Warp 2 fills the stages of page 0, warp 3 those of page 1.  The copies
    // go through the load/store path rather than the bulk-copy engine, which
    // is busy with the QK boxes.  Each stage lands as [n][chunk][slot][64
    // columns] for latent chunks 4n + 2r + {0, 1}; rows past the sequence
    // are written as zeros.
    const int mine = warp - 2;
    uint32_t it = 0;
    PieceIter pi;
    pi.init(P.start, V, lo, hi);
    int v, x0, x1;
    bool ok = true;
    while (ok && pi.next(v, x0, x1)) {
      const int b = v / P.R;
      const int L = P.seq_lens[b];
      for (int x = x0; x < x1 && ok; ++x)
        for (int p = 0; p < 2; ++p, ++it) {
          if (p != mine) continue;
          // same row placement as the QK boxes: shared-memory row i holds
          // slot i + slot0 (slot0 <= 0; a partial page sits at the bottom),
          // and slot0 == kPage marks a page past the context (all zeros)
          int page, slot0;
          page_of(P, b, L, x, p, page, slot0);
          const int s = it % kPvStages;
          const bool got = mbar_wait(smem_u32(&pv_empty[s]), ((it / kPvStages) & 1) ^ 1,
                                     abort_p, 11, it);
          if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
          const uint8_t* src = P.pool + (size_t)page * (kPage * kD * 2);
          const uint32_t dst = sPv + s * kPvStageBytes;
#pragma unroll 8
          for (int i = 0; i < 64; ++i) {
            // one 512-byte row per warp step: 4 chunks x 8 units of 16 B
            const int row = i, q4 = lane >> 3, u = lane & 7;
            const int chunk = 4 * (q4 >> 1) + 2 * (int)rank + (q4 & 1);
            const int srow = row + slot0;
            const uint32_t d = dst + q4 * kChunk + row * 128 + ((u ^ (row & 7)) << 4);
            if (slot0 < kPage && srow >= 0)
              cp_async16(d, src + srow * (kD * 2) + chunk * 128 + u * 16);
            else
              st_shared_zero16(d);
          }
          if (slot0 != 0) fence_proxy_async_smem();
          cp_async_arrive_noinc(smem_u32(&pv_full[s]));
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == 1 && lane == 0 && rank == 1) {
    // ======  peer relay: forward landed PV stages to the leader's barriers  ======
    const uint32_t lead0 = mapa_shared(smem_u32(&pv_full[0]), 0);
    PieceIter pi;
    pi.init(P.start, V, lo, hi);
    int v, x0, x1;
    uint32_t it = 0;
    bool ok = true;
    while (ok && pi.next(v, x0, x1)) {
      for (int x = x0; x < x1 && ok; ++x)
        for (int p = 0; p < 2; ++p, ++it) {
          const int s = it % kPvStages;
          if (!mbar_wait(smem_u32(&pv_full[s]), (it / kPvStages) & 1, abort_p, 14, it)) {
            ok = false;
            break;
          }
          fence_proxy_async_smem();
          mbar_arrive_cluster(lead0 + s * 8);
        }
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // =================  MMA issuer (leader CTA)  =================
    const uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
    const uint32_t idesc_pv = idesc_bf16_f32(128, 256, false, true);
    uint32_t itq = 0, itv = 0;
    int j = 0;  // block counter of this worker
    PieceIter pi;
    pi.init(P.start, V, lo, hi);
    int v, x0, x1, piece = 0;
    bool ok = true;
    int pend = -1;            // block whose PV is pending
    bool pend_first = false;  // ... is the first block of its piece
    int pend_piece = 0;
    auto issue_pv = [&](int jb, bool first, int pc) -> bool {
      if (!mbar_wait(smem_u32(&p_full), jb & 1, abort_p, 4, jb)) return false;
      if (first && pc > 0 && !mbar_wait(smem_u32(&o_empty), (pc - 1) & 1, abort_p, 5, pc))
        return false;
      tc_fence_after();
      for (int p = 0; p < 2; ++p, ++itv) {
        const int s = itv % kPvStages;
        if (!mbar_wait(smem_u32(&pv_full[s]), (itv / kPvStages) & 1, abort_p, 12, itv))
          return false;
        // The stage was written by cp.async and st.shared (generic proxy);
        // the MMA reads it through the async proxy.  The writes are ordered
        // before this thread by the barrier; the proxy fence makes them
        // visible to the MMAs this thread issues next.  (The peer's half
        // is fenced the same way by its relay lane.)
        fence_proxy_async_smem();
        tc_fence_after();
        const uint32_t st = sPv + s * kPvStageBytes;
        for (int n = 0; n < 2; ++n) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = sw128_desc(sP + p * kChunk + kk * 32, 16, 1024);
            const uint64_t bd = sw128_desc(st + n * 2 * kChunk + kk * 2048, kChunk, 1024);
            const uint32_t acc = (first && p == 0 && kk == 0) ? 0u : 1u;
            mma_bf16_ss<2>(tmem + kTmemO + 128 * n, ad, bd, idesc_pv, acc);
          }
        }
        mma_commit_2_mc(smem_u32(&pv_empty[s]), 3);
      }
      mma_commit_2_mc(smem_u32(&pv_done), 3);
      return true;
    };
    while (ok && pi.next(v, x0, x1)) {
      if (!mbar_wait(smem_u32(&q_full), piece & 1, abort_p, 6, piece)) { ok = false; break; }
      tc_fence_after();
      for (int x = x0; x < x1 && ok; ++x, ++j) {
        // QK(j) into S[j & 1]
        const uint32_t sd = tmem + kTmemS + 64 * (j & 1);
        for (int k = 0; k < 9 / kQkChunks; ++k, ++itq) {
          const int s = itq % kQkStages;
          if (!mbar_wait(smem_u32(&qk_full[s]), (itq / kQkStages) & 1, abort_p, 3, itq)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sQk + s * kQkStageBytes;
          for (int cc = 0; cc < kQkChunks; ++cc) {
            const int c = kQkChunks * k + cc;  // 64-column chunk of the 576
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = sw128_desc(sQ + c * kChunk + kk * 32, 16, 1024);
              const uint64_t bd = sw128_desc(st + cc * kChunk + kk * 32, 16, 1024);
              mma_bf16_ss<2>(sd, ad, bd, idesc_qk, (c | kk) ? 1u : 0u);
            }
          }
          mma_commit_2_mc(smem_u32(&qk_empty[s]), 3);
        }
        if (!ok) break;
        mma_commit_2_mc(smem_u32(&s_full[j & 1]), 3);
        if (x == x1 - 1) mma_commit_2_mc(smem_u32(&q_empty), 3);
        if (pend >= 0 && !issue_pv(pend, pend_first, pend_piece)) { ok = false; break; }
        pend = j; pend_first = (x == x0); pend_piece = piece;
      }
      ++piece;
    }
    if (ok && pend >= 0) ok = issue_pv(pend, pend_first, pend_piece);
    if (!ok) {
      // Leaving early: one more commit tracks every MMA issued so far; wait
      // (bounded) for it, so that no MMA still reads shared memory or writes
      // TMEM when the pair frees them.
      mma_commit_2_mc(smem_u32(&mma_drain), 1);
      mbar_wait_bounded(smem_u32(&mma_drain), 0, kDrainNs);
    }
  } else if (warp >= kSoftmaxWarp0) {
    // =================  softmax + epilogue (both CTAs)  =================
    const int tid = threadIdx.x - kSoftmaxWarp0 * 32;  // = TMEM lane
    const int h = tid & 63, half = tid >> 6;
    const uint32_t lane_addr = (uint32_t)(32 * (warp - kSoftmaxWarp0)) << 16;
    const uint32_t lead_pfull = mapa_shared(smem_u32(&p_full), 0);
    const uint32_t lead_oempty = mapa_shared(smem_u32(&o_empty), 0);
    const uint32_t prow = sP + half * kChunk + h * 128;
    PieceIter pi;
    pi.init(P.start, V, lo, hi);
    int v, x0, x1;
    int j = 0;
    bool dead = false;
    while (!dead && pi.next(v, x0, x1)) {
      const int b = v / P.R, rb = v % P.R;
      const int L = P.seq_lens[b];
      const int grow = rb * 128 + 64 * (int)rank + h;      // row within the sequence
      const int tl = P.tail != nullptr ? P.tail[b] : 0;
      const int limit = L + tl - P.S_q + grow / P.H + 1;    // visible tokens t < limit
      float m = -INFINITY, l = 0.f;
      bool o_started = false;
      for (int x = x0; x < x1; ++x, ++j) {
        const bool got = mbar_wait(smem_u32(&s_full[j & 1]), (j >> 1) & 1, abort_p, 7, j);
        uint32_t s_raw[64];
        float mx = -INFINITY;
        // token t of this lane's page: first + c - shift, valid if c >= shift
        const int first = x * kBlk + half * kPage;
        const int valid = min(L - first, kPage);
        const int shift = valid > 0 ? kPage - valid : kPage;
        const int cmax = limit - first + shift;  // columns c < cmax are visible
        if (__all_sync(0xffffffffu, got)) {
          tc_fence_after();
          uint32_t (&a)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s_raw[0]);
          uint32_t (&c2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s_raw[32]);
          const uint32_t sa = tmem + lane_addr + kTmemS + 64 * (j & 1);
          tmem_ld32(sa, a);
          tmem_ld32(sa + 32, c2);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= shift && c < cmax) mx = fmaxf(mx, __uint_as_float(s_raw[c]));
        }
        red_max[j & 1][half][h] = mx;
        // one barrier: partner's max visible, and everyone agrees to go on
        if (named_bar_or(1, 128, !got || *abort_p)) { dead = true; break; }
        mx = fmaxf(mx, red_max[j & 1][half ^ 1][h]);
        const float m_blk = mx * P.scale_log2;
        // Lazy rescale: a row moves its running max only when the block max
        // exceeds it by more than 2^kRescaleLog2.  TMEM loads/stores are
        // warp-collective, so a warp rescales when any of its rows needs it,
        // with alpha = 1 for the other rows.
        const bool need = m_blk > m + kRescaleLog2 || (m == -INFINITY && m_blk > -INFINITY);
        const float alpha = !need ? 1.f : (m == -INFINITY ? 0.f : ex2_approx(m - m_blk));
        const float m_use = need ? m_blk : m;
        uint32_t pk[32];
        float lsum = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c0 = 2 * e;
          const float p0 = (c0 >= shift && c0 < cmax)
                               ? ex2_approx(fmaf(__uint_as_float(s_raw[c0]), P.scale_log2, -m_use))
                               : 0.f;
          const float p1 = (c0 + 1 >= shift && c0 + 1 < cmax)
                               ? ex2_approx(fmaf(__uint_as_float(s_raw[c0 + 1]), P.scale_log2,
                                                 -m_use))
                               : 0.f;
          lsum += p0 + p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        // PV(j-1) must be done before P is overwritten and before O is rescaled
        bool ok = true;
        if (j > 0) ok = mbar_wait(smem_u32(&pv_done), (j - 1) & 1, abort_p, 8, j);
        if (__all_sync(0xffffffffu, ok)) {
          if (o_started && __any_sync(0xffffffffu, need)) {
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
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint32_t addr = prow + ((u ^ (h & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                         "r"(pk[4 * u]), "r"(pk[4 * u + 1]), "r"(pk[4 * u + 2]),
                         "r"(pk[4 * u + 3])
                         : "memory");
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
      // ---------------- epilogue of the piece ----------------
      const int jl = j - 1;
      const bool got = mbar_wait(smem_u32(&pv_done), jl & 1, abort_p, 10, jl);
      red_sum[half][h] = l;
      if (named_bar_or(1, 128, !got || *abort_p)) { dead = true; break; }
      tc_fence_after();
      const float lt = l + red_sum[half ^ 1][h];
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
      named_bar_sync(1, 128);  // red_sum is rewritten by the next piece
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(lead_oempty);
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
    const int32_t* seq_lens, const int32_t* tail, int B, int S_q, int H, float scale, int G,
    const int32_t* start, float* ws_lse, float* ws_o, cudaStream_t st) {
  using namespace dtc;
  CUtensorMap tQ, tQK;
  {
    const uint64_t dims[2] = {(uint64_t)kD, (uint64_t)B * S_q * H};
    const uint64_t strides[1] = {(uint64_t)kD * 2};
    const uint32_t box[2] = {64, 64};
    if (!make_tmap(&tQ, qbuf, 2, dims, strides, box)) return MLA_ERR_CUDA;
  }
  // The pool [n_pages][64 slots][576] seen as 64-column chunks: element
  // (col, slot, chunk, page) at page*73728 + slot*1152 + chunk*128 + col*2 bytes.
  {
    const uint64_t dims[4] = {64, (uint64_t)kPage, 9, (uint64_t)n_pages};
    const uint64_t strides[3] = {(uint64_t)kD * 2, 128, (uint64_t)kD * 2 * kPage};
    const uint32_t box[4] = {64, 64, (uint32_t)kQkChunks, 1};
    if (!make_tmap(&tQK, pool, 4, dims, strides, box)) return MLA_ERR_CUDA;
  }
  DecodeTcParams p;
  p.pool = static_cast<const uint8_t*>(pool);
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
  p.R = (S_q * H) / 128;
  p.G = G;
  p.scale_log2 = scale * 1.4426950408889634f;
  if (cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBytes) != cudaSuccess)
    return MLA_ERR_CUDA;
  decode_tc_kernel<<<2 * G, kThreads, kSmemBytes, st>>>(tQ, tQK, p);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
