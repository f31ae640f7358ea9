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
//     256-token blocks (four 64-token pages).  CTA r holds rows [64r, 64r+64)
//     of Q (72 KB, one TMA load per piece), resident for the whole piece.
//   * QK: pair MMAs (cta_group::2, M = 128 rows, N = 256 tokens, K = 576).
//     CTA r supplies the B half of pages 2r and 2r+1 of the block.  Each SM
//     gets its 64 rows x 256 tokens in TMEM folded onto 128 lanes x 128
//     columns: lane l < 64 holds row l, tokens 0..127; lane l >= 64 holds row
//     l - 64, tokens 128..255.  Per SM every MMA is 64 x 256 x 16, a shape
//     the tensor core runs at full rate (64 x 128 x 16 costs about as much
//     per instruction, so 256-token blocks halve the QK instruction count).
//   * PV: pair MMAs with N = 256 latent columns (two per 16-token step, one
//     per latent half n).  CTA r supplies latent columns [256n + 128r, +128)
//     of all 256 tokens (MN-major B).  A is P in TMEM: in a pair MMA, output
//     lane l reads its A row from TMEM lane l of its own CTA, so lanes l and
//     l + 64 (the same row, the two token halves of S) both need that row's
//     P for all 256 tokens, bf16 pairs in 128 columns.  P(j) overwrites S(j)
//     in place.  O takes 256 TMEM columns per SM, S/P 2 x 128 more: all 512.
//   * QK loads.  Lane 0 of warp 0 in each CTA streams its two pages through a
//     ring of three 32 KB stages; a stage holds two 64-column chunks of both
//     pages, one 16 KB TMA box per page from a 5-D view of the pool:
//     (64 columns, 8 slots, 9 chunks, 8 slot groups, pages).  The box lands as
//     [slot group][chunk][8 slots][128 B], so the two pages' slot groups of a
//     chunk sit at one uniform stride (2 KB) and form the 128-row K-major B
//     operand.  Only the leader arms each stage barrier, for both CTAs' bytes.
//     The page ids are read from the table two blocks ahead.  (L2 prefetch
//     of later blocks' pages, by bulk prefetches or by line prefetches from
//     the softmax warps, was measured slower; so were 16 KB stages.)
//   * PV loads.  Lane 0 of warp 2 fills a ring of three 16 KB stages (one
//     page x 128 latent columns) with one TMA box each from a 3-D view of
//     the pool (64 columns, pool rows, 9 chunks), which lands in the
//     MN-major operand layout; it reads the same pages the QK boxes brought
//     into L2.  The partial last page of a sequence is copied by the whole
//     warp with cp.async instead, with zeros for the slots past the end.
//   * Softmax: eight warps per CTA.  Warps w and w + 4 share TMEM lane
//     quadrant w and take 64 of its 128 columns each, so every thread holds
//     the scores of one row on one page.  Row maxima of the four pages meet
//     in shared memory.  The running max is rescaled lazily: O is rescaled
//     in TMEM only when a row's max grows by more than 2^8, warp-uniformly.
//     Full pages take a path without masks; maxima and row sums run in
//     independent chains and scores go through the packed fp32 FMA.
//     P goes to TMEM over S: warps w and w ^ 2 hold the two token halves of
//     the same rows and swap them through an 8 KB shared buffer, one warp
//     pair per round, four rounds.  P(j) waits for nothing from PV(j - 1):
//     O is rescaled (after PV(j - 1)) only when a row's max moved.  S/P
//     buffer j & 1 is released for QK(j + 2) by a commit after PV(j).
//   * MMA issue.  Two threads of the leader issue the MMAs: lane 0 of warp 1
//     the QK stream, lane 0 of warp 3 the PV stream.  The tensor pipe
//     buffers little beyond the MMA it runs, and every barrier wait, commit
//     and loop step of an issuing thread costs tens to hundreds of cycles;
//     with two issuers one stream's MMAs fill the other's gaps (a single
//     thread interleaving both streams was measured 12% slower).
//   * Pieces (sequence, block range) of a worker write normalised partial
//     outputs and natural-log LSE into slot worker + v of the workspace; the
//     combine kernel merges them.
//
// Shared memory: Q 72 KB + QK ring 96 KB + PV ring 48 KB + P exchange 8 KB
// (also the row sums of the epilogue), 1.2 KB of barriers and row maxima.
//
// Partial and missing pages.  QK boxes always load a whole page; slots past
// the sequence hold whatever the pool holds there and are masked by index in
// the softmax (P = 0).  The PV producer writes zeros for those rows, so no
// unused slot ever reaches O.  Pages past the end load entirely out of
// bounds (zeros) and their page-table entries are never read.
//
// Every mbarrier wait is bounded (MLA_WAIT_NS); on expiry the kernel raises
// MLA_ERR_TIMEOUT in the device status and every role leaves its loop.  On
// the way out the leader's producers wait (bounded) for the boxes they
// armed and each MMA issuer for a last commit of its own; then the pair
// meets at a final cluster barrier and frees its TMEM.
#pragma once

#include "common.cuh"
#include "simt.cuh"

namespace mla {

constexpr bool kDecodeTcReady = true;

namespace dtc {
constexpr int kDC = 512;             // latent width
constexpr int kD = 576;              // cached numbers per token
constexpr int kPage = 64;            // tokens per page
constexpr int kBlk = 256;            // tokens per block (four pages)
constexpr int kPageBytes = kPage * kD * 2;
constexpr int kChunk = 8192;         // 64 rows x 64 columns bf16, one swizzled operand tile
#ifndef MLA_QK_CHUNKS_PER_STAGE
#define MLA_QK_CHUNKS_PER_STAGE 2
#endif
constexpr int kQkCps = MLA_QK_CHUNKS_PER_STAGE;  // 64-column chunks per QK stage
constexpr int kQkBox = kQkCps * kChunk;         // one page x kQkCps chunks
constexpr int kQkStageBytes = 2 * kQkBox;       // both pages of this CTA
constexpr int kQkStages = 98304 / kQkStageBytes;
constexpr int kQkStagesPerBlock = (9 + kQkCps - 1) / kQkCps;
constexpr int kPvStageBytes = 2 * kChunk;  // one page x 128 latent columns
constexpr int kPvStages = 3;
constexpr int kPvStagesPerBlock = 8;       // 4 pages x 2 latent halves
constexpr int kQBytes = 9 * kChunk;        // 64 rows x 576 columns
constexpr int kXBytes = 8192;              // P exchange between TMEM lane halves
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffQk = kOffQ + kQBytes;
constexpr uint32_t kOffPv = kOffQk + kQkStages * kQkStageBytes;
constexpr uint32_t kOffX = kOffPv + kPvStages * kPvStageBytes;
constexpr uint32_t kSmemBytes = kOffX + kXBytes + 1024;  // + alignment
constexpr int kThreads = 384;
constexpr int kSoftmaxWarp0 = 4;
constexpr int kSoftmaxThreads = 256;
// registers per thread: at launch (65536 / 384, rounded down to 8), then
// after the split of the control warpgroup and the softmax warpgroups
constexpr int kRegsLaunch = 168;
constexpr int kRegsControl = 136;
constexpr int kRegsSoftmax = 184;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;       // O_n at columns [128n, 128n + 128)
constexpr uint32_t kTmemS = 256;     // S_b, then P_b, at columns [256 + 128b, +128)
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

// Arrive on named barrier `id` without waiting (a producer's half of a
// producer/consumer handoff; the consumers barrier.sync on it).
__device__ __forceinline__ void named_bar_arrive(int id, int nthreads) {
  asm volatile("barrier.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
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

// Pool page holding page p (0..3) of token block x of sequence b, or -1 when
// that page lies past the sequence (its table entry is not read).  A page id
// outside the pool raises MLA_ERR_BOUNDS and reads as -1 too.
__device__ __forceinline__ int page_of(const DecodeTcParams& P, int b, int L, int x, int p) {
  const int first = x * dtc::kBlk + p * dtc::kPage;
  if (first >= L) return -1;
  const int pg = P.page_table[(long long)b * P.max_pages + first / dtc::kPage];
  if (pg < 0 || pg >= P.n_pages) {
    raise_flag(kFlagBounds);
    return -1;
  }
  return pg;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(dtc::kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmQK,
                     const __grid_constant__ CUtensorMap tmPV,
                     const DecodeTcParams P) {
  using namespace dtc;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t qk_full[kQkStages], qk_empty[kQkStages];
  __shared__ __align__(8) uint64_t pv_full[kPvStages], pv_empty[kPvStages];
  __shared__ __align__(8) uint64_t q_full, q_empty, o_empty, p_full[2][4], pv_done, pv_last;
  __shared__ __align__(8) uint64_t s_full[2], s_free[2], drain_qk, drain_pv;
  __shared__ float red_max[4][64];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int worker = blockIdx.x >> 1;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base + kOffQ, sX = base + kOffX;
  const uint32_t sQk = base + kOffQk, sPv = base + kOffPv;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < kQkStages; ++s) {
      // full barriers: the leader's producer arrives once with the bytes of
      // both CTAs; the peer's boxes only complete transactions on it
      mbar_init(smem_u32(&qk_full[s]), 1);
      mbar_init(smem_u32(&qk_empty[s]), 1);  // MMA commit (multicast)
    }
    for (int s = 0; s < kPvStages; ++s) {
      // one arrival per CTA's PV producer (the leader's carries the
      // transaction bytes of both CTAs' boxes); only the leader's is used
      mbar_init(smem_u32(&pv_full[s]), 2);
      mbar_init(smem_u32(&pv_empty[s]), 1);
    }
    mbar_init(smem_u32(&q_full), 1);
    mbar_init(smem_u32(&q_empty), 1);
    mbar_init(smem_u32(&o_empty), 16);       // 8 softmax warps x 2 CTAs
    // P_b in TMEM, 8 softmax warps x 2 CTAs.  One barrier per P buffer: the
    // softmax of one CTA may reach block j + 1 before the other CTA's
    // softmax has handed over P(j) (nothing ties the two CTAs' softmax
    // together once P no longer waits for the previous PV), and arrivals of
    // two blocks must not meet on one barrier.  Block j + 2 cannot arrive
    // before phase j completes: its S needs PV(j) to have released the
    // buffer.
    for (int b = 0; b < 2; ++b)
      for (int pg = 0; pg < 4; ++pg) mbar_init(smem_u32(&p_full[b][pg]), 8);
    mbar_init(smem_u32(&pv_done), 1);
    mbar_init(smem_u32(&pv_last), 1);   // after the last PV of each piece
    mbar_init(smem_u32(&drain_qk), 1);
    mbar_init(smem_u32(&drain_pv), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&s_full[b]), 1);
      mbar_init(smem_u32(&s_free[b]), 1);   // PV commit: P_b consumed
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmQK);
    tma_prefetch_desc(&tmPV);
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

  // Registers: the control warpgroup (producers, MMA) gives up most
  // of its share to the two softmax warpgroups.
  static_assert(128 * kRegsControl + 256 * kRegsSoftmax <= kRegsLaunch * kThreads &&
                    kRegsLaunch * kThreads <= 65536,
                "register split exceeds the launch allocation");
  if (warp < kSoftmaxWarp0) {
    // (the register budget applies to the code it dominates)
    setmaxnreg_dec<kRegsControl>();
    if (warp == 0 && lane == 0) {
      // ==========  QK producer: Q slices and QK boxes  ==========
      const uint32_t lead_full0 = mapa_shared(smem_u32(&qk_full[0]), 0);
      const uint32_t lead_qfull = mapa_shared(smem_u32(&q_full), 0);
      uint32_t it = 0, q_issued = 0;
      PieceIter pi;
      pi.init(P.start, V, lo, hi);
      int v, x0, x1, piece = 0;
      bool ok = true;
      while (ok && pi.next(v, x0, x1)) {
        const int b = v % P.B, rb = v / P.B;
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
        // This CTA's two pages of each block: their ids are read from the
        // page table two blocks ahead of the boxes (a table read takes as
        // long as a box).
        int cur[2], nxt[2];
        for (int i = 0; i < 2; ++i) {
          cur[i] = page_of(P, b, L, x0, 2 * (int)rank + i);
          nxt[i] = x0 + 1 < x1 ? page_of(P, b, L, x0 + 1, 2 * (int)rank + i) : -1;
        }
        for (int x = x0; x < x1 && ok; ++x) {
          int nn[2], pg[2];
          for (int i = 0; i < 2; ++i) {
            nn[i] = x + 2 < x1 ? page_of(P, b, L, x + 2, 2 * (int)rank + i) : -1;
            pg[i] = cur[i] < 0 ? P.n_pages : cur[i];   // out of bounds: the box reads zeros
            cur[i] = nxt[i];
            nxt[i] = nn[i];
          }
          for (int k = 0; k < kQkStagesPerBlock; ++k, ++it) {
            const int s = it % kQkStages;
            if (!mbar_wait(smem_u32(&qk_empty[s]), ((it / kQkStages) & 1) ^ 1, abort_p, 1, it)) {
              ok = false;
              break;
            }
            const uint32_t fb = lead_full0 + s * 8;
            if (rank == 0) mbar_expect_tx(smem_u32(&qk_full[s]), 2 * kQkStageBytes);
            const uint32_t dst = sQk + s * kQkStageBytes;
            // chunks 2k, 2k+1 of each page (chunk 9 is out of bounds: zeros)
            tma_load_5d_pair(dst, &tmQK, 0, 0, kQkCps * k, 0, pg[0], fb);
            tma_load_5d_pair(dst + kQkBox, &tmQK, 0, 0, kQkCps * k, 0, pg[1], fb);
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
    } else if (warp == 2) {
      // ======  PV producer: this CTA's latent half of every page  ======
      // Stage order per block: page p = 0..3, latent half n = 0..1.  A stage
      // lands as [2 chunks][64 slots][128 B] for latent chunks 4n + 2r +
      // {0, 1} of page p, 128-byte swizzled.  A whole page, or a page past
      // the sequence (out of bounds: zeros), comes as one TMA box completing
      // on the leader's barrier, which the leader arms with both CTAs'
      // bytes.  The partial last page of a sequence is copied by the warp
      // with cp.async and zeros for the slots past the sequence: such a slot
      // holds no cache entry (possibly NaN) and must not reach the MMA even
      // though its P is 0.  Each CTA arrives once per stage on the leader's
      // barrier.
      const uint32_t lead_full0 = mapa_shared(smem_u32(&pv_full[0]), 0);
      uint32_t it = 0;
      PieceIter pi;
      pi.init(P.start, V, lo, hi);
      int v, x0, x1;
      bool ok = true;
      const int rsub = lane >> 4, cc = (lane >> 3) & 1, u = lane & 7;
      while (ok && pi.next(v, x0, x1)) {
        const int b = v % P.B;
        const int L = P.seq_lens[b];
        for (int x = x0; x < x1 && ok; ++x)
          for (int p = 0; p < 4 && ok; ++p) {
            const int pg = page_of(P, b, L, x, p);
            const int valid = pg < 0 ? 0 : min(L - (x * kBlk + p * kPage), kPage);
            for (int n = 0; n < 2; ++n, ++it) {
              const int s = it % kPvStages;
              const bool got = mbar_wait(smem_u32(&pv_empty[s]), ((it / kPvStages) & 1) ^ 1,
                                         abort_p, 11, it);
              if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
              const uint32_t dst = sPv + s * kPvStageBytes;
              const uint32_t fb = lead_full0 + s * 8;
              const int chunk0 = 4 * n + 2 * (int)rank;
              if (valid == 0 || valid == kPage) {
                if (lane == 0) {
                  if (rank == 0) mbar_expect_tx(smem_u32(&pv_full[s]), 2 * kPvStageBytes);
                  tma_load_3d_pair(dst, &tmPV, 0, (pg < 0 ? P.n_pages : pg) * kPage, chunk0, fb);
                  if (rank == 1) mbar_arrive_cluster(fb);
                }
              } else {
                const uint8_t* src =
                    P.pool + (size_t)pg * kPageBytes + (chunk0 + cc) * 128 + u * 16;
                const uint32_t d0 = dst + cc * kChunk + (u << 4);
#pragma unroll 8
                for (int i = 0; i < kPage; i += 2) {
                  const int row = i + rsub;
                  const uint32_t dsw = (d0 + row * 128) ^ ((uint32_t)(row & 7) << 4);
                  if (row < valid)
                    cp_async16(dsw, src + (size_t)row * (kD * 2));
                  else
                    st_shared_zero16(dsw);
                }
                asm volatile("cp.async.wait_all;" ::: "memory");
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                  if (rank == 0) mbar_arrive(smem_u32(&pv_full[s]));
                  else mbar_arrive_cluster(fb);
                }
              }
            }
          }
      }
      if (!ok && rank == 0 && lane == 0) {
        // Leaving early: wait (bounded) for the stages already armed, so
        // that no box lands in this pair's shared memory after it exits (the
        // peer's boxes count on the same barriers).
        for (uint32_t i = it > (uint32_t)kPvStages ? it - kPvStages : 0u; i < it; ++i)
          mbar_wait_bounded(smem_u32(&pv_full[i % kPvStages]), (i / kPvStages) & 1, kDrainNs);
      }
    } else if (warp == 1 && lane == 0 && rank == 0) {
      // =================  QK MMA issuer (leader CTA)  =================
      // QK(j) writes S buffer j & 1 once PV(j - 2) has consumed the P held
      // there (s_free).  The QK and PV streams are issued by two threads of
      // different warps: the tensor pipe holds little more than the MMA it
      // runs, so the cycles one issuer spends between MMA groups (barrier
      // waits, commits, bookkeeping) are covered by the other's MMAs.
      const uint32_t idesc_qk = idesc_bf16_f32(128, 256, false, false);
      // Operand descriptors are formed once; an MMA only adds its tile's
      // offset (in 16-byte units) to the start-address field.
      const uint64_t q_desc = sw128_desc(sQ, 16, 1024);
      // the 16 slot groups of a chunk (both pages) lie 1 KB x kQkCps apart
      const uint64_t qk_desc = sw128_desc(sQk, 16, 1024 * kQkCps);
      PieceIter qi;
      qi.init(P.start, V, lo, hi);
      int v, x0, x1, piece = 0, jq = 0;
      uint32_t itq = 0;
      bool ok = true;
      while (ok && qi.next(v, x0, x1)) {
        ok = mbar_wait(smem_u32(&q_full), piece & 1, abort_p, 4, piece);
        for (int x = x0; x < x1 && ok; ++x, ++jq) {
          if (jq >= 2 && !mbar_wait(smem_u32(&s_free[jq & 1]), ((jq - 2) >> 1) & 1, abort_p, 5, jq)) {
            ok = false;
            break;
          }
          const uint32_t sd = tmem + kTmemS + 128 * (jq & 1);
          for (int k = 0; k < kQkStagesPerBlock; ++k, ++itq) {
            const int s = itq % kQkStages;
            if (!mbar_wait(smem_u32(&qk_full[s]), (itq / kQkStages) & 1, abort_p, 6, itq)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t a0 = q_desc + (uint64_t)((kQkCps * k * kChunk) >> 4);
            const uint64_t b0 = qk_desc + (uint64_t)s * (kQkStageBytes >> 4);
#pragma unroll
            for (int cc = 0; cc < kQkCps; ++cc) {
              if (kQkCps * k + cc >= 9) break;   // past the 576 columns
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss<2>(sd, a0 + (uint64_t)((cc * kChunk + kk * 32) >> 4),
                               b0 + (uint64_t)((cc * 1024 + kk * 32) >> 4), idesc_qk,
                               (k | cc | kk) ? 1u : 0u);
            }
            mma_commit_2_mc(smem_u32(&qk_empty[s]), 3);
          }
          if (ok) mma_commit_2_mc(smem_u32(&s_full[jq & 1]), 3);
        }
        // the Q slice is free once this piece's QK MMAs completed
        if (ok) mma_commit_2_mc(smem_u32(&q_empty), 3);
        ++piece;
      }
      if (!ok) {
        // Leaving early: one more commit tracks every MMA this thread issued;
        // wait (bounded) for it, so that none still reads shared memory or
        // writes TMEM when the pair frees them.
        mma_commit_2_mc(smem_u32(&drain_qk), 1);
        mbar_wait_bounded(smem_u32(&drain_qk), 0, kDrainNs);
      }
    } else if (warp == 3 && lane == 0 && rank == 0) {
      // =================  PV MMA issuer (leader CTA)  =================
      // PV(j) begins on a page once that page of P(j) is in TMEM (the
      // softmax hands P over page by page) and, for the first block of a
      // piece, once the previous piece's epilogue has released O.  A is P(j)
      // in TMEM (S buffer j & 1): lane l holds the row of output lane l, 256
      // tokens as bf16 pairs in 128 columns, so K-step kk of page p starts at
      // column 32p + 8kk.  Once PV(j) has completed, buffer j & 1 is free for
      // QK(j + 2).
      const uint32_t idesc_pv = idesc_bf16_f32(128, 256, false, true);
      const uint64_t pv_desc = sw128_desc(sPv, kChunk, 1024);
      PieceIter vi;
      vi.init(P.start, V, lo, hi);
      int v, x0, x1, piece = 0, jp = 0;
      uint32_t itv = 0;
      bool ok = true;
      while (ok && vi.next(v, x0, x1)) {
        for (int x = x0; x < x1 && ok; ++x, ++jp) {
          if (x == x0 && piece > 0)
            ok = mbar_wait(smem_u32(&o_empty), (piece - 1) & 1, abort_p, 3, piece);
          for (int t = 0; t < kPvStagesPerBlock && ok; ++t, ++itv) {
            // page t / 2 of P(jp) is in TMEM, in all lanes of both CTAs
            if ((t & 1) == 0 &&
                !mbar_wait(smem_u32(&p_full[jp & 1][t >> 1]), (jp >> 1) & 1, abort_p, 2, jp)) {
              ok = false;
              break;
            }
            const int s = itv % kPvStages;
            if (!mbar_wait(smem_u32(&pv_full[s]), (itv / kPvStages) & 1, abort_p, 9, itv)) {
              ok = false;
              break;
            }
            // A partial-page stage was written by cp.async and st.shared
            // (generic proxy) and the MMA reads it through the async proxy.
            // Its writers fenced before arriving; the barrier orders their
            // writes before this thread, and this proxy fence orders them
            // before the MMAs issued next.
            fence_proxy_async_smem();
            tc_fence_after();
            const int pp = t >> 1, n = t & 1;
            const uint32_t a0 = tmem + kTmemS + 128 * (jp & 1) + 32 * pp;
            const uint64_t b0 = pv_desc + (uint64_t)s * (kPvStageBytes >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t acc = (x == x0 && pp == 0 && kk == 0) ? 0u : 1u;
              mma_bf16_ts<2>(tmem + kTmemO + 128 * n, a0 + 8 * kk,
                             b0 + (uint64_t)((kk * 2048) >> 4), idesc_pv, acc);
            }
            mma_commit_2_mc(smem_u32(&pv_empty[s]), 3);
          }
          if (ok) {
            mma_commit_2_mc(smem_u32(&pv_done), 3);
            mma_commit_2_mc(smem_u32(&s_free[jp & 1]), 1);
          }
        }
        if (ok) mma_commit_2_mc(smem_u32(&pv_last), 3);
        ++piece;
      }
      if (!ok) {
        mma_commit_2_mc(smem_u32(&drain_pv), 1);
        mbar_wait_bounded(smem_u32(&drain_pv), 0, kDrainNs);
      }
    }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    // =================  softmax + epilogue (both CTAs)  =================
    const int sw = warp - kSoftmaxWarp0;
    const int quad = sw & 3, ch = sw >> 2;           // TMEM lane quadrant, column half
    const int tl = 32 * quad + lane;                 // TMEM lane
    const int h = tl & 63, hh = tl >> 6;             // row of this CTA, token half
    const int pb = 2 * hh + ch;                      // page of the block this thread scores
    const uint32_t lane_addr = (uint32_t)(32 * quad) << 16;
    const uint32_t lead_pfull = mapa_shared(smem_u32(&p_full[0][0]), 0);
    const uint32_t lead_oempty = mapa_shared(smem_u32(&o_empty), 0);
    // P exchange: warp (quad q, half ch) and warp (q ^ 2, ch) hold the two
    // token halves of the same rows; the two warps writing a page use the
    // halves q & 1 of the buffer, and each reader reads its partner's half
    const uint32_t x_slot = sX + (quad & 1) * 4096 + lane * 128;
    float* red_sum = reinterpret_cast<float*>(smem_raw + (sX - smem_u32(smem_raw)));  // [4][64]
    PieceIter pi;
    pi.init(P.start, V, lo, hi);
    int v, x0, x1;
    int j = 0, pc = 0;
    bool dead = false;
    while (!dead && pi.next(v, x0, x1)) {
      const int b = v % P.B, rb = v / P.B;
      const int L = P.seq_lens[b];
      const int grow = rb * 128 + 64 * (int)rank + h;      // row within the sequence
      const int tail = P.tail != nullptr ? P.tail[b] : 0;
      const int limit = min(L, L + tail - P.S_q + grow / P.H + 1);  // visible tokens t < limit
      float m = -INFINITY, l = 0.f;
      bool o_started = false;
      for (int x = x0; x < x1; ++x, ++j) {
        const bool got = mbar_wait(smem_u32(&s_full[j & 1]), (j >> 1) & 1, abort_p, 7, j);
        float mx = -INFINITY;
        const int cmax = limit - (x * kBlk + pb * kPage);  // columns c < cmax are visible
        // a warp whose 32 rows see all 64 of their columns (every block but
        // a sequence's last, or a causal edge) takes the mask-free path
        const bool full = __all_sync(0xffffffffu, cmax >= 64);
        // this thread's 64 scores, read from TMEM (twice: for the max, then
        // for the exponentials, which keeps the registers of holding all 64
        // across the max exchange free); invisible columns (past the
        // context, causally hidden, or slots of a partial page whose contents
        // are not cache) count as -inf
        const uint32_t sa = tmem + lane_addr + kTmemS + 128 * (j & 1) + 64 * ch;
        const bool all_got = __all_sync(0xffffffffu, got);
        if (all_got) {
          tc_fence_after();
          uint32_t ra[32], rb[32];
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
        red_max[pb][h] = mx;
        // one barrier: the other pages' maxima visible, and everyone agrees
        // to go on
        if (named_bar_or(1, kSoftmaxThreads, !got || *abort_p)) { dead = true; break; }
#pragma unroll
        for (int q2 = 0; q2 < 4; ++q2) mx = fmaxf(mx, red_max[q2][h]);
        const float m_blk = mx * P.scale_log2;
        // Lazy rescale: a row moves its running max only when the block max
        // exceeds it by more than 2^kRescaleLog2.  TMEM loads/stores are
        // warp-collective, so a warp rescales when any of its rows needs it,
        // with alpha = 1 for the other rows.
        const bool need = m_blk > m + kRescaleLog2 || (m == -INFINITY && m_blk > -INFINITY);
        const float alpha = !need ? 1.f : (m == -INFINITY ? 0.f : ex2_approx(m - m_blk));
        const float m_use = need ? m_blk : m;
        // p = 2^(s * scale * log2(e) - m): pairs of scores through the packed
        // fp32 FMA, row sums over four independent packed accumulators
        uint32_t pk[32];
        float lsum;
        {
          uint32_t ra[32], rb[32];
          tmem_ld32(sa, ra);
          tmem_ld32(sa + 32, rb);
          tmem_wait_ld();
          const float2 sc2 = make_float2(P.scale_log2, P.scale_log2);
          const float2 nm2 = make_float2(-m_use, -m_use);
          float2 ls[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) ls[i] = make_float2(0.f, 0.f);
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const uint32_t s0 = e < 16 ? ra[2 * e] : rb[2 * e - 32];
            const uint32_t s1 = e < 16 ? ra[2 * e + 1] : rb[2 * e - 31];
            const float2 xx =
                __ffma2_rn(make_float2(__uint_as_float(s0), __uint_as_float(s1)), sc2, nm2);
            float p0 = ex2_approx(xx.x), p1 = ex2_approx(xx.y);
            if (!full) {
              p0 = 2 * e < cmax ? p0 : 0.f;
              p1 = 2 * e + 1 < cmax ? p1 : 0.f;
            }
            ls[e & 3] = __fadd2_rn(ls[e & 3], make_float2(p0, p1));
            pk[e] = pack_bf16x2(p0, p1);
          }
          const float2 l01 = __fadd2_rn(__fadd2_rn(ls[0], ls[1]), __fadd2_rn(ls[2], ls[3]));
          lsum = l01.x + l01.y;
        }
        // O is rescaled only when some row of this warp moved its max; PV of
        // the previous block accumulates into O and must be done first.
        bool ok = true;
        if (o_started && __any_sync(0xffffffffu, need)) {
          // parity wait: PV(j - 2) is done (S(j) needed its P buffer), so at
          // most one phase is outstanding
          ok = __all_sync(0xffffffffu,
                          mbar_wait(smem_u32(&pv_done), (j - 1) & 1, abort_p, 8, j));
          if (ok) {
            tc_fence_after();
            for (int cc = 0; cc < 4; ++cc) {
              uint32_t r[32];
              const uint32_t oa = tmem + lane_addr + kTmemO + 128 * ch + 32 * cc;
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
        // P(j) goes to TMEM over S(j), as the A operand of PV(j), page by
        // page: every lane needs its row's P on all four pages, and the two
        // warps that hold a page's rows in one lane half hand them to the two
        // warps of the other half through shared memory, one page per round.
        // PV(j) begins on page 0 while later pages are still being swapped.
        // This barrier orders every thread's reads of S and every rescale of
        // O before any write of P (and so before PV(j) starts).
        tc_fence_before();
        if (named_bar_or(2, kSoftmaxThreads, !ok || *abort_p != 0)) { dead = true; break; }
        tc_fence_after();
        const uint32_t pa = tmem + lane_addr + kTmemS + 128 * (j & 1);
        const uint32_t lead_pf = lead_pfull + 8 * (4 * (j & 1));   // p_full[j & 1][0]
        tmem_st32(pa + 32 * pb, pk);          // this thread's own page, its own lane
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(lead_pf + 8 * pb);
#pragma unroll 1
        for (int pg = 0; pg < 4; ++pg) {
          const bool writer = (hh == (pg >> 1)) && (ch == (pg & 1));
          const bool reader = (hh != (pg >> 1)) && (ch == (pg & 1));
          if (pg > 0 && writer) named_bar_sync(6 + pg, 128);   // readers of pg - 1 done
          if (writer) {
#pragma unroll
            for (int u = 0; u < 8; ++u)
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                               x_slot + ((u ^ (lane & 7)) << 4)),
                           "r"(pk[4 * u]), "r"(pk[4 * u + 1]), "r"(pk[4 * u + 2]),
                           "r"(pk[4 * u + 3])
                           : "memory");
            named_bar_arrive(3 + pg, 128);
          }
          if (reader) {
            uint32_t pq[32];
            named_bar_sync(3 + pg, 128);
#pragma unroll
            for (int u = 0; u < 8; ++u)
              asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(pq[4 * u]), "=r"(pq[4 * u + 1]), "=r"(pq[4 * u + 2]),
                             "=r"(pq[4 * u + 3])
                           : "r"(x_slot + ((u ^ (lane & 7)) << 4))
                           : "memory");
            if (pg < 3) named_bar_arrive(7 + pg, 128);          // the next writers may go
            tmem_st32(pa + 32 * pg, pq);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(lead_pf + 8 * pg);
          }
        }
        l = need ? l * alpha + lsum : l + lsum;
        m = m_use;
        o_started = true;
      }
      if (dead) break;
      // ---------------- epilogue of the piece ----------------
      // O is final once PV of the piece's last block is done: pv_last
      // completes once per piece (phase pc).  The next piece's PV waits for
      // this epilogue (o_empty), so no later phase can complete first.  (A
      // parity wait on pv_done could not tell PV(j - 2) from PV(j) when the
      // last two PVs have both completed by now.)
      const bool got = mbar_wait(smem_u32(&pv_last), pc & 1, abort_p, 10, pc);
      ++pc;
      named_bar_sync(2, kSoftmaxThreads);   // the last P swap has left the shared buffer
      red_sum[64 * pb + h] = l;
      if (named_bar_or(1, kSoftmaxThreads, !got || *abort_p)) { dead = true; break; }
      tc_fence_after();
      const float lt = red_sum[h] + red_sum[64 + h] + red_sum[128 + h] + red_sum[192 + h];
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const long long slot = (long long)worker + v;
      const long long row = slot * 128 + 64 * (int)rank + h;
      // this warp writes latent half n = ch of its lanes: columns
      // 256n + 128hh + [0, 128)
      float* dst = P.ws_o + row * kDC + 256 * ch + 128 * hh;
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_addr + kTmemO + 128 * ch + 32 * cc, r);
        tmem_wait_ld();
        float4* d4 = reinterpret_cast<float4*>(dst + 32 * cc);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          d4[i] = make_float4(__uint_as_float(r[4 * i]) * inv, __uint_as_float(r[4 * i + 1]) * inv,
                              __uint_as_float(r[4 * i + 2]) * inv,
                              __uint_as_float(r[4 * i + 3]) * inv);
      }
      if (pb == 0)
        P.ws_lse[row] = lt > 0.f ? (m + log2f(lt)) * 0.69314718055994531f : -INFINITY;
      named_bar_sync(1, kSoftmaxThreads);  // red_sum is rewritten by the next piece
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
  CUtensorMap tQ, tQK, tPV;
  {
    const uint64_t dims[2] = {(uint64_t)kD, (uint64_t)B * S_q * H};
    const uint64_t strides[1] = {(uint64_t)kD * 2};
    const uint32_t box[2] = {64, 64};
    if (!make_tmap(&tQ, qbuf, 2, dims, strides, box)) return MLA_ERR_CUDA;
  }
  // The pool [n_pages][64 slots][576] seen as (64 columns, 8 slots, 9
  // chunks, 8 slot groups, pages): element (col, s, chunk, g, page) at
  // page*73728 + (8g + s)*1152 + chunk*128 + col*2 bytes.  A box of two
  // chunks of one page lands as [g][chunk][s][64 columns].
  {
    const uint64_t dims[5] = {64, 8, 9, 8, (uint64_t)n_pages};
    const uint64_t strides[4] = {(uint64_t)kD * 2, 128, (uint64_t)kD * 2 * 8,
                                 (uint64_t)kPageBytes};
    const uint32_t box[5] = {64, 8, (uint32_t)kQkCps, 8, 1};
    if (!make_tmap(&tQK, pool, 5, dims, strides, box)) return MLA_ERR_CUDA;
  }
  // The pool seen as (64 columns, pool rows, 9 chunks): a box of two chunks
  // of one page lands as [chunk][64 slots][64 columns], the MN-major operand
  // layout of the PV MMAs.
  {
    const uint64_t dims[3] = {64, (uint64_t)n_pages * kPage, 9};
    const uint64_t strides[2] = {(uint64_t)kD * 2, 128};
    const uint32_t box[3] = {64, (uint32_t)kPage, 2};
    if (!make_tmap(&tPV, pool, 3, dims, strides, box)) return MLA_ERR_CUDA;
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
  p.R = (S_q * H + 127) / 128;  // the last row block may be padded
  p.G = G;
  p.scale_log2 = scale * 1.4426950408889634f;
  if (cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBytes) != cudaSuccess)
    return MLA_ERR_CUDA;
  decode_tc_kernel<<<2 * G, kThreads, kSmemBytes, st>>>(tQ, tQK, tPV, p);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
