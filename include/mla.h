/*
 * mla.h -- C ABI of the B200 (sm_100a) MLA decode library (libmla_b200.so).
 *
 * One decode step of DeepSeek-V2's Multi-head Latent Attention, run on the
 * compressed cache with the absorption trick.  Sources for what each call
 * computes (page address and section as printed):
 *
 *   [DF-1]  deepforge.srivtx.xyz "DeepSeek-V2", §1 "Store a latent, rebuild
 *           the keys and values" and the box "MLA: compress once,
 *           reconstruct in attention": c_t = W_DKV h_t (512-dim) plus one
 *           64-dim RoPE key are the only things cached per token per layer;
 *           k = W_UK c, v = W_UV c; being linear, W_UK folds into the query
 *           and W_UV into the output projection ("absorption").
 *   [DF-0]  same page, §1 "The bottleneck at inference time": token t's
 *           query is compared against the keys of all earlier tokens and
 *           their values are mixed (softmax attention over the cache).
 *   [CA-1]  crackai.dev "DeepSeek-V2", "How It Works": up-projections differ
 *           per head; the decoupled RoPE keys carry position separately.
 *   [DF-4]  deepforge "DeepSeek-V2", §4 "Build it yourself", stretch goals:
 *           quantize the latent to 8 bits and measure how much extra error a
 *           production cache would pay.
 *
 * Conventions shared by every call
 *   - All pointers named "device" are CUDA device pointers owned by the
 *     caller; the library never frees or retains them.  Pointers named
 *     "host" are host memory.
 *   - Element counts and strides are in ELEMENTS of the buffer's type.
 *   - dtype MLA_F32: every floating buffer is float32 and all arithmetic is
 *     fp32 (SIMT kernels).  dtype MLA_BF16: activations, weights, the query
 *     buffer and the cache are bf16 (raw 16-bit), accumulation is fp32;
 *     buffers documented as "fp32" stay fp32 in both modes.
 *   - stream is a cudaStream_t (NULL = legacy default stream).  Every call
 *     except mla_get_device_status only enqueues work; none synchronises.
 *   - Host-detectable argument errors return MLA_ERR_INVALID_ARG or
 *     MLA_ERR_UNSUPPORTED before anything is enqueued.  A launch failure
 *     returns MLA_ERR_CUDA.  Errors found on the device (a page id outside
 *     the pool, a bounded wait that ran out) set a per-device status word
 *     that mla_get_device_status reads and clears; the offending access is
 *     skipped, never performed.
 *   - The library allocates no device memory at run time.  Its only device
 *     state is a few static words per device (status, wait diagnostics) and
 *     the fixed scratch array of mla_decode_noalloc.  Callers pass in every
 *     other buffer.
 *   - Calls keep no host state beyond a launch counter: TMA descriptors are
 *     encoded for each call and passed by value to the kernels.  Calls on
 *     different streams and host threads may run concurrently, except
 *     mla_decode_noalloc, whose calls share one scratch array.
 */
#ifndef MLA_B200_H
#define MLA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,   /* null pointer, bad size or stride */
  MLA_ERR_UNSUPPORTED = 2,   /* shape the selected kernels do not cover */
  MLA_ERR_CUDA = 3,          /* a CUDA runtime call failed */
  MLA_ERR_TIMEOUT = 4,       /* device: a bounded wait ran out */
  MLA_ERR_BOUNDS = 5         /* device: an index left its buffer */
} mla_status;

typedef enum { MLA_F32 = 0, MLA_BF16 = 1 } mla_dtype;

/* Model dimensions of one MLA layer.  d_v is the value head width (= d_nope
 * for DeepSeek-V2); page_size is the number of tokens per cache page. */
typedef struct {
  int n_heads;      /* H */
  int d_nope;       /* per-head query/key width without RoPE (128) */
  int d_latent;     /* d_c, latent width (512) */
  int d_rope;       /* d_r, decoupled RoPE key width (64), even */
  int d_v;          /* per-head value width (128) */
  int d_model;      /* hidden size (5120) */
  int page_size;    /* tokens per page (64) */
  float scale;      /* softmax scale, 1/sqrt(d_nope + d_rope) */
  float rope_base;  /* RoPE base (10000) */
  mla_dtype dtype;
} mla_dims;

/* A0 -- dense projection of hidden states ([DF-1]: c_t = W_DKV h_t; the
 * query and RoPE-key projections are the same operation).
 *   y[r, o] = sum_i x[r, i] * w[o, i]      r < rows, o < out_f, i < in_f
 * x: device [rows, in_f], w: device [out_f, in_f], y: device [rows, out_f],
 * all row-major and contiguous, dtype of dims.  fp32 accumulation; bf16 y is
 * rounded to nearest even.  rows >= 0 (0 is a no-op); in_f, out_f >= 1.
 * bf16 needs in_f % 8 == 0 and 16-byte aligned x and w. */
mla_status mla_project(const mla_dims* dims, const void* x, const void* w,
                       void* y, int rows, int in_f, int out_f, void* stream);

/* A1 -- fold W_UK into the query ([DF-1] absorption):
 *   qbuf[t, i, c] = sum_n q[t, i, n] * w_uk[i, n, c],  n < d_nope, c < d_latent
 * q: device, token t head i starts at q + t*q_stride_tok + i*(d_nope+d_rope)
 *    (the first d_nope entries are read);
 * w_uk: device [H, d_nope, d_latent] contiguous;
 * qbuf: device [T, H, d_latent + d_rope] contiguous; only columns
 *    [0, d_latent) are written (mla_rope fills the rest).
 * bf16 needs q_stride_tok % 8 == 0, d_nope % 16 == 0, d_latent % 128 == 0. */
mla_status mla_absorb_q(const mla_dims* dims, const void* q, int q_stride_tok,
                        const void* w_uk, void* qbuf, int T, void* stream);

/* A2 -- rotary position embedding of RoPE parts ([DF-1] decoupled RoPE key,
 * [CA-1]).  For t < T, h < n_heads_x, k < d_rope/2 the pair
 *   (x0, x1) = (x[t*xs_tok + h*xs_head + 2k], ... + 2k + 1)
 * is rotated by the angle pos[t] * rope_base^(-2k/d_rope):
 *   y[.. 2k] = x0*cos - x1*sin,   y[.. 2k+1] = x0*sin + x1*cos.
 * The angle is formed and reduced in fp64, the rotation is done in fp32.
 * x, y: device, dtype of dims, may alias exactly (in place).  pos: device
 * int32 [T], each >= 0. */
mla_status mla_rope(const mla_dims* dims, const void* x, int xs_tok,
                    int xs_head, int n_heads_x, void* y, int ys_tok,
                    int ys_head, const int32_t* pos, int T, void* stream);

/* A3 -- append new tokens to the paged latent cache ([DF-1]: only c_t and
 * the RoPE key are written to memory).  For each t < T:
 *   page = page_table[batch_idx[t]*max_pages + pos[t]/page_size]
 *   pool[page][pos[t] % page_size][0 : d_latent]          = c[t*cs_tok ...]
 *   pool[page][pos[t] % page_size][d_latent : d_latent+d_rope] = kr[t*ks_tok ...]
 * An exact copy of the element bits.  pool: device
 * [n_pages, page_size, d_latent + d_rope]; page_table: device int32
 * [B, max_pages]; batch_idx, pos: device int32 [T].  A page id outside
 * [0, n_pages) or pos/page_size >= max_pages skips that token and raises
 * MLA_ERR_BOUNDS in the device status. */
mla_status mla_cache_append(const mla_dims* dims, const void* c, int cs_tok,
                            const void* kr, int ks_tok,
                            const int32_t* batch_idx, const int32_t* pos,
                            const int32_t* page_table, int max_pages,
                            void* pool, int n_pages, int T, void* stream);

/* 8-bit latent cache ([DF-4]: the stretch goal of quantizing the latent to
 * 8 bits).  One 656-byte row per token:
 *   bytes [0, 512)    c / s in E4M3 (1 sign, 4 exponent bits, bias 7, 3
 *                     mantissa bits; largest finite 448), nearest even,
 *                     saturating
 *   bytes [512, 640)  k_rope / s in IEEE half precision
 *   bytes [640, 644)  s = max(max|c| / 448, max|k_rope| / 65504) as fp32
 *                     (1 for an all-zero row)
 *   bytes [644, 656)  zero
 * s and the quotients are correctly rounded single-precision divisions.  The
 * cache numbers a row stands for are s * [c8 ; k16].  An 8-bit pool is
 * [n_pages][page_size][656] bytes; page tables index it as the bf16 pool.
 * Both calls need dtype MLA_BF16 (their inputs are bf16), d_latent == 512
 * and d_rope == 64 (else MLA_ERR_UNSUPPORTED), and 16-byte aligned buffers. */
#define MLA_FP8_ROW_BYTES 656

/* A3 for the 8-bit cache: quantize each new token's [c ; k_rope] (bf16, as
 * for mla_cache_append, row strides cs_tok and ks_tok multiples of 8) into
 * the slot of (batch_idx[t], pos[t]) of pool8.  A page id outside
 * [0, n_pages) skips the token and raises MLA_ERR_BOUNDS. */
mla_status mla_cache_append_fp8(const mla_dims* dims, const void* c, int cs_tok,
                                const void* kr, int ks_tok,
                                const int32_t* batch_idx, const int32_t* pos,
                                const int32_t* page_table, int max_pages,
                                void* pool8, int n_pages, int T, void* stream);

/* Quantize a whole bf16 pool [n_pages][page_size][576] into the 8-bit pool
 * [n_pages][page_size][656] row by row (same pages and slots).  Slots that
 * hold no token are converted too; their bytes are never read as cache. */
mla_status mla_cache_quantize_fp8(const mla_dims* dims, const void* pool, void* pool8,
                                  int n_pages, void* stream);

/* Workspace bytes mla_decode_fp8 needs (mla_decode's, plus a half copy of
 * the query); 0 for dims the 8-bit cache does not cover. */
size_t mla_decode_fp8_workspace_size(const mla_dims* dims, int B, int S_q,
                                     int num_workers);

/* A4 + A5 on the 8-bit cache: the attention of mla_decode over the cache
 * numbers the 8-bit rows stand for, s * [c8 ; k16] ([DF-0], [DF-1],
 * [DF-4]).  qbuf, page_table, seq_lens, o_lat, lse and the split planning
 * as for mla_decode; pool8 is the 8-bit pool [n_pages][64][656] bytes.  The
 * tensor cores compute in IEEE half precision on the stored numbers: the
 * query is converted to half (exact within half's range), the 8-bit codes
 * to half (exact), each score is the fp32 product of s and the fp32 dot
 * product, and the value product takes 64 * p * s rounded to half as its
 * weights (the 64 keeps them in half's normal range; it is divided out);
 * accumulation is fp32.  Needs dtype MLA_BF16, d_latent == 512, d_rope == 64, page_size ==
 * 64 (else MLA_ERR_UNSUPPORTED), 1 <= S_q <= 2, a 256-byte aligned workspace
 * of mla_decode_fp8_workspace_size bytes, and 16-byte aligned qbuf and
 * pool8.  Device-side errors as for mla_decode. */
mla_status mla_decode_fp8(const mla_dims* dims, const void* qbuf, const void* pool8,
                          int n_pages, const int32_t* page_table, int max_pages,
                          const int32_t* seq_lens, int B, int S_q, int num_workers,
                          void* workspace, size_t ws_bytes, float* o_lat,
                          float* lse, void* stream);

/* A1 + A2 + A3 in one call: everything between the projection and the
 * decode ([DF-1]; the pages describe the steps, not this grouping).
 * y: device [T][y_stride_tok] rows as mla_project writes them for
 * W_A0 = [W_Q; W_DKV; W_KR]:
 *   y[t] = [q_1 .. q_H | c (d_latent) | k_rope_pre (d_rope)],
 *   q_i = [q_nope (d_nope) ; q_rope (d_rope)],  y_stride_tok >= H*(d_nope+d_rope)
 *   + d_latent + d_rope.
 * Effects, each exactly as the separate call would make them:
 *   qbuf[t][i][0 : d_latent]   = W_UK,i^T q_nope        (mla_absorb_q)
 *   qbuf[t][i][d_latent : ]    = RoPE(q_rope, pos[t])    (mla_rope)
 *   y's k_rope_pre of token t  = RoPE(k_rope_pre, pos[t]), in place (mla_rope)
 *   the cache slot of (batch_idx[t], pos[t]) = [c ; roped k_rope]
 *                                                          (mla_cache_append)
 * For bf16 this is one kernel launch: the absorb GEMM's CTAs plus extra CTAs
 * for the RoPE and append work, which the GEMM does not touch.  For fp32 it
 * runs the four calls in turn.  w_uk, qbuf, batch_idx, pos, page_table, pool
 * as in those calls; the same host checks and the same MLA_ERR_BOUNDS
 * reporting apply.  bf16 needs y_stride_tok % 8 == 0. */
mla_status mla_pre_attention(const mla_dims* dims, void* y, int y_stride_tok,
                             const void* w_uk, void* qbuf,
                             const int32_t* batch_idx, const int32_t* pos,
                             const int32_t* page_table, int max_pages,
                             void* pool, int n_pages, int T, void* stream);

/* Which split kernel mla_decode runs for these dims (a plain query of the
 * dispatch, for tests and benchmarks; nothing is launched). */
typedef enum {
  MLA_DECODE_KERNEL_SIMT = 0,  /* CUDA-core kernel (fp32, and bf16 shapes the
                                  tensor-core kernel does not cover) */
  MLA_DECODE_KERNEL_TC = 1     /* tcgen05 tensor-core kernel */
} mla_decode_kernel;

/* For query blocks of S_q tokens and num_workers split workers (0 = the
 * default): *kernel receives an mla_decode_kernel value, *block_tokens the
 * number of cache tokens per work block, *workers the number of split
 * workers the planner uses (worker k takes blocks [k*total/workers,
 * (k+1)*total/workers) of all sequences' blocks in order).  Any output
 * pointer may be NULL.  Returns MLA_ERR_INVALID_ARG for bad dims or S_q
 * outside [1, 2]. */
mla_status mla_decode_config(const mla_dims* dims, int S_q, int num_workers,
                             int* kernel, int* block_tokens, int* workers);

/* Workspace bytes mla_decode needs for B sequences of S_q query tokens and
 * num_workers split workers (0 = the default mla_decode would pick). */
size_t mla_decode_workspace_size(const mla_dims* dims, int B, int S_q,
                                 int num_workers);

/* A4 + A5 -- attention of every query against the latent cache, with the
 * absorbed query ([DF-0], [DF-1]).  For sequence b with L = seq_lens[b]
 * cached tokens (the S_q query tokens included, at positions L-S_q..L-1),
 * query j and head i:
 *   s_t  = scale * qbuf[b, j, i, :] . pool_row(b, t)   over all d_latent+d_rope
 *   p    = softmax over t <= L - S_q + j
 *   o_lat[b, j, i, :] = sum_t p_t * pool_row(b, t)[0 : d_latent]
 *   lse[b, j, i]      = ln sum_t exp(s_t)
 * pool_row(b, t) = pool[page_table[b*max_pages + t/page_size]][t % page_size].
 * The token range of every sequence is split over num_workers workers
 * (0 = one per pair of SMs) with equal token counts per worker; a
 * log-sum-exp combine merges the pieces.
 * qbuf: device [B, S_q, H, d_latent + d_rope]; seq_lens: device int32 [B]
 * with S_q <= seq_lens[b] <= max_pages*page_size; o_lat: device fp32
 * [B, S_q, H, d_latent]; lse: device fp32 [B, S_q, H]; workspace: device,
 * >= mla_decode_workspace_size bytes, 256-byte aligned, contents ignored.
 * bf16 requires d_latent == 512, d_rope == 64, page_size == 64, and
 * S_q*H % 128 == 0; 1 <= S_q <= 2 in both modes. */
mla_status mla_decode(const mla_dims* dims, const void* qbuf, const void* pool,
                      int n_pages, const int32_t* page_table, int max_pages,
                      const int32_t* seq_lens, int B, int S_q, int num_workers,
                      void* workspace, size_t ws_bytes, float* o_lat,
                      float* lse, void* stream);

/* A4 + A5 on one contiguous token range of each sequence, for context
 * parallelism: the token range of a long sequence is split over several
 * caches (one per GPU), each returns the attention over its range, and
 * mla_combine_parts merges them.  The pages give the decode ([DF-0], [DF-1]);
 * the split and merge are an addition of this library.
 * Cache b here holds seq_lens[b] >= 0 tokens: global tokens
 * [G_b - seq_tail[b] - seq_lens[b], G_b - seq_tail[b]) of a sequence with G_b
 * tokens in all, at local positions 0.. in pool/page_table as for mla_decode.
 * The S_q query tokens are the last S_q of the whole sequence, so query j
 * sees local token t iff t < seq_lens[b] + seq_tail[b] - S_q + j + 1.
 * Outputs are those of mla_decode over the visible local tokens; a row that
 * sees none gets o_lat = 0 and lse = -inf.  seq_tail: device int32 [B],
 * >= 0; seq_lens[b] may be 0 (this cache holds none of sequence b).  A
 * negative length or tail, or a length past max_pages*page_size, raises
 * MLA_ERR_BOUNDS in the device status.  With seq_tail all zero and
 * seq_lens[b] >= S_q this is mla_decode.  Workspace as for mla_decode. */
mla_status mla_decode_partial(const mla_dims* dims, const void* qbuf,
                              const void* pool, int n_pages,
                              const int32_t* page_table, int max_pages,
                              const int32_t* seq_lens, const int32_t* seq_tail,
                              int B, int S_q, int num_workers, void* workspace,
                              size_t ws_bytes, float* o_lat, float* lse,
                              void* stream);

/* Merge attention results over disjoint token sets (the log-sum-exp merge of
 * mla_decode's own split-KV combine, here across callers' parts):
 *   m = max_p lse_p,  z = sum_p exp(lse_p - m),
 *   o_lat = sum_p exp(lse_p - m) * o_p / z,  lse = m + ln z,
 * with parts of lse = -inf contributing nothing and a row with no visible
 * token in any part giving o_lat = 0, lse = -inf.
 * o_parts: device fp32 [n_parts][rows][d_latent]; lse_parts: device fp32
 * [n_parts][rows]; o_lat: device fp32 [rows][d_latent]; lse: device fp32
 * [rows].  rows = B * S_q * H for mla_decode_partial outputs. */
mla_status mla_combine_parts(const mla_dims* dims, const float* o_parts,
                             const float* lse_parts, int n_parts, int rows,
                             float* o_lat, float* lse, void* stream);

/* A4 + A5 without caller-provided scratch.  The pages have no counterpart
 * for this call; it exists for callers that cannot allocate device memory:
 * code running under a host framework that owns every byte of device memory
 * through its own allocator (so a library must not allocate behind its
 * back), or latency-critical loops where cudaMalloc/cudaFree, which can
 * synchronise the device, are not allowed.
 *
 * Same arguments and results as mla_decode minus workspace/ws_bytes.  The
 * workspace lives in a fixed 64 MiB array in the library's device memory
 * (MLA_NOALLOC_SCRATCH_BYTES), which every GPU that loads the library holds
 * until the process exits.  A call whose mla_decode_workspace_size(dims, B,
 * S_q, num_workers) exceeds it returns MLA_ERR_UNSUPPORTED before launching
 * anything (the tensor-core path needs about 257 KiB per (worker + 128 query
 * rows of one sequence), e.g. 53 MiB for 128 sequences with the default 74
 * workers).  The first call on each device looks up the array's device
 * address (cudaGetSymbolAddress) with that device current; make that first
 * call before any stream capture.  Nothing in the array needs to start at
 * zero; it keeps the last call's contents.  All calls on a device share the
 * one array, so calls whose kernels overlap on the GPU (different streams
 * without ordering) race on it.  The call itself allocates nothing. */
#define MLA_NOALLOC_SCRATCH_BYTES (64u << 20)
/* The size of that array in bytes, as the library was built
 * (MLA_NOALLOC_SCRATCH_BYTES of its own copy of this header). */
size_t mla_decode_noalloc_scratch_bytes(void);
mla_status mla_decode_noalloc(const mla_dims* dims, const void* qbuf,
                              const void* pool, int n_pages,
                              const int32_t* page_table, int max_pages,
                              const int32_t* seq_lens, int B, int S_q,
                              int num_workers, float* o_lat, float* lse,
                              void* stream);

/* Scratch bytes mla_out_proj needs for T tokens. */
size_t mla_out_proj_scratch_size(const mla_dims* dims, int T);

/* A6 -- apply W_UV per head, then the output projection ([DF-1]: W_UV folds
 * into the output side):
 *   o[t, i, v]   = sum_c w_uv[i, v, c] * o_lat[t, i, c]
 *   out[t, m]    = sum_{i,v} w_o[m, i*d_v + v] * o[t, i, v]
 * o_lat: device fp32 [T, H, d_latent] (rounded to bf16 for the bf16 path);
 * w_uv: device [H, d_v, d_latent]; w_o: device [d_model, H*d_v];
 * scratch: device, >= mla_out_proj_scratch_size bytes, 256-byte aligned;
 * out: device fp32 [T, d_model]. */
mla_status mla_out_proj(const mla_dims* dims, const float* o_lat,
                        const void* w_uv, const void* w_o, void* scratch,
                        size_t scratch_bytes, float* out, int T, void* stream);

/* P1 -- chunked prefill, rebuild step ([DF-1]: k = W_UK c, v = W_UV c per
 * head; the non-absorbed form, which pays once many new queries share every
 * rebuilt key).  For the L cached tokens t < L of ONE sequence:
 *   ctx[t, :]       = pool[page_row[t / page_size]][t % page_size][:]
 *   k_nope[t, i, n] = sum_c w_uk[i, n, c] * ctx[t, c]      c < d_latent
 *   v[t, i, e]      = sum_c w_uv[i, e, c] * ctx[t, c]
 * pool: device [n_pages, page_size, d_latent + d_rope]; page_row: device
 * int32, the sequence's page-table row (ceil(L / page_size) entries are
 * read); w_uk: device [H, d_nope, d_latent]; w_uv: device [H, d_v,
 * d_latent]; ctx: device [L, d_latent + d_rope] (out); k_nope: device
 * [L, H, d_nope] (out); v: device [L, H, d_v] (out).  fp32 accumulation,
 * outputs rounded to bf16.  bf16 only, DeepSeek-V2 widths (d_nope = d_v =
 * 128, d_latent = 512, d_rope = 64), else MLA_ERR_UNSUPPORTED.  All buffers
 * 16-byte aligned.  L = 0 is a no-op.  A page id outside [0, n_pages)
 * zeroes that row of ctx and raises MLA_ERR_BOUNDS in the device status. */
mla_status mla_prefill_rebuild_kv(const mla_dims* dims, const void* pool, int n_pages,
                                  const int32_t* page_row, int L, const void* w_uk,
                                  const void* w_uv, void* ctx, void* k_nope, void* v,
                                  void* stream);

/* P2 -- chunked prefill attention, causal ([DF-0]), on the rebuilt keys and
 * values ([DF-1]: k_{i,t} = [k_nope[t, i, :] ; ctx[t, d_latent:]], the RoPE
 * key shared by all heads; v_{i,t} = v[t, i, :]).  The T queries are the
 * last T tokens of the sequence: query j sits at position L - T + j and
 * attends to the tokens t <= L - T + j.  For j < T and head i:
 *   s_t = scale * (q[j, i, :] . k_{i,t}),   p = softmax of s over those t
 *   o[j, i, :] = sum_t p_t v[t, i, :],       lse[j, i] = ln sum_t exp(s_t)
 * q: device bf16, query j head i at q + j*q_stride_tok + i*(d_nope+d_rope),
 * [q_nope ; q_rope] with RoPE already applied (e.g. the A0 output after
 * mla_rope in place); ctx, k_nope, v: as written by mla_prefill_rebuild_kv;
 * o: device bf16 [T, H, d_v] (out, the input of the W_O projection, which
 * mla_project applies); lse: device fp32 [T, H] (out).  0 <= T <= L
 * (T = 0 is a no-op); q_stride_tok % 8 == 0; shapes as for
 * mla_prefill_rebuild_kv; all buffers 16-byte aligned. */
mla_status mla_prefill_attention(const mla_dims* dims, const void* q, int q_stride_tok,
                                 const void* ctx, const void* k_nope, const void* v, int T,
                                 int L, void* o, float* lse, void* stream);

/* Synchronises `stream`, then returns and clears the device status word of
 * the current device (MLA_OK, MLA_ERR_TIMEOUT or MLA_ERR_BOUNDS; TIMEOUT
 * wins if both were raised), or MLA_ERR_CUDA if the stream failed. */
mla_status mla_get_device_status(void* stream);

/* Where the first bounded wait that ran out on the current device gave up
 * since the last call: out4 = {site, info, parity, CTA index}, all zero if
 * none did.  Sites: 1-10 split-decode kernel (1 producer slot free, 2 query
 * slice free, 3 MMA operands landed, 4 P ready, 5 O free, 6 query landed,
 * 7 S ready, 8-10 PV done), 21-23 GEMM, 30-39 prefill attention (30 value
 * stage free, 31 key stage free, 32 query landed, 33 keys landed, 34 P ready,
 * 35 values landed, 36 S buffer free, 37 S ready, 38-39 PV done).  Reads and clears the record
 * (synchronous copy; call after mla_get_device_status). */
mla_status mla_get_wait_diag(uint32_t* out4);

/* Static, human-readable text for a status code. */
const char* mla_status_string(mla_status s);

/* Self-test of the failure path: enqueues one kernel whose only wait is on
 * an mbarrier that nothing completes, bounded to wait_ns nanoseconds; the
 * kernel then raises MLA_ERR_TIMEOUT in the device status and returns.  No
 * fault, trap or hang is involved. */
mla_status mla_selftest_wait_timeout(unsigned long long wait_ns, void* stream);

/* Number of kernel launches the library has enqueued since load (for
 * benchmark bookkeeping; incremented on the host). */
uint64_t mla_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* MLA_B200_H */
