/*
 * decattn.h -- C ABI of libdecattn.so: GQA decode attention over a paged KV
 * cache with dynamic split-KV scheduling, for NVIDIA B200 (sm_100a).
 *
 * The operation ("PaddlePaddle/HALOps" README, Highlights, GQA attention item):
 * paged-KV decode attention with BF16 or FP8 KV cache, grouped-query heads and
 * speculative decoding (several query tokens per request), with split-KV
 * parallelism and an adaptive reduction.
 * The scheduling ("HPC-Ops: Tencent's CUDA Kernel Library for LLM Inference Hot
 * Paths", section "How the kernels are organized around specific workload
 * shapes"): before each decode step the requests are cut into uniform KV tiles,
 * the tiles are balanced across CTAs by greedy bin-packing, and a combine
 * kernel merges the split results.
 *
 * For query row (b, t, qh) with h = qh / (n_q_heads / n_kv_heads) and KV length
 * Lb = seq_lens[b], the visible keys are j = 0 .. Lb - T + t (the T query
 * tokens are the last T tokens of the cache; bottom-right causal). With
 * s_j = sm_scale * <q[b][t][qh], K[b,h,j]>:
 *     out[b][t][qh] = sum_j softmax(s)_j * V[b,h,j],   lse[b][t][qh] = ln sum_j e^{s_j}.
 * K[b,h,j] is row (j % P) of block [page_table[b][j / P]][h] of k_pages (FP8:
 * the code's value times kv_scales[0][page][h]; V likewise with kv_scales[1]).
 * A row with no visible key gets out = 0 and lse = -inf.
 *
 * Conventions for every call:
 *  - "device" pointers are CUDA device memory on the current device; "host"
 *    pointers are ordinary host memory. The caller allocates and owns every
 *    buffer; the library never allocates, never frees and keeps no state
 *    between calls other than per-device attributes it caches.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). dec_attn_plan and
 *    dec_attn_run only enqueue work on it: they never synchronise, so both may
 *    be captured into a CUDA graph.
 *  - Errors that the host can see (null or misaligned pointers, unsupported
 *    shapes, buffers too small) return a negative decattn_status and enqueue
 *    nothing. Errors only the device can see (a page id outside the pool, more
 *    tiles than the plan can hold, a pipeline wait that gives up) never trap:
 *    they set a status word in the plan buffer's header, which
 *    dec_attn_read_status() returns.
 *  - The planner, split and combine kernels are chained with programmatic
 *    dependent launch: each later kernel may be scheduled while the earlier one
 *    drains and waits on the device until it has finished.
 */
#ifndef DECATTN_H
#define DECATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DECATTN_API __attribute__((visibility("default")))
#else
#define DECATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DECATTN_OK = 0,
  DECATTN_EINVAL = -1,   /* invalid argument: null pointer, negative size, inconsistent plan/shape */
  DECATTN_ENOTSUP = -2,  /* valid but unsupported: head_dim, page size, tile length, group size, dtype */
  DECATTN_ESMALL = -3,   /* a caller buffer (plan or workspace) is too small */
  DECATTN_ECUDA = -4,    /* a CUDA runtime call failed (launch, attribute query) */
  DECATTN_ETIMEOUT = -5, /* device: a pipeline wait gave up (the kernel returned early) */
  DECATTN_EDEVICE = -6,  /* device: bad input seen by a kernel (page id outside the pool, negative
                            seq_len, seq_len beyond the page-table row) */
  DECATTN_EALIGN = -7,   /* a pointer is not 16-byte aligned */
  DECATTN_ECAPACITY = -8 /* device: the tiles of seq_lens exceed the plan's capacity */
} decattn_status;

/* KV element type of the pools, and how the products are formed:
 *   DECATTN_KV_BF16          bf16 pages;
 *   DECATTN_KV_FP8E4M3       OCP E4M3 pages with fp32 per-(page, KV head) scales; q keeps bf16
 *                            precision (two E4M3 parts) and P keeps about 12 significant bits
 *                            (three E4M3 parts on the tcgen05 kernel, head_dim 128 and G*T <= 16;
 *                            f16 hi + lo on the warp-MMA kernel otherwise): the result is checked
 *                            against the fp64 oracle on the dequantised pages (out 2e-3, lse 1e-4);
 *   DECATTN_KV_FP8E4M3_MMA8  the same pages and scales, with both products on E4M3 tensor cores
 *                            (the HPC-Ops article at sdftguanye.com, section on fine-grained task
 *                            scheduling and data rearrangement: an FP8 attention kernel): q rounded to
 *                            one E4M3 part per row (power-of-two row scale 2^E, E = 7 -
 *                            floor(log2 max|q_row|)), and P rounded to E4M3 after scaling by
 *                            (V page scale) * C, C a power of two per 128-key chunk. Its own
 *                            tolerance: the oracle runs on the rounded q, and P's rounding is
 *                            bounded per row (see the tests). head_dim 128 and G*T <= 16 only
 *                            (DECATTN_ENOTSUP otherwise). */
typedef enum { DECATTN_KV_BF16 = 0, DECATTN_KV_FP8E4M3 = 1, DECATTN_KV_FP8E4M3_MMA8 = 2 } decattn_kv_dtype;

/* Host-side handle of a plan. dec_attn_plan fills it; dec_attn_run reads it. The
 * work list itself lives in the caller's device buffer `buf`. */
typedef struct {
  void *buf;          /* device: plan buffer (header + tile list), caller-owned */
  size_t buf_bytes;
  int32_t batch;
  int32_t n_kv_heads;
  int32_t tile_len;   /* tokens per uniform KV tile */
  int32_t n_bins;     /* CTAs of the split kernel; one bin of tiles per CTA */
  int64_t max_units;  /* capacity of the tile list */
  int32_t sparse;     /* 1 for a plan made by dec_attn_plan_sparse */
  int32_t reserved_;
} dec_attn_plan_t;

/* Problem shape shared by dec_attn_workspace_bytes and dec_attn_run. */
typedef struct {
  int32_t batch;              /* B >= 0 requests */
  int32_t n_q_heads;          /* Hq, a multiple of n_kv_heads */
  int32_t n_kv_heads;         /* Hkv */
  int32_t head_dim;           /* d: 64 or 128 */
  int32_t q_tokens;           /* T >= 1 query tokens per request (T > 1: speculative decode) */
  int32_t page_size;          /* P tokens per page: a multiple of 16, at most 256 */
  int32_t num_pages;          /* pages in the pool */
  int32_t max_pages_per_seq;  /* row stride of page_table */
  int32_t kv_dtype;           /* decattn_kv_dtype */
  float sm_scale;             /* softmax scale; <= 0 selects 1/sqrt(head_dim) */
} dec_attn_shape;

/* Number of bins (split-kernel CTAs) the library uses on `device` when a plan is
 * made with n_bins = 0: SM count x CTAs resident per SM. Returns < 0 on error. */
DECATTN_API int dec_attn_default_bins(int device);

/* A tile length for dec_attn_plan, from sizes the host knows. The pages fix uniform KV tiles
 * ("HPC-Ops ...", "How the kernels are organized around specific workload shapes") but give no
 * rule for their length; this one weighs the two costs the length trades: long tiles leave the
 * busiest CTA more tokens than the average (the greedy bins differ by up to one tile), short
 * tiles write and re-read more partial results and pay a fixed cost per tile more often.
 * Candidates are page_size * 2^k up to 8192; with U = n_kv_heads * total_kv_tokens / tl tiles
 * over n_bins bins, the estimate is
 *   ceil(U / n_bins) * (tl * 2 * head_dim * elem + 8192) + U * rows * (head_dim + 1) * 8 / n_bins
 * (elem = 2 for bf16, 1 for E4M3; rows = G * T query rows per KV head; 8192 = the fixed cost of a
 * tile in KV bytes). The smallest estimate wins, the shorter tile on a tie. Host only (no CUDA
 * call): n_bins > 0 must be given, e.g.
 * dec_attn_default_bins(device). Returns the tile length (a multiple of page_size and of 16), or
 * DECATTN_EINVAL for invalid arguments. */
DECATTN_API int dec_attn_default_tile_len(int batch, int n_kv_heads, int64_t total_kv_tokens, int page_size,
                                          int head_dim, int rows_per_kv_head, int kv_dtype, int n_bins);

/* Bytes of the device plan buffer for a plan of `batch` requests whose KV lengths
 * sum to at most max_total_kv_tokens. n_bins = 0 selects dec_attn_default_bins of
 * the current device. Returns 0 for invalid arguments. */
DECATTN_API size_t dec_attn_plan_bytes(int batch, int n_kv_heads, int tile_len, int64_t max_total_kv_tokens, int n_bins);

/* Planner ("HPC-Ops ...", "How the kernels are organized around specific workload
 * shapes": uniform KV tiles assigned before each decode step and balanced across
 * CTAs by greedy bin-packing). One single-block kernel on `stream`:
 *   1. each pair (b, h) is cut into n_b = ceil(Lb / tile_len) tiles
 *      [i*tl, min((i+1)*tl, Lb)); cost of a tile = its token count;
 *   2. tiles are stably sorted by cost, largest first ((b, h, i) order on ties);
 *   3. in that order each tile goes to the least-loaded bin (lowest index on ties);
 *   4. a bin keeps its tiles in assignment order.
 * A tile of a pair with n_b > 1 writes its partial result to slot
 * pair_off[b*Hkv+h] + i; a pair with n_b == 1 writes the final output directly.
 *   seq_lens  device int32 [batch]: KV length of each request (>= 0).
 *   tile_len  > 0 and a multiple of 16; dec_attn_run further needs it to be a
 *             multiple of the page size.
 *   plan_buf  device, plan_bytes >= dec_attn_plan_bytes(...), 16-byte aligned.
 *   plan      host, filled on success.
 * Device-side failures (sum of tiles above capacity, negative seq_len) set the
 * plan's status (DECATTN_ECAPACITY / DECATTN_EDEVICE); a later dec_attn_run then
 * writes nothing and reports the same status. */
DECATTN_API int dec_attn_plan(const int32_t *seq_lens, int batch, int n_kv_heads, int tile_len, int64_t max_total_kv_tokens,
                  int n_bins, void *plan_buf, size_t plan_bytes, dec_attn_plan_t *plan, void *stream);

/* Block-sparse decode planner ("HPC-Ops ...", "How the kernels are organized around specific
 * workload shapes": sparse attention takes a precomputed block mask and skips the masked-out KV
 * tiles). Same greedy rule as dec_attn_plan, over the kept tiles only:
 *   tile_mask  device uint32 [batch][n_kv_heads][mask_words]: bit i % 32 of word i / 32 of row
 *              (b, h) keeps tile i = keys [i*tl, min((i+1)*tl, Lb)) of request b, KV head h;
 *              bits of tiles past a request's last tile are ignored, tiles past the row's
 *              mask_words words count as masked; 4-byte aligned.
 * Every query row of (b, h) then attends to the keys of the kept tiles only (with the causal
 * rule for T > 1); a pair with no kept tile gets out = 0, lse = -inf. A pair's kept tiles are
 * numbered j = 0, 1, ... in tile order; their partial slots are the prefix over pairs of kept
 * tiles plus j, and a pair with one kept tile writes the final output. The plan is used with
 * dec_attn_run / dec_attn_split / dec_attn_combine / dec_attn_plan_export unchanged; its
 * buffer needs dec_attn_plan_sparse_bytes (4 bytes per tile of capacity more than a dense plan).
 * Per-tile FP8 scales are the case of per-(page, head) scales equal across a tile's pages.
 * Other arguments, errors and the launch as dec_attn_plan. */
DECATTN_API size_t dec_attn_plan_sparse_bytes(int batch, int n_kv_heads, int tile_len, int64_t max_total_kv_tokens,
                                              int n_bins);
DECATTN_API int dec_attn_plan_sparse(const int32_t *seq_lens, const uint32_t *tile_mask, int mask_words, int batch,
                                     int n_kv_heads, int tile_len, int64_t max_total_kv_tokens, int n_bins,
                                     void *plan_buf, size_t plan_bytes, dec_attn_plan_t *plan, void *stream);

/* Writes the explicit work list of a finished plan (the device plan stores full tiles in
 * closed form): bin_off device int32 [n_bins + 1] (CSR offsets), units device int32
 * [max_units][8] with one record per tile {b, h, tok_begin, tok_end, seq_len, slot, i, 0}
 * in bin order, and *n_units (device int32) = the tile count, or -1 if the plan failed or
 * max_units is too small. seq_lens must be the values the plan was made from. One
 * single-block kernel on `stream`; for tests and diagnostics. */
DECATTN_API int dec_attn_plan_export(const dec_attn_plan_t *plan, const int32_t *seq_lens, int32_t *bin_off,
                                     void *units, int64_t max_units, int32_t *n_units, void *stream);

/* Bytes of the device workspace dec_attn_run needs: room for the partial (o, lse)
 * of every tile the plan can hold (fp32, [tiles][G*T][d+1]) after a 256-byte
 * reserved header.
 * Returns 0 for invalid arguments. */
DECATTN_API size_t dec_attn_workspace_bytes(const dec_attn_shape *shape, const dec_attn_plan_t *plan);

/* Split + combine ("PaddlePaddle/HALOps" README, Highlights, GQA attention item;
 * "HPC-Ops ...", "How the kernels are organized around specific workload
 * shapes": a combine kernel merges the split results). Enqueues, on `stream`:
 *   - the split kernel: CTA k walks bin k of the plan; for each tile it stages the
 *     page-table-indirected K/V rows through a shared-memory pipeline (TMA), computes
 *     the G*T query rows of its KV head against them with an online softmax in
 *     fp32 and writes the tile's normalised partial (o, lse) -- or, for a request
 *     held in one tile, the final out/lse;
 *   - the combine kernel: merges the partials of every row by log-sum-exp:
 *     M = max_i lse_i, w_i = e^{lse_i - M}, out = sum_i w_i o_i / sum_i w_i,
 *     lse = M + ln sum_i w_i (a partial with no visible key has lse -inf, weight 0).
 * Arguments (all device pointers 16-byte aligned, except page_table, seq_lens, lse):
 *   q          bf16 [B][T][Hq][d]
 *   k_pages    [num_pages][Hkv][P][d], bf16 or FP8 E4M3 ("fn") codes
 *   v_pages    same layout as k_pages
 *   page_table int32 [B][max_pages_per_seq]: physical page of logical page p of
 *              request b (entries past ceil(Lb/P) are not read)
 *   seq_lens   int32 [B]: must hold the values the plan was made from
 *   kv_scales  fp32 [2][num_pages][Hkv] (K scales, then V scales); FP8 only, else NULL
 *   plan       host handle from dec_attn_plan (same batch and n_kv_heads)
 *   workspace  device, workspace_bytes >= dec_attn_workspace_bytes(shape, plan)
 *   out        fp32 [B][T][Hq][d];  lse  fp32 [B][T][Hq] (natural log)
 * Supported: head_dim 64 or 128; page_size a multiple of 16 up to 256;
 * tile_len a multiple of page_size; q_tokens T <= 8 and G*T <= 64 query rows per KV head
 * (G = n_q_heads / n_kv_heads: grouped-query heads and speculative tokens together). Anything
 * else returns DECATTN_ENOTSUP before any launch. */
DECATTN_API int dec_attn_run(const dec_attn_shape *shape, const void *q, const void *k_pages, const void *v_pages,
                 const int32_t *page_table, const int32_t *seq_lens, const float *kv_scales,
                 const dec_attn_plan_t *plan, void *workspace, size_t workspace_bytes, float *out, float *lse,
                 void *stream);

/* Size of the fixed device scratch behind dec_attn_run_noalloc: 64 MiB per GPU. */
#define DECATTN_NOALLOC_SCRATCH_BYTES (64u << 20)

/* dec_attn_run without a caller-supplied workspace, for callers that cannot allocate device
 * memory: a plugin hosted by an engine that owns all device memory through its own pool and
 * offers no allocation hook, or a deployment that fixes its device memory budget up front and
 * forbids allocation while decoding. It allocates nothing (no cudaMalloc / cudaFree, no
 * allocating library call): the workspace is a file-scope device array of
 * DECATTN_NOALLOC_SCRATCH_BYTES inside this library. The pages describe no such variant; it
 * is a deployment convenience of this library.
 *   Arguments, results and errors as dec_attn_run, minus workspace / workspace_bytes.
 *   DECATTN_ESMALL if dec_attn_workspace_bytes(shape, plan) exceeds the scratch (nothing is
 *   enqueued then); DECATTN_ECUDA if the scratch's device address cannot be looked up.
 *   The first call on a device (with that device current) looks up the array's device address
 *   and loads the module that holds it; make that first call before any stream capture. The
 *   array then stays allocated on that GPU until the process exits. The address is cached per
 *   device together with the CUDA context it was looked up in, and is valid in that context
 *   only: after cudaDeviceReset the next call finds a new context and looks it up again (so
 *   that call, too, should come before any capture).
 *   All calls on one device share the array; its contents are left over from the last call and
 *   need no clearing (the split kernel writes every partial the combine reads and resets the
 *   combine counters). Calls whose work overlaps on the GPU (e.g. on two streams) race on it:
 *   serialise them. */
DECATTN_API int dec_attn_run_noalloc(const dec_attn_shape *shape, const void *q, const void *k_pages,
                                     const void *v_pages, const int32_t *page_table, const int32_t *seq_lens,
                                     const float *kv_scales, const dec_attn_plan_t *plan, float *out, float *lse,
                                     void *stream);

/* The two stages of dec_attn_run as separate calls (same arguments, same checks):
 * dec_attn_split enqueues only the split kernel, dec_attn_combine only the combine
 * kernel, which reads the partials the split kernel left in `workspace`. dec_attn_run(...) ==
 * dec_attn_split(...) followed by dec_attn_combine(...) on the same stream. Useful to time or
 * overlap the stages. The split kernel zeroes the combine's per-row counters, and the combine
 * returns every counter it used to zero after merging its row, so dec_attn_combine may also be
 * repeated on the partials of one dec_attn_split (e.g. to time the combine alone). */
DECATTN_API int dec_attn_split(const dec_attn_shape *shape, const void *q, const void *k_pages, const void *v_pages,
                               const int32_t *page_table, const int32_t *seq_lens, const float *kv_scales,
                               const dec_attn_plan_t *plan, void *workspace, size_t workspace_bytes, float *out,
                               float *lse, void *stream);
DECATTN_API int dec_attn_combine(const dec_attn_shape *shape, const void *q, const void *k_pages, const void *v_pages,
                                 const int32_t *page_table, const int32_t *seq_lens, const float *kv_scales,
                                 const dec_attn_plan_t *plan, void *workspace, size_t workspace_bytes, float *out,
                                 float *lse, void *stream);

/* Synchronises `stream`, then returns the planner's status if it failed, else the
 * first device-detected error of any split kernel run on this plan since the plan
 * was made (the planner clears it), else DECATTN_OK. `workspace` is accepted for
 * symmetry with dec_attn_run and not read. For tests and diagnostics, not for the
 * hot path. */
DECATTN_API int dec_attn_read_status(const dec_attn_plan_t *plan, const void *workspace, void *stream);

/* The CUDA error behind the last DECATTN_ECUDA returned on the calling host thread: the failing
 * step and CUDA's error string, e.g. "prefill kernel launch: too many resources requested for
 * launch". Writes at most len - 1 characters and a terminating zero into buf (NULL: nothing
 * written); returns the full message length (0: no DECATTN_ECUDA on this thread yet). Host only. */
DECATTN_API size_t dec_attn_last_error(char *buf, size_t len);

/* For tests of the bounded pipeline waits; the pages have no counterpart (it exists so that the
 * failure path of every wait can be exercised without a GPU fault). Every mbarrier wait of the
 * split and prefill kernels gives up after a limit (2 s by default), sets DECATTN_ETIMEOUT and
 * lets the CTA leave in order (copies already issued land first, tensor memory is freed). This
 * call sets, for the launches that follow it in this process:
 *   limit_ns   the wait limit in ns, 1e5 .. 2e9 (0: back to the default);
 *   skip_fill  >= 0: CTA 0's producer leaves that one pipeline fill out (ring fill of the split
 *              kernels, K block of the prefill kernel), so that the waits on it run out and the
 *              run ends with DECATTN_ETIMEOUT; -1: none (the default).
 * Returns DECATTN_EINVAL for values outside those ranges. Not thread-safe against launches on
 * other threads; not for production use. */
DECATTN_API int dec_attn_test_set_waits(uint64_t limit_ns, int32_t skip_fill);

/* Static text for a decattn_status value. */
DECATTN_API const char *dec_attn_status_string(int status);

/* Fused pre-processing of a decode step ("PaddlePaddle/HALOps" README, Highlights, GQA
 * attention item: fused pre/post-processing around paged-KV decode). The pages name the step
 * without defining it; the reading implemented, in one kernel on `stream`:
 *   - rotary position embedding, rotate-half form: for i < d/2, theta_i = rope_base^(-2i/d),
 *     and the pair (x_i, x_{i+d/2}) of a row at position pos becomes
 *     (x_i cos(pos theta_i) - x_{i+d/2} sin(pos theta_i), x_{i+d/2} cos(pos theta_i) + x_i sin(pos theta_i)),
 *     computed in fp32 from an fp64 angle and rounded to bf16 (nearest, ties to even);
 *   - the T = shape->q_tokens new tokens of request b sit at positions Lb - T + t, t < T:
 *     seq_lens must already count them, exactly as dec_attn_run expects;
 *   - q_out[b][t][qh] = rotated q_new[b][t][qh]; the rotated k_new[b][t][h] and the unchanged
 *     v_new[b][t][h] are written to page page_table[b][pos / P], slot pos % P, of KV head h;
 *   - a token with pos < 0 (Lb < T) has no slot: nothing is written for it and its q row is
 *     copied unrotated (the rotation at position 0).
 * Run it before dec_attn_plan / dec_attn_run of the same step, on the same stream, passing
 * q_out as their q. It is launched with programmatic stream serialisation and waits for the
 * previous kernel of the stream before reading anything.
 * Arguments (device pointers; 4-byte aligned for head_dim 128, 2-byte for 64):
 *   shape       batch, n_q_heads, n_kv_heads, head_dim (64 or 128), q_tokens, page_size,
 *               num_pages, max_pages_per_seq, kv_dtype (DECATTN_KV_BF16 only; sm_scale unused)
 *   q_new       bf16 [B][T][Hq][d];  k_new, v_new  bf16 [B][T][Hkv][d]
 *   page_table  int32 [B][max_pages_per_seq];  seq_lens  int32 [B]
 *   rope_base   > 0 (10000 in the usual configuration)
 *   q_out       bf16 [B][T][Hq][d], may be q_new (rotated in place)
 *   k_pages, v_pages  bf16 [num_pages][Hkv][P][d], updated in place
 *   status      optional device int32: a page id outside [0, num_pages), or a page past the
 *               row's max_pages_per_seq entries, skips that token's K/V write and sets
 *               DECATTN_EDEVICE here (first error wins; the caller zeroes it). May be NULL.
 * Returns DECATTN_ENOTSUP for FP8 KV (dec_attn_append_rope_fp8 takes those pools and their
 * scales) or another head_dim, DECATTN_EINVAL / DECATTN_EALIGN for bad
 * arguments (nothing enqueued), DECATTN_ECUDA if the launch fails. */
DECATTN_API int dec_attn_append_rope(const dec_attn_shape *shape, const void *q_new, const void *k_new,
                                     const void *v_new, const int32_t *page_table, const int32_t *seq_lens,
                                     float rope_base, void *q_out, void *k_pages, void *v_pages, int32_t *status,
                                     void *stream);

/* dec_attn_append_rope for an E4M3 cache (the same passage: fused pre/post-processing around
 * paged-KV decode over a BF16 / FP8 KV cache). The pages give one scale per (page, KV head) and do
 * not say how a page takes new rows; the reading implemented keeps the scale covering the page's
 * valid rows (|value| <= 448 * scale) and re-rounds older rows only when it must:
 *   - q rows: exactly as dec_attn_append_rope (rotated, rounded to bf16, into q_out);
 *   - per page and KV head touched by the new tokens, separately for K and V: x = the new rows'
 *     values (k rotated as above, in fp32), A = max |x| over the page's new rows; the page's older
 *     rows are its slots before the first new one. The scale becomes s' = max(s, A / 448) when there
 *     are older rows, else A / 448 (1 when A = 0). When s' > s every older code c is re-rounded to
 *     E4M3(value(c) * (s / s')); the new rows are stored as E4M3(x / s'). E4M3(.) is fp32 rounded to
 *     the nearest E4M3 value, ties to even, saturating at +-448.
 * Arguments as dec_attn_append_rope, with shape->kv_dtype DECATTN_KV_FP8E4M3 (or _MMA8: the same
 * pages), k_pages / v_pages E4M3 codes [num_pages][Hkv][P][d] (no alignment needed) and
 *   kv_scales  device fp32 [2][num_pages][Hkv] (K scales, then V), updated in place, 4-byte aligned.
 * Two kernels on `stream` (q rows, then the pages), each waiting for the previous kernel before it
 * reads. Pages of different requests must be distinct (as for every entry point); a page id outside
 * the pool sets DECATTN_EDEVICE in `status` and that page is left unwritten. Returns
 * DECATTN_ENOTSUP for a bf16 shape or another head_dim, DECATTN_EINVAL / DECATTN_EALIGN for bad
 * arguments (nothing enqueued), DECATTN_ECUDA if a launch fails. */
DECATTN_API int dec_attn_append_rope_fp8(const dec_attn_shape *shape, const void *q_new, const void *k_new,
                                         const void *v_new, const int32_t *page_table, const int32_t *seq_lens,
                                         float rope_base, void *q_out, void *k_pages, void *v_pages, float *kv_scales,
                                         int32_t *status, void *stream);

/* Prefill: causal attention of many query rows per request over the paged KV cache (the
 * prefill side of "PaddlePaddle/HALOps" README, Highlights, GQA attention item: variable-length
 * prefill and paged-KV decode over a BF16 KV cache, GQA). The shape's q_tokens = T query rows of
 * request b are its last T positions, already in the pages: row t attends to keys
 * 0 .. seq_lens[b] - T + t (the decode's bottom-right causal rule; rows before position 0 see
 * nothing and get out = 0, lse = -inf). Output as dec_attn_run (out fp32 [B][T][Hq][128], lse
 * natural log [B][T][Hq]); no plan and no workspace. Runs on tcgen05 tensor cores: one CTA per
 * two tiles of 128 query rows that read the same keys (two q heads of one KV head when
 * n_q_heads / n_kv_heads is even, else two adjacent row blocks of one head); q, K and V arrive by
 * TMA in 128-key blocks, and out is written by TMA stores (so q and out need the 16-byte
 * alignment below; their rows are 256 and 512 bytes). Rows of a request are independent of the
 * other requests: no cross-request state.
 *   shape       batch, n_q_heads, n_kv_heads, head_dim (128), q_tokens (T >= 1), page_size (a
 *               multiple of 16), num_pages, max_pages_per_seq, kv_dtype (DECATTN_KV_BF16),
 *               sm_scale (0: 1/sqrt(head_dim));
 *   q           device bf16 [B][T][Hq][128], 16-byte aligned;
 *   k_pages, v_pages, page_table, seq_lens   as dec_attn_run;
 *   out, lse    device fp32 outputs (out 16-byte aligned);
 *   status      optional device int32 (may be NULL): DECATTN_EDEVICE for a page id outside the
 *               pool or a negative length, DECATTN_ETIMEOUT if a pipeline wait gave up.
 * Returns DECATTN_ENOTSUP for other dtypes, head dims or page sizes, DECATTN_EINVAL /
 * DECATTN_EALIGN for bad arguments (nothing is launched), DECATTN_ECUDA if the launch fails. */
DECATTN_API int dec_attn_prefill(const dec_attn_shape *shape, const void *q, const void *k_pages, const void *v_pages,
                                 const int32_t *page_table, const int32_t *seq_lens, float *out, float *lse,
                                 int32_t *status, void *stream);

/* Variable-length prefill (the same passage: "variable-length prefill"): request b has its own
 * number of query rows Tb = cu_q_lens[b + 1] - cu_q_lens[b] >= 0, its last Tb positions, and the
 * rows of all requests are packed back to back. Row t < Tb of request b is packed row
 * cu_q_lens[b] + t and attends to keys 0 .. seq_lens[b] - Tb + t (rows before position 0 see
 * nothing: out = 0, lse = -inf). By definition each request is computed as dec_attn_prefill of
 * that request alone with T = Tb. Same kernel and tolerances as dec_attn_prefill.
 *   shape        as dec_attn_prefill, with q_tokens = the largest Tb of the batch (>= 1): it sizes
 *                the grid; a request with more rows is reported as below and left unwritten;
 *   q            device bf16 [total_q_rows][Hq][128], 16-byte aligned;
 *   cu_q_lens    device int32 [batch + 1]: non-decreasing row offsets, cu_q_lens[0] = 0 and
 *                cu_q_lens[batch] = total_q_rows (4-byte aligned);
 *   total_q_rows host: the number of packed rows;
 *   out, lse     device fp32 [total_q_rows][Hq][128] and [total_q_rows][Hq] (out 16-byte aligned);
 *   status       optional device int32: DECATTN_EDEVICE also when a request's offsets fall outside
 *                [0, total_q_rows] or its Tb exceeds q_tokens (that request is not written).
 * The ragged last 32-row group of each request is written with plain stores, the rest by TMA
 * stores, so rows of one request never overwrite another's. Returns as dec_attn_prefill. */
DECATTN_API int dec_attn_prefill_varlen(const dec_attn_shape *shape, const void *q, const void *k_pages,
                                        const void *v_pages, const int32_t *page_table, const int32_t *seq_lens,
                                        const int32_t *cu_q_lens, int64_t total_q_rows, float *out, float *lse,
                                        int32_t *status, void *stream);

/* Prefill over an FP8 (E4M3) KV cache (the same passage: prefill and paged-KV decode across
 * BF16 / FP8 KV caches). The same attention as dec_attn_prefill / dec_attn_prefill_varlen over
 * the dequantised cache, K = code * (page scale) and V likewise (the scales of
 * dec_attn_run's DECATTN_KV_FP8E4M3). Two launches on the stream: a pass widens the pages each
 * request uses into the workspace, K and V as RN_bf16(RN_fp32(code * scale)) (a relative error
 * of at most 2^-9 per element against the exact product), in a bf16 pool laid out like the
 * caller's (page i of request b at b * max_pages_per_seq + i) with its own page table; then the
 * bf16 prefill kernel runs on it. So the result differs from attention over the exact products
 * by the effect of that rounding on scores and values, besides the bf16 kernel's own.
 *   shape         as dec_attn_prefill with kv_dtype DECATTN_KV_FP8E4M3;
 *   q             device bf16 [B][T][Hq][128] (cu_q_lens NULL) or [total_q_rows][Hq][128] (packed);
 *   k_pages, v_pages   device E4M3 [num_pages][Hkv][P][128], 16-byte aligned;
 *   kv_scales     device fp32 [2][num_pages][Hkv] (K scales, then V), 4-byte aligned;
 *   page_table, seq_lens   as dec_attn_run;
 *   cu_q_lens     NULL: every request has q_tokens rows and total_q_rows must be batch * q_tokens;
 *                 else as dec_attn_prefill_varlen;
 *   workspace     device, 16-byte aligned, at least dec_attn_prefill_fp8_workspace_bytes(shape)
 *                 bytes (caller-owned; its contents are overwritten);
 *   out, lse, status   as dec_attn_prefill (status also reports a page id outside the pool seen by
 *                 the widening pass).
 * Returns DECATTN_ESMALL if the workspace is too small and otherwise as dec_attn_prefill; every
 * check happens before the first launch (nothing is enqueued on an error). */
DECATTN_API int64_t dec_attn_prefill_fp8_workspace_bytes(const dec_attn_shape *shape);
DECATTN_API int dec_attn_prefill_fp8(const dec_attn_shape *shape, const void *q, const void *k_pages,
                                     const void *v_pages, const float *kv_scales, const int32_t *page_table,
                                     const int32_t *seq_lens, const int32_t *cu_q_lens, int64_t total_q_rows,
                                     void *workspace, int64_t workspace_bytes, float *out, float *lse,
                                     int32_t *status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* DECATTN_H */
