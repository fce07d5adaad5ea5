/*
 * ds4a.h -- C ABI of the B200 (sm_100a) DeepSeek-V4 hybrid attention hot path:
 * KV compressor, Lightning-Indexer top-k, and shared K=V multi-query attention
 * with a per-head sink merged with the sliding window (CSA), or over every
 * pooled entry (HCA).
 *
 * Sources of the operations (page title, then section / equation):
 *   [V4-inside] "DeepSeek V4 Inside: One Token Through Every Block"
 *   [beyond]    "DeepSeek-v4 Beyond Basics", sections 3.2.2 and 3.3
 *   [module1]   "Phase 1 Module 1 - The model & the cost of attention"
 *   [hf-doc]    "DeepSeek-V4" (Transformers documentation)
 *
 * Conventions shared by every call
 * --------------------------------
 * - Ownership: the caller owns every buffer.  The library allocates nothing
 *   per call; scratch memory ("workspace") is passed in by the caller and
 *   sized by the *_workspace queries.  Library state: one device error word
 *   per device, and an optional launch trace (ds4a_trace_*), off by default.
 * - Execution: every call is asynchronous on the given CUDA stream (NULL =
 *   the legacy default stream).  Pointers named "device" must be device (or
 *   managed) memory of the current device; "host" pointers are host memory.
 * - Host threads: the compute calls may be made from several host threads
 *   at once (the library's host state is a few per-device caches, filled
 *   once under atomics or a lock); the launch trace is not thread safe, and
 *   ds4a_check reads and clears the one error word of the current device.
 * - Overlap: the library's kernels are launched with programmatic dependent
 *   launch, so a kernel may start while the library kernel before it on the
 *   stream is still running.  It waits for that kernel before it reads what
 *   a library call writes (pool, scores, indices, workspace) and before it
 *   writes anything, but it may read its pure inputs (queries, raw C/Z
 *   rows, weights, positions, window rows) earlier.  Those inputs must
 *   therefore not be written by a still-running library kernel: produce
 *   them with ordinary stream work (any kernel or copy that is not part of
 *   this library orders fully), never by feeding one call's output buffer
 *   to the next call as an input.
 * - Storage types: ds4a_bf16 is a bfloat16 bit pattern.  Arithmetic is
 *   float32 (bf16 x bf16 products accumulated in float32 on tensor cores).
 * - Layouts: contiguous row-major, dimensions listed outermost first; batch
 *   strides, where given, are in elements.  Every bf16 / float / int32 array
 *   must start on a 16-byte boundary.
 * - Positions are absolute and 0-based.  A compressed entry i of ratio m is
 *   visible to a query at position t iff i < floor((t + 1) / m).  The window
 *   of a query at t is positions max(0, t - window + 1) .. t, read from a
 *   ring at slot (position mod win_cap).
 * - Return codes: DS4A_OK, or DS4A_EINVAL (null / misaligned pointer, bad
 *   size or configuration; nothing is launched), DS4A_EUNSUPPORTED (no kernel
 *   for this shape), DS4A_ECUDA (a launch failed), DS4A_ENOSPACE (workspace
 *   too small).  Errors found by kernels (an index out of range, a negative
 *   position, a bounded wait that ran out) are recorded in the device error
 *   word and reported by ds4a_check; kernels never trap.
 */
#ifndef DS4A_H
#define DS4A_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t ds4a_bf16;
typedef struct CUstream_st* ds4a_stream; /* same type as cudaStream_t */

enum {
  DS4A_OK = 0,
  DS4A_EINVAL = 1,
  DS4A_EUNSUPPORTED = 2,
  DS4A_ECUDA = 3,
  DS4A_EDEVICE = 4,
  DS4A_ETIMEOUT = 5,
  DS4A_ENOSPACE = 6
};

/* Bits of the device error word (ds4a_check). */
enum {
  DS4A_DEV_BAD_INDEX = 1u, /* an index >= N_c or < -1 was skipped             */
  DS4A_DEV_BAD_POS = 2u,   /* a negative query position was skipped          */
  DS4A_DEV_TIMEOUT = 4u    /* a bounded wait inside a kernel ran out          */
};

/* One attention layer.  Flash-0731 CSA: {64, 512, 64, 128, 64, 128, 512, 4,
 * 1/sqrt(512), 10000, 1e-6}; HCA: the same with ratio 128 ([V4-inside]
 * config JSON and knob table).
 *   n_heads   query heads H (all share one K=V head)
 *   head_dim  D, channels of a query head and of a K=V row
 *   rope_dim  R, the last R channels carry interleaved-pair RoPE
 *   window    W, sliding-window length (0 = no window)
 *   idx_heads H_I, idx_dim D_I: indexer heads and their width
 *   topk      k, entries kept by the indexer
 *   ratio     m, tokens per compressed entry (CSA 4, HCA 128)
 *   sm_scale  softmax scale (1/sqrt(D))
 *   rope_base theta_j = rope_base^(-2j/R)
 *   rms_eps   RMSNorm epsilon */
typedef struct ds4a_layer_cfg {
  int32_t n_heads, head_dim, rope_dim, window, idx_heads, idx_dim, topk, ratio;
  float sm_scale, rope_base, rms_eps;
} ds4a_layer_cfg;

/*
 * ds4a_compress -- KV compressor ([beyond] 3.2.2 eqs. 9-12 for CSA with
 * overlapping blocks; 3.3 eqs. 20-23 for HCA; [V4-inside] "How does CSA
 * compress 8 tokens into 4 KV entries?").
 *
 * For entry i and channel ch, one softmax over the logits
 *   Z^a[i*m + r][ch] + B^a[r][ch]                     (r < m, own block)
 *   Z^b[(i-1)*m + r][ch] + B^b[r][ch]                 (r < m, previous block;
 *                                                      CSA only, i >= 1)
 * weights the matching C^a / C^b values; their sum is the entry.  With
 * norm_g the entry is then RMS-normalised (eps cfg->rms_eps) times norm_g,
 * and RoPE at position i*m rotates its last cfg->rope_dim channels.  Without
 * norm_g (indexer keys) the weighted sum is stored as is.
 *
 *   B, T_tok, c   streams ca/cb/za/zb are device bf16 [B, T_tok, c]; row r is
 *                 token tok_begin + r.  cb == NULL (and zb, bias_b NULL)
 *                 selects the single-stream HCA form.
 *   bias_a/b      device float [m, c] (m = cfg->ratio)
 *   norm_g        device float [c] or NULL
 *   entries       entry_begin .. entry_end-1 are written; every token they
 *                 read must lie in [tok_begin, tok_begin + T_tok)
 *   pool          device bf16; entry i of batch b goes to
 *                 pool + b * pool_bstride + i * c
 * c must be even and <= 1024, and a multiple of 8 when above 512 (a
 * multiple of 8 takes 16-byte vector loads);
 * cfg->rope_dim <= c when norm_g is given.
 */
int ds4a_compress(const ds4a_layer_cfg* cfg, int B, int T_tok, int tok_begin, int c,
                  const ds4a_bf16* ca, const ds4a_bf16* cb, const ds4a_bf16* za,
                  const ds4a_bf16* zb, const float* bias_a, const float* bias_b,
                  const float* norm_g, int entry_begin, int entry_end, ds4a_bf16* pool,
                  int64_t pool_bstride, ds4a_stream stream);

/* Bytes of the per-layer compressor state ds4a_compress_append keeps for B
 * sequences of width c: overlap != 0 (CSA, two streams) holds 4 streams
 * (C^a, C^b, Z^a, Z^b) x 2m token rows; overlap == 0 (HCA) 2 streams (C, Z)
 * x m rows; bf16 each. */
size_t ds4a_compress_state_bytes(const ds4a_layer_cfg* cfg, int B, int c, int overlap);

/*
 * ds4a_compress_append -- the compressor's decode-time cache ([hf-doc] cache
 * layers: the CSA / HCA compressors keep a buffer of raw rows, a count and,
 * for CSA, the overlap state between calls; the entries are those of
 * ds4a_compress, [beyond] 3.2.2 eqs. 9-12 and 3.3 eqs. 20-23).
 *
 * One call per decoded token.  Sequence b's new token at position pos[b]
 * brings its rows ca[b], za[b] (and cb[b], zb[b] for CSA); they are stored in
 * the sequence's state at slot pos[b] mod 2m (CSA) or mod m (HCA).  When the
 * token closes entry i = (pos[b] + 1) / m - 1 (that is, (pos[b] + 1) mod m
 * == 0), the entry is compressed from the state exactly as ds4a_compress
 * computes it from the full streams and written to pool[b][i]; otherwise
 * nothing else happens.  Sequences may sit at different positions.
 *
 *   pos       device int32 [B]; every sequence must append its tokens in
 *             order, one per call (the state holds only the last 2m or m
 *             tokens; rows of tokens never appended read as whatever the
 *             state held -- zero it to start a sequence at position 0)
 *   ca .. zb  device bf16 [B, c]: the new token's rows (cb == NULL: HCA)
 *   bias_a/b, norm_g   as ds4a_compress
 *   state     device bf16, ds4a_compress_state_bytes(cfg, B, c, cb != NULL)
 *             bytes, caller-owned, layout [B][stream][slot][c]
 *   N_cap     pool capacity in entries; an entry index >= N_cap is skipped
 *             and recorded as DS4A_DEV_BAD_INDEX, a negative position as
 *             DS4A_DEV_BAD_POS
 *   pool      device bf16, entry i of sequence b at pool + b * pool_bstride
 *             + i * c
 * The state is read after the preceding library kernels finish (it is a
 * library output), so calls chain on one stream without host syncs.
 */
int ds4a_compress_append(const ds4a_layer_cfg* cfg, int B, int c, const int32_t* pos,
                         const ds4a_bf16* ca, const ds4a_bf16* cb, const ds4a_bf16* za,
                         const ds4a_bf16* zb, const float* bias_a, const float* bias_b,
                         const float* norm_g, ds4a_bf16* state, int N_cap, ds4a_bf16* pool,
                         int64_t pool_bstride, ds4a_stream stream);

/*
 * Block-scaled cache storage ([V4-inside] "What does HCA change?", paper
 * 2.3.4: the K=V cache keeps its RoPE dims in BF16 and the other dims in FP8;
 * the indexer keys are FP4).  Element formats and block scaling after the
 * OCP Microscaling (MX) formats: 32 consecutive values share one
 * power-of-two scale stored as E8M0 (exponent + 127), the smallest power of
 * two that keeps the block's largest magnitude within the element format;
 * elements round to nearest even.  FP8 is E4M3 (largest 448), FP4 is E2M1
 * (largest 6).
 *
 *   DS4A_MX_KV_FP8   one K=V entry of D dims (the last R in BF16) is a row of
 *                    ds4a_kv_fp8_row_bytes(D, R) bytes:
 *                      [0, D-R)          E4M3 codes of dims 0 .. D-R-1
 *                      [D-R, D+R)        BF16 of dims D-R .. D-1, as stored
 *                      [D+R, D+R+(D-R)/32)  E8M0 scales, one per 32 dims
 *                      zero padding to a multiple of 16 (592 bytes at the
 *                      Flash shape D = 512, R = 64)
 *   DS4A_MX_IDX_FP4  one indexer key of D_I dims is D_I/2 bytes of E2M1 codes
 *                    (element 2i in the low nibble) in a codes array, and
 *                    D_I/32 E8M0 scales in a separate scales array
 * Strides of block-scaled pools are in entries (rows).
 */
enum { DS4A_MX_KV_FP8 = 1, DS4A_MX_IDX_FP4 = 2 };

/* Bytes of one DS4A_MX_KV_FP8 row (0 when D - R is not a multiple of 32 or
 * R not a multiple of 8). */
size_t ds4a_kv_fp8_row_bytes(int D, int R);

/* bf16 K=V rows in[n][in_stride] -> DS4A_MX_KV_FP8 rows out (out_stride
 * bytes apart, a multiple of 16).  Device pointers, 16-byte aligned. */
int ds4a_quantize_kv_fp8(int n_rows, int D, int R, const ds4a_bf16* in, int64_t in_stride, uint8_t* out,
                         int64_t out_stride, ds4a_stream stream);

/* bf16 indexer keys in[n][in_stride] (D a multiple of 32) -> codes [n][D/2]
 * and scales [n][D/32] (DS4A_MX_IDX_FP4).  Device pointers; in and codes
 * 16-byte aligned. */
int ds4a_quantize_idx_fp4(int n_rows, int D, const ds4a_bf16* in, int64_t in_stride, uint8_t* codes,
                          uint8_t* scales, ds4a_stream stream);

/*
 * ds4a_compress_append_mx -- ds4a_compress_append writing the entries in a
 * block-scaled format: the entry is computed as ds4a_compress_append does,
 * rounded to bf16 (the ABI's storage type), then quantised.
 *   format   DS4A_MX_KV_FP8 (K=V entries; R = cfg->rope_dim when norm_g is
 *            given, else 0) or DS4A_MX_IDX_FP4 (indexer keys)
 *   pool     device, entry i of sequence b at row b * pool_bstride + i of
 *            the format's rows (FP8: row bytes; FP4: c/2 code bytes)
 *   scales   FP4 only: device, c/32 bytes per entry, same row numbering
 *   pool_bstride  entries between sequences (>= N_cap)
 * c must be a multiple of 64 and c - R a multiple of 32 (DS4A_EUNSUPPORTED
 * otherwise).  Everything else is as ds4a_compress_append.
 */
int ds4a_compress_append_mx(const ds4a_layer_cfg* cfg, int B, int c, const int32_t* pos,
                            const ds4a_bf16* ca, const ds4a_bf16* cb, const ds4a_bf16* za,
                            const ds4a_bf16* zb, const float* bias_a, const float* bias_b,
                            const float* norm_g, ds4a_bf16* state, int N_cap, int format, uint8_t* pool,
                            uint8_t* scales, int64_t pool_bstride, ds4a_stream stream);

/*
 * ds4a_compress_append_jobs -- one decode step of up to two compressors of
 * the same layer (a CSA layer's K=V entries and its indexer keys) in one
 * call: each job is exactly ds4a_compress_append (format 0) or
 * ds4a_compress_append_mx (format DS4A_MX_*) with the fields below, and
 * the same B, positions and N_cap.  Two CSA-shaped jobs (overlap, c a
 * multiple of 8) run in one launch, so the second does not wait for the
 * first; otherwise the jobs run one after the other.  (No counterpart on
 * the pages: a launch-count choice.)
 */
typedef struct ds4a_append_job {
  int32_t c;                          /* channels */
  int32_t format;                     /* 0 (bf16 entries), DS4A_MX_KV_FP8 or DS4A_MX_IDX_FP4 */
  const ds4a_bf16 *ca, *cb, *za, *zb; /* the new token's rows [B, c]; cb NULL: HCA form */
  const float *bias_a, *bias_b;       /* [m, c] */
  const float* norm_g;                /* [c] or NULL */
  ds4a_bf16* state;                   /* ds4a_compress_state_bytes(cfg, B, c, cb != NULL) bytes */
  void* pool;                         /* bf16 entries, or the block-scaled rows */
  uint8_t* scales;                    /* FP4 scales, else NULL */
  int64_t pool_bstride;               /* elements (bf16) or entries (block-scaled) between sequences */
} ds4a_append_job;

int ds4a_compress_append_jobs(const ds4a_layer_cfg* cfg, int B, const int32_t* pos, int N_cap,
                              const ds4a_append_job* jobs, int n_jobs, ds4a_stream stream);

/* Bytes of workspace ds4a_index_topk needs for these sizes. */
size_t ds4a_index_topk_workspace(const ds4a_layer_cfg* cfg, int B, int T_q, int N_c);

/*
 * ds4a_index_topk -- Lightning Indexer score and top-k selector ([beyond]
 * 3.2.2 eqs. 13-17; [module1] "The indexer"; [hf-doc] mask layout).
 *
 *   I[t][s] = sum_h w[t][h] * ReLU(q[t][h] . K[s])   for visible s
 * keeps the cfg->topk highest scores per query (ties to the lower index) and
 * writes their indices ascending, padded with -1 when fewer are visible.
 *
 *   q_pos   device int32 [B, T_q]      query positions
 *   q_idx   device bf16 [B, T_q, H_I, D_I]
 *   w_idx   device bf16 [B, T_q, H_I]
 *   k_idx   device bf16, batch b's entries at k_idx + b * k_bstride,
 *           [N_c, D_I] each (the indexer-key pool)
 *   idx_out device int32 [B, T_q, k]
 *   score_out device float [B, T_q, k] (score of each kept index, -inf for
 *           -1 slots) or NULL
 *   ws      device workspace of ws_bytes >= ds4a_index_topk_workspace(...)
 */
int ds4a_index_topk(const ds4a_layer_cfg* cfg, int B, int T_q, const int32_t* q_pos,
                    const ds4a_bf16* q_idx, const ds4a_bf16* w_idx, const ds4a_bf16* k_idx,
                    int64_t k_bstride, int N_c, int32_t* idx_out, float* score_out, void* ws,
                    size_t ws_bytes, ds4a_stream stream);

/*
 * ds4a_index_topk_fp4 -- ds4a_index_topk over FP4 indexer keys
 * (DS4A_MX_IDX_FP4): the score uses the keys' exact values (code times
 * scale); queries and weights stay bf16.
 *   k_codes   device, batch b's keys at k_codes + (b * k_bstride) * D_I/2
 *   k_scales  device, batch b's keys at k_scales + (b * k_bstride) * D_I/32
 *   k_bstride keys between sequences, a multiple of 4
 * The Flash indexer shape only (64 heads x 128), N_c a multiple of 4
 * (DS4A_EUNSUPPORTED otherwise); both arrays 16-byte aligned.
 */
int ds4a_index_topk_fp4(const ds4a_layer_cfg* cfg, int B, int T_q, const int32_t* q_pos,
                        const ds4a_bf16* q_idx, const ds4a_bf16* w_idx, const uint8_t* k_codes,
                        const uint8_t* k_scales, int64_t k_bstride, int N_c, int32_t* idx_out,
                        float* score_out, void* ws, size_t ws_bytes, ds4a_stream stream);

/*
 * ds4a_index_topk_noalloc -- ds4a_index_topk for callers that cannot
 * allocate device memory (engines that reserve all HBM for their caches at
 * start-up, C plugin hosts that pass no allocator, decode loops that must
 * avoid cudaMalloc/cudaFree's implicit synchronisation).  The pages have no
 * counterpart: it is an interface choice of this library.
 *
 * Same arguments and result as ds4a_index_topk without the workspace: the
 * score scratch is a device array inside the library, 2^21 floats (8 MiB),
 * held by every GPU that loads the library until the process exits.
 *   - B * T_q * N_c above 2097152 returns DS4A_ENOSPACE (use
 *     ds4a_index_topk with a workspace instead).
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current); make that first call before any
 *     stream capture.
 *   - Every call on a device shares the one array: calls whose kernels
 *     overlap on the GPU (other streams, other host threads) race.  The
 *     array keeps the last call's contents; a call reads only scores it has
 *     written itself, so nothing needs clearing.
 *   - It calls no cudaMalloc, cudaFree or allocating library routine.
 */
int ds4a_index_topk_noalloc(const ds4a_layer_cfg* cfg, int B, int T_q, const int32_t* q_pos,
                            const ds4a_bf16* q_idx, const ds4a_bf16* w_idx,
                            const ds4a_bf16* k_idx, int64_t k_bstride, int N_c,
                            int32_t* idx_out, float* score_out, ds4a_stream stream);

/* Bytes of workspace the attend calls can use for these sizes: the float
 * partial results of key splits, which spread the keys of few queries over
 * more SMs.  Passing less (NULL included) is allowed: the work is then split
 * less, down to one split per query, which needs none. */
size_t ds4a_attend_workspace(const ds4a_layer_cfg* cfg, int B, int T_q, int N_c, int sparse);

/*
 * ds4a_sparse_attend -- CSA core attention ([beyond] 3.2.2 eq. 19 and 3.3
 * eqs. 24-27; [V4-inside] layer-0 SWA sink example and the CSA example with
 * one compressed and two window keys; [hf-doc] partial RoPE, sink, window).
 *
 * Per query (b, t) at position p and head h:
 *   q^ = RoPE_p(RMSNorm(q[b][t][h]) * q_norm_g)
 *   keys = pool[idx[b][t][j]] for idx >= 0, then the window rows
 *   z = q^ . kv * sm_scale;  p = exp(z) / (sum exp(z) + exp(sink[h]))
 *   o = sum p * kv;  out[b][t][h] = RoPE_{-p}(o) on the last R channels
 * K and V are the same row (shared K=V MQA).
 *
 *   q       device bf16 [B, T_q, H, D]; q_norm_g device float [D]
 *   pool    device bf16, batch b at pool + b * pool_bstride, [N_c, D]
 *   idx     device int32 [B, T_q, k] ascending, -1 padded (ds4a_index_topk)
 *   win     device bf16, batch b at win + b * win_bstride, [win_cap, D]: the
 *           raw K=V rows of the window, slot = position mod win_cap
 *   sink    device float [H]
 *   out     device bf16 [B, T_q, H, D]
 *   ws      device workspace (may be NULL with ws_bytes 0)
 */
int ds4a_sparse_attend(const ds4a_layer_cfg* cfg, int B, int T_q, const int32_t* q_pos,
                       const ds4a_bf16* q, const float* q_norm_g, const ds4a_bf16* pool,
                       int64_t pool_bstride, int N_c, const int32_t* idx, const ds4a_bf16* win,
                       int win_cap, int64_t win_bstride, const float* sink, ds4a_bf16* out,
                       void* ws, size_t ws_bytes, ds4a_stream stream);

/*
 * ds4a_hca_attend -- HCA core attention ([beyond] 3.3; [V4-inside] "What
 * does HCA change?"; [hf-doc] HCA layer).  As ds4a_sparse_attend with the
 * keys = every visible pool entry (i < floor((p+1)/m), i < N_c), then the
 * window.  With N_c = 0 it is the sliding-window-only layer.
 */
int ds4a_hca_attend(const ds4a_layer_cfg* cfg, int B, int T_q, const int32_t* q_pos,
                    const ds4a_bf16* q, const float* q_norm_g, const ds4a_bf16* pool,
                    int64_t pool_bstride, int N_c, const ds4a_bf16* win, int win_cap,
                    int64_t win_bstride, const float* sink, ds4a_bf16* out, void* ws,
                    size_t ws_bytes, ds4a_stream stream);

/* Grouped low-rank output projection of one layer ([beyond] 3.3 after eq.
 * 26; [V4-inside] layer-0 section, grouped W_O with the 64 Flash heads in
 * o_groups = 8; [hf-doc] grouped o_a projection followed by o_b).  Flash:
 * {64, 512, 8, 1024, 4096}.
 *   n_heads, head_dim  H, D of the attention output
 *   n_groups           g: consecutive heads H/g form a group
 *   group_rank         r: width of a group's intermediate projection
 *   hidden             width of the layer's output */
typedef struct ds4a_oproj_cfg {
  int32_t n_heads, head_dim, n_groups, group_rank, hidden;
} ds4a_oproj_cfg;

/* Bytes of workspace ds4a_out_proj needs for M tokens: when M is too small
 * for the row and output tiles to fill the SMs, K is split and each split's
 * float partial sums are kept apart and added in split order (the result
 * does not depend on scheduling); else 0. */
size_t ds4a_out_proj_workspace(const ds4a_oproj_cfg* cfg, int M);

/*
 * ds4a_out_proj -- for each token t:
 *   mid[t][j*r + i] = sum_c W_a[j][i][c] * o[t][j*(H/g)*D + c]   (group j)
 *   y[t][n]         = sum_c W_b[n][c] * mid[t][c]                (c < g*r)
 * with bf16 storage and float32 accumulation on the tensor cores (mid is
 * stored as bf16 and read back by the second product).
 *
 *   o     device bf16 [M, H, D] (the attention output, heads in order)
 *   w_a   device bf16 [g][r][(H/g)*D]  (each group's weight, rows = outputs)
 *   w_b   device bf16 [hidden][g*r]
 *   mid   device bf16 [M, g*r]  (output)
 *   y     device bf16 [M, hidden] (output)
 *   ws    device workspace of ds4a_out_proj_workspace(cfg, M) bytes
 * (H/g)*D must be a multiple of 64, r and hidden multiples of 256
 * (DS4A_EUNSUPPORTED otherwise).
 */
int ds4a_out_proj(const ds4a_oproj_cfg* cfg, int M, const ds4a_bf16* o, const ds4a_bf16* w_a,
                  const ds4a_bf16* w_b, ds4a_bf16* mid, ds4a_bf16* y, void* ws, size_t ws_bytes,
                  ds4a_stream stream);

/* Failure-detection self test (no counterpart on the pages): launches one
 * block that waits, through the same bounded mbarrier wait the tensor-core
 * kernels use, on a barrier no thread ever arrives at, with a limit of
 * limit_cycles SM cycles (1 .. 2^32) instead of the kernels' ~2 s.  The
 * wait runs out, the block records DS4A_DEV_TIMEOUT in the error word,
 * writes 2 to *status_out (device int32; 1 would mean the barrier
 * completed) and exits, so ds4a_check then returns DS4A_ETIMEOUT and the
 * context stays usable.  No GPU fault is involved. */
int ds4a_selftest_wait_timeout(int64_t limit_cycles, int32_t* status_out, ds4a_stream stream);

/*
 * ds4a_sparse_attend_fp8 / ds4a_hca_attend_fp8 -- ds4a_sparse_attend and
 * ds4a_hca_attend over a DS4A_MX_KV_FP8 pool: every pool row enters the
 * products with its exact values (E4M3 code times the block's scale, the
 * RoPE dims as stored); window rows stay bf16.
 *   pool          device, batch b's rows at pool + (b * pool_bstride) *
 *                 ds4a_kv_fp8_row_bytes(D, R), 16-byte aligned
 *   pool_bstride  rows between sequences (>= N_c)
 * The Flash shape only (64 heads x 512, RoPE 64; DS4A_EUNSUPPORTED
 * otherwise).  Everything else is as the bf16 calls.
 */
int ds4a_sparse_attend_fp8(const ds4a_layer_cfg* cfg, int B, int T_q, const int32_t* q_pos,
                           const ds4a_bf16* q, const float* q_norm_g, const uint8_t* pool,
                           int64_t pool_bstride, int N_c, const int32_t* idx, const ds4a_bf16* win,
                           int win_cap, int64_t win_bstride, const float* sink, ds4a_bf16* out,
                           void* ws, size_t ws_bytes, ds4a_stream stream);
int ds4a_hca_attend_fp8(const ds4a_layer_cfg* cfg, int B, int T_q, const int32_t* q_pos,
                        const ds4a_bf16* q, const float* q_norm_g, const uint8_t* pool,
                        int64_t pool_bstride, int N_c, const ds4a_bf16* win, int win_cap,
                        int64_t win_bstride, const float* sink, ds4a_bf16* out, void* ws,
                        size_t ws_bytes, ds4a_stream stream);

/* Synchronise the stream, then read and clear the current device's error
 * word.  Returns DS4A_OK, DS4A_EDEVICE (bad index / position),
 * DS4A_ETIMEOUT (a bounded wait ran out) or DS4A_ECUDA (a CUDA error is
 * pending).  bits_out (host, nullable) receives the DS4A_DEV_* bits. */
int ds4a_check(ds4a_stream stream, uint32_t* bits_out);

/* Static text for a return code. */
const char* ds4a_strerror(int code);

/* Launch trace (for benchmarking): while enabled, every kernel launch is
 * bracketed by CUDA events on its stream.  ds4a_trace_read synchronises the
 * device and copies up to cap records (kernel name, milliseconds) into the
 * host arrays, returning how many launches were recorded; names point to
 * static strings.  Enabling clears the trace.  Not thread safe. */
int ds4a_trace_enable(int on);
int ds4a_trace_read(const char** names, float* ms, int cap);

/* Library version, major * 10000 + minor * 100 + patch. */
int ds4a_version(void);

#ifdef __cplusplus
}
#endif
#endif /* DS4A_H */
