/*
 * idx.h — C ABI of libidx.so, a B200 (sm_100a) implementation of the
 * DeepSeek-V3.2 lightning indexer's hot path:
 *
 *   keys:    rotate (scaled Hadamard-128) → block-FP8 quantise → append to the
 *            per-sequence FP8 key cache;
 *   scores:  S[t,s] = k_scale[s] · Σ_{h<64} w[t,h] · ReLU(q_fp8[t,h] · k_fp8[s]);
 *   select:  the min(k, visible) highest-scoring cached positions per query row.
 *
 * Around that path: the front end before it (the three projections on the
 * tensor cores: idx_project; query RoPE, key LayerNorm + RoPE, fused with the
 * quantiser: idx_front_quant_append), the attention after it
 * (sparse latent attention over the selected positions: idx_sparse_mla_decode),
 * and split-T selection of one sequence over several GPUs (idx_gather_scores,
 * idx_merge_topk).
 *
 * Sources (web pages on DeepSeek-V3.2-Exp's lightning indexer):
 *   "Index scores"          — score equation S^I, fp8_index docstring, Indexer.forward excerpt;
 *   "Index key cache"       — k_cache / k_scale_cache buffers, append before scoring;
 *   "Hadamard rotation"     — rotation equation and orthonormality note;
 *   NKI "DeepSeek-V3.2 Sparse Indexer Kernel API Reference" — caller-owned cache written in
 *                             place, int32 positions, int32 unordered top-k set, finite mask
 *                             bound, front-end parameters (cos / sin tables, LayerNorm gain, bias);
 *   "Join query parts"      — MQA decode excerpt: the attention that consumes the selection.
 *
 * Conventions for every call below.
 *   - All array arguments are DEVICE pointers to row-major, contiguous memory
 *     owned by the caller.  The library never allocates device memory and never
 *     synchronises in these calls; work is enqueued on `stream` (a cudaStream_t;
 *     NULL = the legacy default stream) and runs asynchronously.
 *   - bf16 arrays are passed as uint16_t bit patterns; FP8 arrays hold e4m3fn
 *     codes as uint8_t.
 *   - Index head count H = 64 and head dimension D = 128 are fixed.
 *   - Return value: IDX_OK (0) when the work was enqueued, or a negative IDX_ERR_*
 *     for an argument error detected on the host (nothing is enqueued then).
 *     Errors that depend on device data (positions, lengths) are detected in the
 *     kernels, which then skip the offending sequence and set a bit in a device
 *     error word; idx_status() reports and clears it.
 *   - Query row i (0 ≤ i < n) of sequence b sits at position lengths[b] − n + i
 *     (the call's new rows are the last n cached positions).  Key s is visible to
 *     that row iff s < lengths[b] and, when causal != 0, s ≤ its position.
 *     visible(b,i) = causal ? lengths[b] − n + i + 1 : lengths[b].
 *   - Scale format `fmt`: IDX_FMT_FP32 stores scale = fl32(max(amax,1e-4)/448);
 *     IDX_FMT_UE8M0 rounds that up to a power of two.  Both store float32.
 */
#ifndef IDX_H_
#define IDX_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define IDX_API __attribute__((visibility("default")))
#else
#define IDX_API
#endif

typedef struct CUstream_st* idx_stream_t;

#define IDX_HEADS 64
#define IDX_DIM 128
#define IDX_ROPE_DIM 64    /* leading features the rotary embedding turns */
#define IDX_MAX_LEN 131072 /* largest lengths[b] / max_len a score call accepts */

enum idx_fmt { IDX_FMT_FP32 = 0, IDX_FMT_UE8M0 = 1 };

/* Key-scale storage read by the *_ex score calls: fp32 values, or one e8m0
 * byte per key (OCP MX scale format: value 2^(byte − 127)), as written by
 * idx_quant_append_e8 — 129 instead of 132 cache bytes per key. */
enum idx_scale_storage { IDX_SCALE_F32 = 0, IDX_SCALE_E8M0 = 1 };

/* Score element type written by idx_score_ex. */
enum idx_score_dtype { IDX_SCORE_F32 = 0, IDX_SCORE_BF16 = 1 };

/* The most negative finite bfloat16, −(2 − 2^−7)·2^127: a finite mask value a
 * bf16 consumer reads unchanged ("DeepSeek-V3.2 Sparse Indexer Kernel API
 * Reference" page, Notes: masked slots are clamped to a finite bound because a
 * bf16 max-select turns −inf into NaN).  Exact in fp32. */
#define IDX_MASK_BOUND_BF16 (-3.38953138925153547590470800371487866880e+38f)

enum idx_status_code {
  IDX_OK = 0,
  IDX_ERR_NULL = -1,        /* a required pointer is NULL */
  IDX_ERR_SHAPE = -2,       /* a size is negative, zero where it must not be, or too large */
  IDX_ERR_FMT = -3,         /* fmt is not IDX_FMT_FP32 / IDX_FMT_UE8M0 */
  IDX_ERR_K = -4,           /* k <= 0 */
  IDX_ERR_ALIGN = -5,       /* a pointer is not 16-byte aligned where required */
  IDX_ERR_LAUNCH = -6,      /* the CUDA launch failed (the CUDA error is in idx_last_cuda_error) */
  IDX_ERR_DEVICE = -7,      /* idx_status: a kernel set the device error word */
  IDX_ERR_CUDA = -8,        /* idx_status: the stream itself reported a CUDA error */
  IDX_ERR_UNSUPPORTED = -9, /* no device code for this GPU (not sm_100) */
  IDX_ERR_SCRATCH = -10     /* the scratch is too small: idx_score_topk_noalloc's fixed scratch, idx_project's ws */
};

/* Bits of the device error word (returned by idx_device_error_bits). */
#define IDX_DEV_ERR_TIMEOUT 0x1u  /* a bounded wait inside a kernel gave up */
#define IDX_DEV_ERR_POSITION 0x2u /* idx_quant_append: positions[b] < 0 or positions[b] + n > T_cap */
#define IDX_DEV_ERR_LENGTH 0x4u   /* score/top-k: lengths[b] < n or lengths[b] > max_len */

/*
 * idx_quant — "Hadamard rotation" page (rotation equation) followed by the
 * block-FP8 quantisation of groups of 128 features.
 *   x_bf16  [rows, 128]  bf16 input rows.
 *   x_fp8   [rows, 128]  out: e4m3 codes of fl32(y / scale), y = bf16(H·x/√128).
 *   x_scale [rows]       out: float32 scale per row.
 * rows may be 0 (nothing is enqueued).  x_bf16 and x_fp8 must be 16-byte aligned.
 */
IDX_API int idx_quant(const uint16_t* x_bf16, int64_t rows, uint8_t* x_fp8, float* x_scale, int fmt,
              idx_stream_t stream);

/*
 * idx_quant_queries — queries of `tokens` rows of 64 heads: the same rotation
 * and quantisation per (token, head), and the head weights folded as on the
 * "Index scores" page (1/√64 into the weights, 1/√128 with the query's scale):
 *   w[t,h] = fl32(fl32(fl32(w_raw[t,h]·0.125)·q_scale[t,h])·fl32(128^-1/2)).
 *   q_bf16 [tokens, 64, 128], w_raw [tokens, 64] float32 in;
 *   q_fp8 [tokens, 64, 128] out; w [tokens, 64] float32 out (the folded weights
 *   idx_score / idx_score_topk take).  The query scales are not stored.
 *   q_bf16 and q_fp8 must be 16-byte aligned.
 */
IDX_API int idx_quant_queries(const uint16_t* q_bf16, const float* w_raw, int64_t tokens, uint8_t* q_fp8, float* w,
                      int fmt, idx_stream_t stream);

/*
 * idx_quant_append — "Index key cache" page: rotate and quantise n new keys of
 * each of B sequences and write them in place at slots positions[b] … +n−1.
 *   k_bf16        [B, n, 128] bf16.
 *   positions     [B] int32 first slot per sequence.
 *   k_cache       [B, T_cap, 128] uint8 (e4m3), written in place.
 *   k_scale_cache [B, T_cap] float32, written in place.
 * A sequence with positions[b] < 0 or positions[b] + n > T_cap is skipped and
 * IDX_DEV_ERR_POSITION is raised.  k_bf16 and k_cache must be 16-byte aligned.
 */
IDX_API int idx_quant_append(const uint16_t* k_bf16, const int32_t* positions, int B, int n, uint8_t* k_cache,
                     float* k_scale_cache, int T_cap, int fmt, idx_stream_t stream);

/*
 * idx_quant_append_e8 — idx_quant_append with fmt = IDX_FMT_UE8M0 and each key's
 * power-of-two scale stored as its e8m0 byte (2^(byte − 127); the byte is the
 * fp32 exponent field of the scale) in k_scale_e8 [B, T_cap] uint8 — the "e8m0"
 * of the fp8_index docstring ("Index scores" page).  Read by the *_ex score
 * calls with IDX_SCALE_E8M0.  Arguments, alignment and errors as idx_quant_append.
 */
IDX_API int idx_quant_append_e8(const uint16_t* k_bf16, const int32_t* positions, int B, int n, uint8_t* k_cache,
                                uint8_t* k_scale_e8, int T_cap, idx_stream_t stream);

/*
 * idx_quant_queries_append — idx_quant_queries and idx_quant_append of one
 * indexer call in a single launch (the two are independent row sets of the
 * same rotation + quantisation).  Arguments as in the two calls; either part
 * may be empty (tokens = 0, or B = 0 / n = 0).
 */
IDX_API int idx_quant_queries_append(const uint16_t* q_bf16, const float* w_raw, int64_t tokens, uint8_t* q_fp8,
                                     float* w, const uint16_t* k_bf16, const int32_t* positions, int B, int n,
                                     uint8_t* k_cache, float* k_scale_cache, int T_cap, int fmt,
                                     idx_stream_t stream);

/*
 * idx_front_quant_append — the indexer's front end after its projections, in
 * the order of the Indexer.forward excerpt, fused with idx_quant_queries_append:
 * queries get the rotary embedding; keys get the LayerNorm (k_norm), then the
 * rotary embedding; both are then rotated and quantised, the keys appended and
 * the weights folded as in idx_quant_queries_append.
 *   q_proj [B, n, 64, 128] bf16: the query projection (wq_b of the low-rank
 *          query), 16-byte aligned.
 *   w_raw [B, n, 64] fp32: the weight projection of the hidden state.
 *   k_proj [B, n, 128] bf16: the key projection (wk of the hidden state), 16-byte aligned.
 *   rope_cos, rope_sin [B, n, IDX_ROPE_DIM / 2] fp32: cos θ_i and sin θ_i of
 *          each token's position (the NKI page's cos / sin tables); feature
 *          i and i + 32 (i < 32) are the pair turned by θ_i (not interleaved);
 *          features 64 … 127 are not turned.
 *   ln_gain, ln_bias [128] fp32, ln_eps ≥ 0: the key LayerNorm (biased
 *          variance, eps under the square root).
 *   positions, B, n, q_fp8, w, k_cache, k_scale_cache, T_cap, fmt: as in
 *          idx_quant_queries_append (tokens = B·n).
 * Arithmetic: float64 with one rounding per operation (sums over features in
 * feature order), each step's result rounded to bf16, then the rotation and
 * quantisation of idx_quant.  Errors as idx_quant_queries_append, plus
 * IDX_ERR_SHAPE for a negative, infinite or NaN ln_eps.
 */
IDX_API int idx_front_quant_append(const uint16_t* q_proj, const float* w_raw, const uint16_t* k_proj,
                                   const float* rope_cos, const float* rope_sin, const float* ln_gain,
                                   const float* ln_bias, float ln_eps, const int32_t* positions, int B, int n,
                                   uint8_t* q_fp8, float* w, uint8_t* k_cache, float* k_scale_cache, int T_cap,
                                   int fmt, idx_stream_t stream);

/*
 * idx_project — the three projections that open the Indexer.forward excerpt
 * ("Index scores" page): q = wq_b(qr) viewed as 64 heads of 128 features,
 * k = wk(x), and the head weights weights_proj(x.float()).
 *   x      [tokens, hidden] bf16 (hidden a multiple of 64), the hidden state.
 *   qr     [tokens, q_lora] bf16 (q_lora a multiple of 64), the low-rank query.
 *   wq_b   [64·128, q_lora] bf16, wk [128, hidden] bf16: Linear weights [out, in].
 *   w_proj [64, hidden] fp32.
 *   q_proj [tokens, 64, 128] bf16 out, k_proj [tokens, 128] bf16 out: the fp32
 *          products (tensor cores, fp32 accumulation) rounded to nearest-even bf16;
 *          ready for idx_front_quant_append.
 *   w_raw  [tokens, 64] fp32 out: Σ_k x·w_proj in fp32 on the tensor cores, with
 *          w_proj split into three bf16 parts hi + mid + lo (equal to it within
 *          2^-24 relative), each part's products summed in fp32, the three sums
 *          added (lo + mid) + hi.
 *   ws / ws_bytes: scratch of at least idx_project_workspace_size(tokens, hidden,
 *          q_lora) bytes (16-byte aligned, required): the three bf16 parts of
 *          w_proj (written every call) and the fp32 partial sums of products split
 *          over K when few tokens cannot fill the GPU (added in a fixed order).
 * All pointers except w_proj must be 16-byte aligned.  Errors: IDX_ERR_SHAPE,
 * IDX_ERR_NULL (ws included), IDX_ERR_ALIGN, IDX_ERR_SCRATCH (ws_bytes too small).
 */
IDX_API size_t idx_project_workspace_size(int64_t tokens, int hidden, int q_lora);
IDX_API int idx_project(const uint16_t* x, const uint16_t* qr, int64_t tokens, int hidden, int q_lora,
                        const uint16_t* wq_b, const uint16_t* wk, const float* w_proj, uint16_t* q_proj,
                        uint16_t* k_proj, float* w_raw, void* ws, size_t ws_bytes, idx_stream_t stream);

/*
 * idx_score — "Index scores" page: score equation and fp8_index docstring
 * (FP8 q·k → fp32 logits, ReLU, × head weight, sum over heads, × key scale),
 * with the causal mask of the Indexer.forward excerpt.
 *   q_fp8  [B, n, 64, 128] e4m3 codes; w [B, n, 64] folded weights (idx_quant_queries).
 *   k_cache [B, T_cap, 128], k_scale_cache [B, T_cap]; lengths [B] int32.
 *   max_len: host-side upper bound on lengths[b] (n ≤ max_len ≤ min(T_cap, IDX_MAX_LEN));
 *            it sizes the launch.
 *   scores [B, n, ld] float32 out: S for visible keys, −inf for every other column < ld.
 *          ld ≥ 1; columns ≥ ld are not computed.
 * q_fp8 and k_cache must be 16-byte aligned (they are read by TMA).
 */
IDX_API int idx_score(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache, const float* k_scale_cache,
              const int32_t* lengths, int B, int n, int T_cap, int max_len, int causal, float* scores, int64_t ld,
              idx_stream_t stream);

/*
 * idx_score_ex — idx_score with the storage and output options of the NKI
 * indexer page (its Notes on the finite mask bound) and of the fp8_index
 * docstring (the key scale "e8m0 here"):
 *   k_scale      [B, T_cap] key scales: float32 (scale_fmt = IDX_SCALE_F32) or
 *                uint8 e8m0 bytes (IDX_SCALE_E8M0; T_cap a multiple of 16),
 *                16-byte aligned.
 *   scores       [B, n, ld] of score_dtype: IDX_SCORE_F32, or IDX_SCORE_BF16
 *                (each fp32 score rounded to nearest even).
 *   mask_value   written to every masked column: −inf as idx_score, or a
 *                finite bound such as IDX_MASK_BOUND_BF16 (NaN is rejected).
 * An e8m0 scale is the same power of two as the fp32 ue8m0 scale, so the
 * scores equal idx_score's on a cache filled with IDX_FMT_UE8M0.
 * Returns IDX_ERR_FMT for an unknown scale_fmt or score_dtype.
 */
IDX_API int idx_score_ex(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache, const void* k_scale,
                         int scale_fmt, const int32_t* lengths, int B, int n, int T_cap, int max_len, int causal,
                         void* scores, int64_t ld, int score_dtype, float mask_value, idx_stream_t stream);

/*
 * idx_score_visible — the scores of idx_score for the visible keys only, as
 * the score + top-k path computes them into its workspace: one persistent CTA
 * per SM, each streaming an equal share of all (row block, 128-key tile)
 * pairs of the call.
 *   Arguments as in idx_score, with ld ≥ max_len and w 16-byte aligned.
 *   scores [B, n, ld]: S for visible keys, −inf from each row's visible count
 *          up to the end of its last 128-key tile; columns past that tile are
 *          left unwritten (their contents are unspecified).
 * Calls with more than 4096 blocks of query rows are served by idx_score.
 */
IDX_API int idx_score_visible(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache,
                              const float* k_scale_cache, const int32_t* lengths, int B, int n, int T_cap,
                              int max_len, int causal, float* scores, int64_t ld, idx_stream_t stream);

/*
 * idx_topk — Indexer.forward excerpt (top min(index_topk, ·) per row) and the
 * NKI page's output convention (int32, unordered set), on scores already in memory.
 *   scores [B, n, ld] float32 (finite for visible keys); lengths [B]; causal as above.
 *   indices [B, n, k] int32 out: the k_t = min(k, visible(b,i)) positions with the
 *   highest scores, in unspecified order, in columns 0 … k_t−1; columns k_t … k−1
 *   hold −1.  Ties at the k_t-th score are broken arbitrarily.
 *   max_len as in idx_score (and ≤ ld).  ws / ws_bytes: not used, pass NULL / 0.
 */
IDX_API int idx_topk(const float* scores, const int32_t* lengths, int B, int n, int64_t ld, int max_len, int causal, int k,
             int32_t* indices, void* ws, size_t ws_bytes, idx_stream_t stream);

/*
 * Split-T selection: one sequence's keys split over G GPUs (or G slices on one
 * GPU).  The Indexer.forward excerpt selects the row's top min(index_topk, ·)
 * and then checks with a broadcast that every rank agrees; here each rank
 * selects the k best of its own slice (idx_topk on its scores), turns them into
 * (score, global position) pairs with idx_gather_scores, the ranks exchange the
 * pairs (one all-gather of k·8 bytes per row), and idx_merge_topk selects the
 * row's k best among the G·k candidates.  Exact: a key of the row's top k is in
 * its own slice's top k.
 */
typedef struct {
  float score;   /* the key's score */
  int32_t pos;   /* its position in the whole sequence; −1 marks an empty slot */
} idx_cand_t;    /* 8 bytes */

/*
 * idx_gather_scores
 *   scores [rows, ld] float32 (device): this slice's scores, row r at r·ld.
 *   idx [rows, k] int32 (device): slice-local positions from idx_topk, −1 = empty.
 *   counts [rows] int32 (device) or NULL: keys of row r held in this slice;
 *          positions ≥ counts[r] count as empty.  (A slice holding none of a
 *          row's keys is scored and selected with a length of 1 — the scorer
 *          requires lengths ≥ n — and its one position is dropped here.)
 *   offset: the slice's first global position (added to every valid position).
 *   cand [rows, k] idx_cand_t (device, caller-owned, 8-byte aligned) out:
 *   (scores[r·ld + idx], idx + offset); empty slots give (−inf, −1).
 *   Errors: IDX_ERR_SHAPE (rows, k < 0 or ld ≤ 0), IDX_ERR_NULL; nothing to do
 *   when rows·k = 0.
 */
IDX_API int idx_gather_scores(const float* scores, int64_t ld, const int32_t* idx, int64_t rows, int k,
                              const int32_t* counts, int32_t offset, idx_cand_t* cand, idx_stream_t stream);

/*
 * idx_merge_topk
 *   cand [G, rows, kin] idx_cand_t (device): rank g's candidates of row r at
 *   (g·rows + r)·kin — the layout of an all-gather of the per-rank [rows, kin]
 *   outputs of idx_gather_scores.  Empty slots (pos −1) are skipped; the others
 *   need finite scores and distinct positions.
 *   out [rows, k] int32 (device, caller-owned): the positions of the
 *   k_t = min(k, valid candidates) highest scores in columns 0 … k_t−1 (a set,
 *   ties at the k_t-th score broken arbitrarily), −1 after.
 *   Limits: G·kin ≤ 16384.  Errors: IDX_ERR_SHAPE, IDX_ERR_K (k ≤ 0), IDX_ERR_NULL.
 *   One CTA per row.
 */
IDX_API int idx_merge_topk(const idx_cand_t* cand, int G, int64_t rows, int kin, int k, int32_t* out,
                           idx_stream_t stream);

/*
 * idx_sparse_mla_decode — the attention that consumes the selection ("Join
 * query parts" page, MQA decode excerpt): for one decode token per sequence,
 * each head scores the selected cache rows, takes the softmax over them and
 * returns the latent output.
 *   q [B, H, 576] bf16: per head the absorbed content query (512) followed by
 *          the rotary query (64); H a multiple of 16.
 *   kv [B, T_cap, 576] bf16 (16-byte aligned): per position the latent (512)
 *          followed by the rotary key (64).
 *   indices [B, k] int32: the selected positions (the indexer's output for the
 *          token); entries < 0 or ≥ T_cap select nothing.
 *   softmax_scale: finite; s = softmax_scale · q·kv.
 *   out [B, H, 512] fp32 (caller-owned): Σ_t softmax(s)_t · kv[t, 0:512]
 *          over the selected t; 0 for a row that selects nothing.
 * Arithmetic: when H is a multiple of 128 (and q 16-byte aligned), on the
 * tensor cores — bf16 products accumulated in fp32, the softmax weights
 * rounded to bf16 for the weighted sum (their sum taken as rounded), chunks of
 * 64 positions; otherwise fp32 on the CUDA cores (online softmax over chunks
 * of 32 positions).  Errors: IDX_ERR_SHAPE (B < 0, H not a positive multiple of 16,
 * T_cap ≤ 0, a non-finite scale), IDX_ERR_K (k ≤ 0), IDX_ERR_NULL, IDX_ERR_ALIGN.
 */
IDX_API int idx_sparse_mla_decode(const uint16_t* q, const uint16_t* kv, const int32_t* indices, int B, int H,
                                  int64_t T_cap, int k, float softmax_scale, float* out, idx_stream_t stream);

/*
 * idx_score_topk — scores and top-k in one call, arguments as in idx_score /
 * idx_topk.  Decode-shaped calls (n ≤ 2) run one kernel in which a row's scores
 * never leave on-chip memory.  Prefill-shaped calls (n > 2) given a workspace of
 * at least idx_workspace_size(B, n, max_len, k) bytes (16-byte aligned) write
 * the scores there and select with the top-k kernel (faster: selections of
 * different rows overlap); without one they use the single-kernel path.
 */
IDX_API int idx_score_topk(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache, const float* k_scale_cache,
                   const int32_t* lengths, int B, int n, int T_cap, int max_len, int causal, int k,
                   int32_t* indices, void* ws, size_t ws_bytes, idx_stream_t stream);

/*
 * idx_score_topk_ex — idx_score_topk with the key scales stored as fp32
 * (scale_fmt = IDX_SCALE_F32) or as e8m0 bytes (IDX_SCALE_E8M0, T_cap a
 * multiple of 16).  The selected set equals idx_score_topk's on a cache filled
 * with IDX_FMT_UE8M0.
 */
IDX_API int idx_score_topk_ex(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache, const void* k_scale,
                              int scale_fmt, const int32_t* lengths, int B, int n, int T_cap, int max_len,
                              int causal, int k, int32_t* indices, void* ws, size_t ws_bytes, idx_stream_t stream);

/*
 * idx_score_topk_noalloc — idx_score_topk for callers that cannot allocate
 * device memory when they call (for example while their stream is being
 * captured into a CUDA graph, or inside a plugin enqueue step that must not
 * allocate).  The pages have no counterpart: this is a deployment variant.
 * Prefill-shaped calls keep their score workspace in a buffer the library
 * owns: a file-scope device array of 64 MiB (B·n·max_len ≤ 16 Mi scores),
 * held on every GPU that loads the library until the process exits.  Larger
 * calls return IDX_ERR_SCRATCH before anything is enqueued — for example two
 * sequences of 2048 new rows over 16 384 keys (256 MiB of scores): call
 * idx_score_topk with a workspace for those.  Decode-shaped calls need no scratch.
 *   - The first call on a device, of any shape, looks up the buffer's device
 *     address (no allocation); make that first call before any stream capture.
 *   - Every call reuses the same buffer and rewrites all of the part it uses,
 *     so nothing needs clearing, but calls that overlap on the GPU (other
 *     streams, other threads) race on it: serialise them.
 *   - It calls no cudaMalloc / cudaFree; arguments otherwise as idx_score_topk.
 */
IDX_API int idx_score_topk_noalloc(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache,
                                   const float* k_scale_cache, const int32_t* lengths, int B, int n, int T_cap,
                                   int max_len, int causal, int k, int32_t* indices, idx_stream_t stream);

/* Workspace bytes idx_score_topk uses for these sizes: 0 for decode-shaped
 * calls (n ≤ 2), B·n·max_len·4 (fp32 scores) for prefill-shaped ones. */
IDX_API size_t idx_workspace_size(int B, int n, int max_len, int k);

/*
 * idx_status — synchronises `stream`, then reads and clears the device error
 * word.  Returns IDX_OK, IDX_ERR_DEVICE (bits available from
 * idx_device_error_bits) or IDX_ERR_CUDA.
 */
IDX_API int idx_status(idx_stream_t stream);
IDX_API unsigned int idx_device_error_bits(void); /* bits seen by the last idx_status call */
IDX_API const char* idx_error_string(int code);
IDX_API int idx_last_cuda_error(void); /* cudaError_t of the last failed launch, 0 if none */

/*
 * idx_e4m3_encode — the float32 → e4m3fn conversion the quantiser uses (round to
 * nearest even, saturate to ±448, sign of zero kept), exposed so that it can be
 * checked value by value.  x [count] float32 in, out [count] uint8 codes.
 */
IDX_API int idx_e4m3_encode(const float* x, int64_t count, uint8_t* out, idx_stream_t stream);

/*
 * Fault-injection control for tests: when `flags` has bit 0 set, the next score
 * launches make one bounded wait in each CTA wait for a barrier that nothing
 * signals, with the wait budget set to `budget_ns`; the kernels then report
 * IDX_DEV_ERR_TIMEOUT and return.  idx_debug_set(0, 0) restores normal
 * operation (2 s wait budget).
 */
IDX_API void idx_debug_set(unsigned int flags, unsigned long long budget_ns);

/*
 * Profiling aid: when the debug flags have bit 1 set, score launches record per
 * CTA (first 8192 CTAs) 16 words: [0] entry, [1] set-up done, [2] first
 * accumulator ready, [3] key stream done, [4] selection done, [5] exit
 * (globaltimer ns), [7] SM id, [8..14] steps inside the first row's
 * selection, [15] its candidate count.  idx_debug_trace copies them to
 * host_out (max_ctas × 16 words) after synchronising the device.
 */
IDX_API int idx_debug_trace(unsigned long long* host_out, int max_ctas);

#ifdef __cplusplus
}
#endif

#endif /* IDX_H_ */
