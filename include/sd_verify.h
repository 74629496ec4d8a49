/*
 * sd_verify.h -- C ABI of the B200 (sm_100a) speculative-decoding verify step.
 *
 * The verify step of draft-then-verify decoding: a drafter proposes k tokens, the target
 * scores the k drafts plus one more position (k+1 positions) in one forward pass, accepts a
 * prefix of the drafts and emits one token of its own ("Gemma 4 MTP: drafter drafts, target
 * verifies", sections "basic structure of speculative decoding" and "drafter internal
 * architecture"; Gemma 4 MTP serving guide, section 4 "execution flow").  The calls below
 * are the data-parallel parts of that step:
 *
 *   sd_verify_attn   k+1 causal queries per sequence over a paged bf16 KV cache (GQA,
 *                    sliding or global layer), appending the k+1 new K/V rows
 *   sd_draft_xattn   the drafter's read-only cross-attention into the same cache
 *   sd_lm_head       logits over the vocabulary, dense or two-stage clustered
 *   sd_accept        lossless acceptance, correction / bonus draw (or greedy at T = 0)
 *   sd_commit        committed length, committed slots, rollback, next hidden row
 *   sd_linear        one dense projection of a few token rows with a normalising / gathering
 *                    prologue and a store, residual-add or gated-GELU epilogue (the drafter's
 *                    and the target's layers around their attention)
 *
 * Conventions shared by every call
 *   - Every data pointer is a caller-owned DEVICE buffer, densely packed in the layout
 *     stated for it (row-major, last index fastest).  Descriptors are HOST structs read
 *     during the call only.  The library allocates no device memory; scratch space is the
 *     caller's workspace (ws, ws_bytes), sized by the matching *_workspace_size call.  A
 *     workspace needs no initialisation and carries nothing from one call to the next, so
 *     calls that share one must not overlap on the GPU.
 *   - Calls are stream-ordered and return after enqueueing; results are valid once the
 *     stream has reached them.  The library keeps no state between calls except a
 *     per-device status word (sd_device_status_read).
 *   - Host-side validation returns a status synchronously and launches nothing.  A failed
 *     launch returns SD_ERR_CUDA.  Out-of-range indices found on the device (a block id
 *     outside [0, num_blocks), a token id outside [0, vocab)) are never dereferenced: the
 *     kernel skips the access and records SD_ERR_DEVICE in the status word.  Every wait
 *     inside a kernel is bounded; a wait that runs out records SD_ERR_TIMEOUT and the
 *     kernel returns.
 *   - bf16 is IEEE-754 binary32 truncated to its upper 16 bits (torch.bfloat16).
 */
#ifndef SD_VERIFY_H
#define SD_VERIFY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st *sd_stream;

typedef enum {
  SD_OK = 0,
  SD_ERR_INVALID_ARG = 1, /* null pointer, inconsistent or out-of-range descriptor field */
  SD_ERR_UNSUPPORTED = 2, /* valid request outside what the kernels implement */
  SD_ERR_WORKSPACE = 3,   /* ws_bytes smaller than the *_workspace_size result */
  SD_ERR_CUDA = 4,        /* a CUDA runtime or driver call failed */
  SD_ERR_TIMEOUT = 5,     /* (status word) a bounded device wait ran out */
  SD_ERR_DEVICE = 6       /* (status word) an out-of-range index met on the device */
} sd_status;

typedef enum { SD_F32 = 0, SD_BF16 = 1 } sd_dtype;

/* ---------------------------------------------------------------------------------------
 * Attention over a paged KV cache.
 *
 * Cache layout: k_cache, v_cache [num_blocks, h_kv, block_size, head_dim]; logical position
 * p of sequence b lives in physical block block_table[b * max_blocks_per_seq + p / block_size]
 * at row p % block_size.  Query head h reads kv head h / (h_q / h_kv).
 */
typedef struct {
  int batch;              /* B >= 1 */
  int n_q;                /* query positions per sequence: k+1 for sd_verify_attn, 1 for
                             sd_draft_xattn */
  int h_q, h_kv;          /* h_q % h_kv == 0; (h_q / h_kv) * n_q <= 64 */
  int head_dim;           /* bf16: 64, 128, 256 or 512; f32: a multiple of 32, <= 512 */
  int block_size;         /* bf16: a multiple of 16; f32: >= 1 */
  int max_blocks_per_seq; /* columns of block_table */
  int num_blocks;         /* physical blocks in the cache */
  int window;             /* <= 0: global layer; > 0: a query at position t reads the keys
                             p in [t - window + 1, t] (window keys including its own) */
  float scale;            /* logit scale, e.g. 1 / sqrt(head_dim) */
  sd_dtype dtype;         /* element type of q, k_new, v_new, caches and out */
  int q_offset;           /* sd_draft_xattn with q_pos == NULL: the query of sequence b sits
                             at ctx_len[b] + q_offset (step j of a drafter chain: j) */
} sd_attn_desc;

/*
 * Verify attention ("Gemma 4 MTP: drafter drafts, target verifies", section "drafter internal
 * architecture": the target verifies k+1 positions in one forward pass).
 *
 * With L_b = ctx_len[b] committed tokens, the n_q new rows k_new[b, j], v_new[b, j] are first
 * written to positions L_b + j (j < n_q) of the cache; then query j of sequence b, at position
 * t = L_b + j, attends causally to keys p in [lo, t] (lo = max(0, t - window + 1) for a
 * sliding layer, 0 for a global one):
 *     out[b, j, h] = softmax_p(scale * q[b, j, h] . K_p) . V_p      (float32 accumulation)
 *
 *   q      [B, n_q, h_q, head_dim]       k_new, v_new [B, n_q, h_kv, head_dim]
 *   out    [B, n_q, h_q, head_dim]       block_table  int32 [B, max_blocks_per_seq]
 *   ctx_len int32 [B], not modified (sd_commit advances it)
 * The blocks holding positions up to L_b + n_q - 1 must be allocated in block_table.
 * out must not alias q, the caches or the workspace.
 */
size_t sd_verify_attn_workspace_size(const sd_attn_desc *desc);
sd_status sd_verify_attn(const sd_attn_desc *desc, const void *q, const void *k_new,
                         const void *v_new, void *k_cache, void *v_cache,
                         const int32_t *block_table, const int32_t *ctx_len, void *out,
                         void *ws, size_t ws_bytes, sd_stream stream);

/*
 * Drafter cross-attention into the target's cache ("Gemma 4 MTP: drafter drafts, target
 * verifies", section "drafter internal architecture": each drafter layer attends directly to
 * the target's KV cache; Google blog as summarised by GeekNews, section "MTP drafter internal
 * optimisations": the drafter shares the target's KV cache).  Read-only.  desc->n_q must be 1.
 * The query of sequence b sits at position q_pos[b] and attends to the committed keys
 * p in [lo, min(q_pos[b], L_b - 1)], lo relative to q_pos[b] as above; an empty range gives a
 * zero output row.
 *   q, out [B, 1, h_q, head_dim]      q_pos int32 [B] (>= 0), or NULL for
 *   q_pos[b] = ctx_len[b] + desc->q_offset
 */
size_t sd_draft_xattn_workspace_size(const sd_attn_desc *desc);
sd_status sd_draft_xattn(const sd_attn_desc *desc, const void *q, const void *k_cache,
                         const void *v_cache, const int32_t *block_table,
                         const int32_t *ctx_len, const int32_t *q_pos, void *out, void *ws,
                         size_t ws_bytes, sd_stream stream);

/* ---------------------------------------------------------------------------------------
 * LM head (Gemma 4 MTP serving guide, section 1, and the GeekNews summary, section "MTP
 * drafter internal optimisations": a 256k-token vocabulary whose final logit projection is a
 * large cost; the edge drafters group the vocabulary into clusters to cut it).
 */
typedef struct {
  int m;            /* rows of h (B * n_q for the target head) */
  int d;            /* hidden width; bf16: a multiple of 64 */
  int vocab;        /* V */
  int ld_logits;    /* floats between consecutive logit rows; 0 means vocab */
  int n_clusters;   /* clustered mode: C clusters of cluster_size tokens, C * cluster_size
                       == vocab */
  int cluster_size;
  int top_c;        /* 0: dense mode; else clusters kept per row (1 <= top_c <= n_clusters,
                       top_c <= 64) */
  sd_dtype dtype;   /* element type of h, w and centroids (bf16; f32 in dense mode too) */
} sd_head_desc;

/*
 * Dense (top_c == 0):
 *     logits[i * ld + v] = sum_c h[i, c] * w[v, c]        float32 output and accumulation
 *   h [m, d], w [vocab, d]; centroids, cluster_tokens and sel_clusters are unused (NULL ok).
 * Clustered (top_c > 0), a drafter-side approximation (it must not replace the target's dense
 * head: the acceptance rule needs the target's true p):
 *   score[i, c] = h[i] . centroids[c]; the top_c clusters of row i (higher score first, equal
 *   scores ordered by lower cluster id) are written to sel_clusters[i, 0..top_c) in ascending
 *   id order; logits[i * ld + cluster_tokens[c, j]] = h[i] . w[c, j] for kept clusters c and
 *   -inf for every other token.
 *   h [m, d], centroids [n_clusters, d], w cluster-major [n_clusters, cluster_size, d],
 *   cluster_tokens int32 [n_clusters, cluster_size] (a permutation of 0..vocab-1),
 *   sel_clusters int32 [m, top_c].
 */
size_t sd_lm_head_workspace_size(const sd_head_desc *desc);
sd_status sd_lm_head(const sd_head_desc *desc, const void *h, const void *w,
                     const void *centroids, const int32_t *cluster_tokens, float *logits,
                     int32_t *sel_clusters, void *ws, size_t ws_bytes, sd_stream stream);

/* ---------------------------------------------------------------------------------------
 * Acceptance.  The pages cite Leviathan et al., "Fast Inference from Transformers via
 * Speculative Decoding", for the rule (Google blog translation, section "how speculative
 * decoding works") and state its property: the output is distributed exactly as decoding
 * with the target alone ("Gemma 4 MTP: drafter drafts, target verifies", section "basic
 * structure of speculative decoding").
 *
 * For sequence b: p_i = softmax(z_{b,i-1} / T), q_i = softmax(y_{b,i-1} / T), i = 1..k.
 * Draft d_i is accepted iff u_i < p_i(d_i) / q_i(d_i); the first rejection at i stops the
 * scan and emits x ~ norm(max(0, p_i - q_i)) (p_i if that is all zero); if all k drafts are
 * accepted, the bonus token x ~ p_{k+1}.  T == 0 is greedy: accept iff d_i == argmax z_{b,i-1},
 * emit argmax z_{b,a} (lowest id on ties).
 * Random numbers: Philox4x32-10 (Salmon et al., SC'11) with key (seed_lo, seed_hi) and
 * counter (c0, r, step_lo, purpose), r = b * (k+1) + i the logit row:
 *   u of row r        = (word0(c0 = 0, purpose 0) >> 8) * 2^-24
 *   V of token v, row r: the 64-bit word w = words (2(v&1)+1, 2(v&1)) of c0 = v >> 1 with the
 *   draw's purpose, V = top 24 significant bits of w scaled into (0, 1); draws are
 *   exponential races: x = argmax_v ln w_v - ln(-ln(1 - V_v)).
 * k == 0 makes the call a plain draw of one token from softmax(z_b / T) (the drafter's own
 * sampling, with purpose 2).  (seed, step, purpose) triples must not repeat across calls.
 */
typedef struct {
  int batch;
  int k;               /* drafts per sequence, 0..15 */
  int vocab;
  float temperature;   /* 0: greedy; > 0: sampling temperature */
  uint64_t seed;
  uint64_t step;       /* low 32 bits enter the counter */
  int purpose;         /* Philox purpose of the draw: 1 target, 2 drafter (>= 1) */
  int ld_target;       /* floats between target rows r = b*(k+1)+i; 0 means vocab */
  int ld_draft;        /* floats between draft rows b*k+i; 0 means vocab */
  int ld_out;          /* int32 between sequences of out_tokens; 0 means k+1 */
  const uint64_t *step_ptr; /* nullable DEVICE word: when set, the step entering the counter
                               is *step_ptr + step, read when the kernels run (a decode loop
                               replayed from a CUDA graph advances it with sd_commit) */
} sd_accept_desc;

/*
 *   target_logits float32 rows r = b*(k+1)+i, i <= k;  draft_logits float32 rows b*k+i, i < k
 *   (unused when k == 0 or T == 0; NULL ok); draft_tokens int32 [B, k] (NULL ok if k == 0).
 *   n_accepted int32 [B]; out_tokens int32 rows of length k+1: d_1..d_a, x, then -1.
 *   margin_flags int32 [B] (nullable): 1 where a decision of the sequence may have come out
 *   differently in exact arithmetic: an acceptance test with |u - p/q| < 1e-4; a greedy
 *   argmax whose two largest logits differ by less than 1e-4 * max(1, |largest|); a draw whose
 *   winner's lowest possible key is not 1e-4 above every other token's highest possible key,
 *   with each probability taken to within 1e-5 * (p + q) and each ln E and logit / T to within
 *   1e-5 (1e-5 * (1 + |logit / T|) for a draw from p); a draw from p because every residual
 *   weight came out 0.  Sequences not flagged are the exact rule's outcome.
 */
size_t sd_accept_workspace_size(const sd_accept_desc *desc);
sd_status sd_accept(const sd_accept_desc *desc, const float *target_logits,
                    const float *draft_logits, const int32_t *draft_tokens,
                    int32_t *n_accepted, int32_t *out_tokens, int32_t *margin_flags,
                    void *ws, size_t ws_bytes, sd_stream stream);

/*
 * sd_accept_noalloc -- the same computation as sd_accept, for callers that cannot allocate
 * device memory (for example code that must not call cudaMalloc inside a latency-critical
 * serving loop, or a host framework that only lends out its own input and output buffers).
 * There is no counterpart on the pages; it exists only for such callers.
 *
 * The caller still passes every input and output; the scratch space is a fixed array of
 * SD_ACCEPT_NOALLOC_MAX_SCRATCH bytes compiled into the library, which every GPU that loads the
 * library holds until the process exits.  A request whose sd_accept_workspace_size exceeds that
 * limit is rejected with SD_ERR_WORKSPACE before anything is launched (at V = 262144 the limit
 * covers up to 282 sequences at k = 6, 389 at k = 2).  The first call on a device, and the
 * first after the device's context changes (e.g. after a device reset), looks up the array's
 * device address (cudaGetSymbolAddress), so make that first call before any stream capture.
 * All calls share the one array: calls that may overlap on the GPU (other streams, other host
 * threads) race and must be ordered by the caller.  Nothing in the array needs clearing by the
 * caller: the state that must start at zero is reset by every call.  Allocates nothing.
 */
#define SD_ACCEPT_NOALLOC_MAX_SCRATCH (4u << 20)
sd_status sd_accept_noalloc(const sd_accept_desc *desc, const float *target_logits,
                            const float *draft_logits, const int32_t *draft_tokens,
                            int32_t *n_accepted, int32_t *out_tokens, int32_t *margin_flags,
                            sd_stream stream);

/* ---------------------------------------------------------------------------------------
 * Commit ("Gemma 4 MTP: drafter drafts, target verifies", section "basic structure of
 * speculative decoding": only the prefix up to the rejected position is kept; Gemma 4 MTP
 * serving guide, section 4: drafts after the first rejection are discarded).
 *
 * With a = n_accepted[b] (0 <= a <= k) and L = ctx_len[b] on entry:
 *   ctx_len[b]                 <- L + a + 1
 *   committed_slots[b, j]       = block_table[b, p / bs] * bs + p % bs for p = L + j, j <= a,
 *                                 -1 for a < j <= k                      (int32 [B, k+1])
 *   next_hidden[b, :]           = hidden[b, a, :]   (hidden [B, k+1, d] -> next_hidden [B, d];
 *                                 both may be NULL to skip)
 *   poison (n_poison > 0): the rows of the rolled-back positions L+a+1 .. L+k are set to NaN
 *   in every listed cache (debugging aid; the next verify step overwrites them).
 *   step_ptr (nullable): *step_ptr += 1 once the commit is done.
 */
typedef struct {
  void *cache;          /* [num_blocks, h_kv, block_size, head_dim] sharing block_table */
  int h_kv;
  int head_dim;
  sd_dtype dtype;
} sd_poison_cache;

typedef struct {
  int batch;
  int k;
  int block_size;
  int max_blocks_per_seq;
  int num_blocks;       /* for the bounds check of block ids */
  int d;                /* width of a hidden row (0 if hidden is NULL) */
  sd_dtype hidden_dtype;
  int n_poison;         /* entries in poison (0: no poisoning) */
  const sd_poison_cache *poison;  /* HOST array of n_poison entries */
  uint64_t *step_ptr;   /* nullable DEVICE word: incremented by one after the commit */
} sd_commit_desc;

sd_status sd_commit(const sd_commit_desc *desc, const int32_t *block_table, int32_t *ctx_len,
                    const int32_t *n_accepted, int32_t *committed_slots, const void *hidden,
                    void *next_hidden, sd_stream stream);

/* ---------------------------------------------------------------------------------------
 * Drafter dense layers ("Gemma 4 MTP: drafter drafts, target verifies", section "drafter
 * internal architecture": the drafter has a token embedder of its own and a block of 4
 * transformer layers, and its forward pass takes the target's last-layer activation together
 * with the drafter embedding of the last token; Gemma 4 MTP serving guide, section 4: the
 * drafter predicts its candidates as a chain).  One call is one projection of m token rows
 * with an optional prologue and a fused epilogue.  A drafter layer is four calls around
 * sd_draft_xattn: W_q (normalised input), W_o (added to the residual stream), the gated MLP's
 * gate and up rows (normalised input, gated epilogue), W_d (added to the residual stream).
 *
 *   input row r, k columns:
 *     x'[r, c] = x[r, c]                        c <  k - k_gather
 *     x'[r, c] = table[t_r, c - (k - k_gather)] c >= k - k_gather (an embedding row)
 *     t_r = tokens[r * ld_tokens + (token_sel ? token_sel[r] : 0)]
 *   prologue (norm_gain != NULL):
 *     x'[r, c] <- x'[r, c] / sqrt(mean_c x'[r, c]^2 + norm_eps) * norm_gain[c]
 *   y[r, i] = sum_c bf16(x'[r, c]) * W[i, c]    (float32 accumulation in a fixed order: the
 *                                                result does not depend on the launch)
 *   epilogue:
 *     SD_EPI_STORE  out[r, i] = y[r, i]                           out_dtype f32 or bf16
 *     SD_EPI_ADD    out[r, i] += y[r, i]                          out_dtype f32 (a residual
 *                                                                 stream)
 *     SD_EPI_GEGLU  out[r, f] = gelu(y[r, gate(f)]) * y[r, up(f)] out_dtype bf16, n / 2
 *                   columns; gelu(z) = z/2 (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))); W holds
 *                   gate and up rows in blocks of 16: rows 16t .. 16t+7 are the gate rows of
 *                   features 8t .. 8t+7, rows 16t+8 .. 16t+15 their up rows
 *   norm_out (nullable, needs norm_gain): bf16 [m, ld_norm_out], the normalised rows
 *                   bf16(x') (the drafter's output row, the input of its LM head)
 *
 *   x      [m, ld_x] of x_dtype (f32 or bf16); its first k - k_gather columns are read
 *   W      bf16 [n, k] row-major
 *   table  bf16 [table_rows, ld_table]; k_gather columns of row t_r are read
 *   tokens, token_sel   int32; token_sel[r] in [0, max(ld_tokens, 1))
 *   out    [m, ld_out] of out_dtype
 * Limits: 0 <= m <= 64 (m = 0 launches nothing), n a multiple of 16, k a multiple of 32,
 * k_gather a multiple of 8 (0: no gather), ld_x and ld_table multiples of 4 elements, x, W and
 * table 16-byte aligned; out must not overlap x, table, W, norm_out or the workspace.  A token id
 * outside [0, table_rows) or a token_sel outside its range is not dereferenced: the row reads
 * zeros and SD_ERR_DEVICE is recorded.
 * Workspace (desc->ws, desc->ws_bytes >= sd_linear_workspace_size(desc), 16-byte aligned, no
 * initialisation needed): the staged bf16 input rows x', and for a K dimension split over several
 * CTAs their partial sums and per-tile tickets.  The size depends on m, n, k and the current
 * device's SM count.  The partial sums are added in a fixed order, so the result does not
 * depend on the launch or the timing.
 */
typedef enum { SD_EPI_STORE = 0, SD_EPI_ADD = 1, SD_EPI_GEGLU = 2 } sd_epilogue;

typedef struct {
  int m;                  /* token rows */
  int n;                  /* rows of W (output features; 2x the output columns for GEGLU) */
  int k;                  /* columns of W: input width including the gathered columns */
  sd_dtype x_dtype;       /* element type of x */
  int64_t ld_x;           /* row stride of x (elements) */
  int k_gather;           /* trailing input columns taken from table (0: none) */
  int64_t ld_table;       /* row stride of table (elements) */
  int64_t table_rows;     /* rows of table (token ids are checked against it) */
  int64_t ld_tokens;      /* stride of tokens between rows */
  const float *norm_gain; /* DEVICE f32 [k], or NULL for no normalisation */
  float norm_eps;         /* e.g. 1e-6 */
  sd_epilogue epilogue;
  sd_dtype out_dtype;
  int64_t ld_out;         /* row stride of out (elements) */
  void *norm_out;         /* nullable DEVICE bf16 [m, ld_norm_out] */
  int64_t ld_norm_out;
  void *ws;               /* DEVICE workspace */
  size_t ws_bytes;
} sd_linear_desc;

size_t sd_linear_workspace_size(const sd_linear_desc *desc);
sd_status sd_linear(const sd_linear_desc *desc, const void *x, const void *W, void *out,
                    const void *table, const int32_t *tokens, const int32_t *token_sel,
                    sd_stream stream);

/* ---------------------------------------------------------------------------------------
 * Status.
 */
const char *sd_status_string(sd_status s);
/* Copies the current device's status word (0 = no device-side error so far) to *out.
 * Synchronises the stream. */
sd_status sd_device_status_read(int *out, sd_stream stream);
/* Resets the current device's status word to 0 (stream-ordered). */
sd_status sd_device_status_clear(sd_stream stream);
/* Self-test of the bounded device wait that every kernel's barrier waits use: one thread waits
 * on a barrier that nothing completes, gives up after the wait limit (2 s) and records
 * SD_ERR_TIMEOUT in the status word; the context stays usable.  Stream-ordered; the launch
 * status is returned.  (No counterpart in the pages: it checks this library's failure path.) */
sd_status sd_selftest_bounded_wait(sd_stream stream);
/* Library version: major * 10000 + minor * 100 + patch. */
int sd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SD_VERIFY_H */
