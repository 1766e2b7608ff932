/*
 * stem.h — C ABI of the Stem long-context prefill hot path on NVIDIA B200 (sm_100a).
 *
 * The method (sources are cited by page title and section):
 *  - "Stem: Rethinking Causal Information Flow in Sparse Attention", AngelSlim
 *    documentation (stem.md), §2.1 Block-Level Scoring, §2.2 Top-k Schedule,
 *    §2.3 Block-Sparse Attention, §6 parameter table.
 *  - the same paper's gist.science summaries (zh §2.1 TPD, §2.2 OAM, §2.3 flow;
 *    de §2 Methodik A/B/C).
 *  - the youleyou article on Stem and the HPC-BSA operator, §2.2 (log form of
 *    the metric) and §3.1 (skip decisions made outside the inner loop; skipped
 *    blocks are equivalent to -inf scores).
 *
 * Pipeline: stem_prefill = stem_score (value-norm bonus + anti-diagonal
 * downsampled scoring + block max-pool) -> stem_select (token position-decay
 * budget + top-k with sink and window blocks, emitted as CSR block lists) ->
 * stem_bsa_fwd (causal block-sparse flash attention over the listed blocks).
 *
 * Conventions common to every entry point:
 *  - All tensor pointers are DEVICE pointers unless the name ends in _host.
 *  - The library allocates nothing.  The caller owns every buffer, including
 *    the workspace `ws`, whose size stem_plan() reports.
 *  - Every compute call is asynchronous on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream) and performs no host<->device copy and no
 *    host synchronisation.
 *  - Argument errors are detected on the host and returned before anything is
 *    enqueued.  Errors the GPU detects (a malformed block list, a pipeline
 *    wait that ran out) are written to a status word inside `ws`; read it with
 *    stem_read_device_status().  Each compute call clears that word first.
 *  - Tensors: q [T, Hq, d], k and v [T, Hkv, d], d contiguous, rows of all
 *    sequences packed back to back (cu_seqlens), every base pointer 16-byte
 *    aligned.  d must be 128 and Hq a multiple of Hkv (grouped-query attention:
 *    query head h reads KV head h / (Hq/Hkv)).
 *  - Blocks: each sequence is cut into NB_s = ceil(L_s / 128) blocks of 128
 *    tokens (the last one may be partial).  Global block index g runs over
 *    the blocks of sequence 0, then sequence 1, ...; NBtot = sum NB_s and
 *    nb_max = max NB_s.  Row r = h * NBtot + g of every per-row array belongs
 *    to query head h and query block g.
 */
#ifndef STEM_H
#define STEM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define STEM_API __attribute__((visibility("default")))
#else
#define STEM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so the header needs no CUDA include. */
typedef struct CUstream_st* stem_stream_t;

typedef enum {
  STEM_OK = 0,
  STEM_ERR_INVALID_ARG = 1,          /* a size, parameter or pointer is out of its documented range */
  STEM_ERR_UNSUPPORTED = 2,          /* valid but not implemented here (e.g. head_dim != 128) */
  STEM_ERR_WORKSPACE_TOO_SMALL = 3,  /* ws_bytes below what stem_plan() reported for this call */
  STEM_ERR_MISALIGNED = 4,           /* a tensor base pointer is not 16-byte aligned */
  STEM_ERR_CUDA = 5,                 /* a CUDA runtime/driver call failed (launch, tensor-map encode) */
  STEM_ERR_TIMEOUT = 6,              /* device: a pipeline wait exceeded its bound; outputs are invalid */
  STEM_ERR_BAD_BLOCKLIST = 7         /* device: a CSR entry was out of range or not strictly ascending;
                                        the offending entry was skipped */
} stem_status_t;

typedef enum { STEM_BF16 = 0, STEM_FP8_E4M3 = 1 } stem_dtype_t;

/* How keep_ratio sets k_start of the position-decay budget (the pages leave the
 * mapping open):
 *   RELATIVE (default): k_start of query block i is ceil(rho * (i + 1)), i.e. a
 *            fraction of the i+1 causal key blocks of that row;
 *   ABSOLUTE: k_start = ceil(rho * NB_s) for every row of the sequence. */
typedef enum { STEM_BUDGET_RELATIVE = 0, STEM_BUDGET_ABSOLUTE = 1 } stem_budget_mode_t;

/* Form of the value-magnitude bonus of the output-aware metric. */
typedef enum {
  STEM_BONUS_LOG = 0,          /* beta * max(0, ln ||v||^2)  [gist-zh §2.2; gist-de §2 C] */
  STEM_BONUS_STANDARDIZED = 1  /* beta * ReLU(standardized ln ||v||^2)  [AngelSlim doc §2.1;
                                  the statistics' scope is this library's reading] */
} stem_bonus_mode_t;

/* Granularity of the block lists under GQA. */
typedef enum {
  STEM_LIST_PER_HEAD = 0,  /* every query head selects its own blocks */
  STEM_LIST_PER_GROUP = 1  /* one list per (KV head, query block), selected on the
                              elementwise max of its query heads' scores (NaN as
                              -inf) and written to every query head of the group */
} stem_list_mode_t;

/* Where the top-k selection runs (the results are the same, bit for bit). */
typedef enum {
  STEM_SELECT_SEPARATE = 0,  /* a selection kernel, one warp per list, after the scoring kernel */
  STEM_SELECT_FUSED = 1      /* the scoring CTAs select the rows they scored, after their last key
                                tile (per-head lists of at most 5888 blocks; otherwise as SEPARATE) */
} stem_select_mode_t;

/* Method parameters (AngelSlim documentation §6 defaults in brackets). */
typedef struct {
  int32_t block_size;     /* block of the scores, lists and attention [128]: 128 or 64 (the
                             "64x128 or 128x128" KV blocks of the HPC-BSA article §3.1);
                             with 64, sequences of at most 2,097,152 tokens
                             (STEM_ERR_UNSUPPORTED beyond) */
  int32_t stride;         /* scoring downsampling stride s [8]; 4 or 8 are supported */
  int32_t chunk_size;     /* scoring query-chunk width [2048]; > 0; does not change results */
  double  norm;           /* extra scoring normalisation n [1.0]; > 0 */
  double  beta;           /* weight of the value-magnitude bonus [0.2]; >= 0 */
  double  keep_ratio;     /* rho in (0, 1] */
  double  mu;             /* decay factor (stem_alpha of this layer) in (0, 1] [1.0; 0.7 best] */
  int32_t sink_blocks;    /* initial blocks always kept [4]; >= 0 */
  int32_t window_blocks;  /* trailing causal blocks always kept, the diagonal included [4]; >= 1 */
  double  softmax_scale;  /* attention logit scale; 0 selects 1/sqrt(head_dim) */
  int32_t budget_mode;    /* stem_budget_mode_t */
  int32_t bonus_mode;     /* stem_bonus_mode_t [STEM_BONUS_LOG] */
  int32_t list_mode;      /* stem_list_mode_t [STEM_LIST_PER_HEAD] */
  int32_t select_mode;    /* stem_select_mode_t [STEM_SELECT_SEPARATE]; no effect on results */
} stem_params_t;

/* Query/key/value description shared by all calls. */
typedef struct {
  int32_t dtype;                  /* stem_dtype_t of q, k and v */
  int32_t num_seqs;               /* >= 1 */
  int32_t total_tokens;           /* T = cu_seqlens[num_seqs] */
  const int32_t* cu_seqlens;      /* device [num_seqs + 1], cu[0] = 0, non-decreasing */
  const int32_t* cu_seqlens_host; /* host copy of the same offsets (used for planning and
                                     launch geometry; read during the call only) */
  int32_t num_q_heads;            /* Hq */
  int32_t num_kv_heads;           /* Hkv, divides Hq */
  int32_t head_dim;               /* d; must be 128 */
  const void* q;                  /* [T, Hq, d] bf16 or e4m3 bytes */
  const void* k;                  /* [T, Hkv, d] */
  const void* v;                  /* [T, Hkv, d] */
  const float* q_scale;           /* fp8 only: device [Hq]  dequantisation scales (value = e4m3 * scale) */
  const float* k_scale;           /* fp8 only: device [Hkv] */
  const float* v_scale;           /* fp8 only: device [Hkv] */
} stem_qkv_t;

/* K and V in a page pool instead of packed storage (the paged fp8 KV path of
 * AngelSlim doc §5; bf16 pages work the same way).  Token t of sequence s is
 * row t % page_size of page page_table[s * max_pages_per_seq + t / page_size];
 * each row is [Hkv, d] like a packed token row. */
typedef struct {
  int32_t page_size;          /* tokens per page; a multiple of 64 */
  int32_t num_pages;          /* pages in the pool (num_pages * page_size < 2^31) */
  int32_t max_pages_per_seq;  /* row length of page_table; pages must cover every
                                 sequence rounded up to a multiple of 128 tokens */
  const int32_t* page_table;  /* device int32 [num_seqs][max_pages_per_seq] */
  const void* k_pages;        /* device [num_pages, page_size, Hkv, d] bf16 or e4m3 bytes */
  const void* v_pages;        /* device, same shape */
} stem_paged_kv_t;

/* Sizes derived on the host from (cu_seqlens_host, params); data-independent. */
typedef struct {
  int64_t nb_total;          /* NBtot */
  int64_t nb_max;            /* nb_max */
  int64_t num_rows;          /* Hq * NBtot (length of budgets; row_ptr has num_rows + 1) */
  int64_t nnz;               /* total listed blocks = sum of the budgets over all rows */
  int64_t nnz_per_head;      /* nnz / Hq */
  size_t  scores_bytes;      /* bytes of the fp32 score matrix [Hq][NBtot][nb_max] */
  size_t  vbonus_bytes;      /* bytes of the fp32 bonus [Hkv][NBtot] */
  size_t  ws_bytes;          /* workspace for stem_score / stem_select / stem_bsa_fwd
                                (includes vwide_bytes) */
  size_t  ws_prefill_bytes;  /* workspace for stem_prefill (holds scores and the CSR) */
  double  attn_flops;        /* 4 d Hq * (sum over listed blocks of query-key pairs), causal
                                pairs only on the diagonal block */
  double  dense_attn_flops;  /* the same with every causal block listed */
  double  score_flops;       /* 2 * s * d * Hq * (16 x 16 group pairs per causal block pair) */
  size_t  vwide_bytes;       /* fp8: the workspace's f16 copy of V [T, Hkv, d] that the
                                attention reads (T * Hkv * d * 2 bytes); 0 for bf16 */
} stem_plan_t;

/* Validate (qkv, params) and fill *out.  Host only; touches no device memory
 * (only cu_seqlens_host is read).  [AngelSlim doc §2.2 / gist-zh §2.1: the
 * budget k(i) = floor(k_start - k_start (1 - mu) i / N) is data-independent,
 * so nnz and every size are known before any kernel runs.] */
STEM_API stem_status_t stem_plan(const stem_qkv_t* qkv, const stem_params_t* params, stem_plan_t* out);

/* Block scores [AngelSlim doc §2.1; gist-zh §2.2 OAM and §2.3 anti-diagonal
 * downsampling; gist-de §2 C].
 *   x[hk][g]      = ln max_{t in block g} ||v_t||^2
 *   vbonus[hk][g] = beta * max(0, x)                       (STEM_BONUS_LOG)
 *                   beta * max(0, (x - mean) / std)        (STEM_BONUS_STANDARDIZED:
 *                   mean and population std of the finite x of the same sequence
 *                   and KV head; 0 where x is not finite or std = 0)
 *   D[h][a][b]    = sum_{u<s} q[a s + u, h] . k[b s + s-1-u, h/G] / (sqrt(d) s n)
 *   scores[h][g][j] = max over the query groups a of block g and key groups b of
 *                     block j of D + vbonus[h/G][g0+j]   for j <= i (local index);
 *                     -inf for i < j < nb_max.
 * Layout: scores fp32 [Hq][NBtot][nb_max] (row r = h*NBtot+g, column = key block
 * index local to the sequence); vbonus fp32 [Hkv][NBtot] (may be NULL, then the
 * workspace holds it).  Groups whose first token is past the sequence end are
 * ignored; missing tokens of the last group count as zero. */
STEM_API stem_status_t stem_score(const stem_qkv_t* qkv, const stem_params_t* params,
                         float* scores, float* vbonus,
                         void* ws, size_t ws_bytes, stem_stream_t stream);

/* Position-decay budgets and top-k block lists [gist-zh §2.1 TPD; AngelSlim doc
 * §2.2 sink and window blocks; youleyou §3.1 compacted lists].
 *   c = i + 1, F = {0 .. min(S,c)-1} u {max(0,c-W) .. i}
 *   k_start = ceil(rho * c) (RELATIVE) or ceil(rho * NB_s) (ABSOLUTE)
 *   k = floor(k_start - ((k_start * (1 - mu)) * i) / NB_s)   (IEEE fp64, this order)
 *   b = min(c, max(k, |F|))
 *   row = F u the b-|F| best other causal blocks by (score desc, index asc),
 *         NaN ranked as -inf, written in ascending order.
 * STEM_LIST_PER_GROUP: the rows of the G query heads of a KV head share one list,
 *         selected on the elementwise max of their score rows.
 * Outputs: budgets int32 [Hq*NBtot], row_ptr int32 [Hq*NBtot + 1] (row_ptr[0] = 0),
 * col_idx int32 [nnz] (key-block indices local to the sequence). */
STEM_API stem_status_t stem_select(const stem_qkv_t* qkv, const stem_params_t* params,
                          const float* scores, int32_t* budgets, int32_t* row_ptr,
                          int32_t* col_idx, void* ws, size_t ws_bytes, stem_stream_t stream);

/* stem_score and stem_select in one call: same arguments and outputs as the two
 * calls (scores, vbonus, budgets, row_ptr, col_idx), results bit for bit equal.
 * With select_mode = STEM_SELECT_FUSED, per-head lists and nb_max <= 5888 each
 * scoring CTA selects the rows it has just scored (the budgets run first), so
 * the scores are read back from L2 and no separate selection pass runs;
 * otherwise (the default) the two passes run in turn. */
STEM_API stem_status_t stem_score_select(const stem_qkv_t* qkv, const stem_params_t* params,
                                float* scores, float* vbonus,
                                int32_t* budgets, int32_t* row_ptr, int32_t* col_idx,
                                void* ws, size_t ws_bytes, stem_stream_t stream);

/* Causal block-sparse attention over caller-given CSR lists [gist-zh §2.3 exact
 * softmax over the chosen blocks only; youleyou §3.1].
 *   For query token t of block i of row r: keys = union over j in
 *   col_idx[row_ptr[r] .. row_ptr[r+1]) of the tokens u of block j with u <= t.
 *   out[t][h] = sum softmax(sigma q_t . k_u) v_u,  lse[h][t] = ln sum exp(sigma q_t . k_u),
 *   sigma = softmax_scale (or 1/sqrt(d)), times q_scale*k_scale for fp8.
 * out bf16 [T, Hq, d]; lse fp32 [Hq][T].  Lists must be strictly ascending with
 * 0 <= j <= i; a violating entry is skipped and STEM_ERR_BAD_BLOCKLIST recorded.
 * An empty row gives out = 0 and lse = -inf.  fp8: Q K^T runs on the e4m3
 * operands; P is kept in f16 and P.V runs as an f16 product against V widened
 * to f16 in the workspace (exact: every e4m3 value is an f16 value), since an
 * e4m3 P (three mantissa bits) would miss the fp8 output tolerance.
 * params->list_mode = STEM_LIST_PER_GROUP declares that the rows of the query
 * heads of each KV group are identical (as stem_select writes them): each CTA
 * then computes two query heads of one query block and stages each K/V tile
 * once for both.  Rows of a pair that differ are reported as
 * STEM_ERR_BAD_BLOCKLIST (the second head is then computed on the first
 * head's list). */
STEM_API stem_status_t stem_bsa_fwd(const stem_qkv_t* qkv, const stem_params_t* params,
                           const int32_t* row_ptr, const int32_t* col_idx,
                           void* out, float* lse,
                           void* ws, size_t ws_bytes, stem_stream_t stream);

/* stem_bsa_fwd with K and V read through a page table (qkv->k and qkv->v are
 * not used and may be NULL; q, cu_seqlens and the fp8 scales as for
 * stem_bsa_fwd).  Results equal stem_bsa_fwd's on the packed K/V the pages
 * hold, bit for bit.  Page rows past a sequence's last token (up to its next
 * multiple of the block size) are read: they must hold finite values, zeros
 * for example.
 * A page number outside [0, num_pages) reads zeros.  STEM_ERR_INVALID_ARG for
 * a page size that is not a positive multiple of 64 or a table too short for
 * some sequence. */
STEM_API stem_status_t stem_bsa_fwd_paged(const stem_qkv_t* qkv, const stem_paged_kv_t* kv,
                                 const stem_params_t* params,
                                 const int32_t* row_ptr, const int32_t* col_idx,
                                 void* out, float* lse,
                                 void* ws, size_t ws_bytes, stem_stream_t stream);

/* score -> select -> attention on one stream with no host round trip (the
 * selection placed as in stem_score_select).
 * row_ptr_out / col_idx_out may be NULL (the workspace then holds the lists);
 * ws_bytes >= plan.ws_prefill_bytes. */
STEM_API stem_status_t stem_prefill(const stem_qkv_t* qkv, const stem_params_t* params,
                           void* out, float* lse,
                           int32_t* row_ptr_out, int32_t* col_idx_out,
                           void* ws, size_t ws_bytes, stem_stream_t stream);

/* stem_prefill for inputs and outputs in host memory, with the transfers
 * overlapped with the computation.
 *   qkv        describes the layer as for stem_prefill; qkv->q, k, v point to
 *              DEVICE buffers of the full [T, H, d] size, which this call fills.
 *   q_host, k_host, v_host  the inputs in host memory, same layout (page-locked
 *              memory is needed for the copies to run asynchronously).
 *   out_dev, lse_dev        device buffers for O and LSE (as stem_prefill's).
 *   out_host, lse_host      host destinations for O bf16 [T, Hq, d] and LSE
 *              fp32 [Hq][T].
 *   ws, ws_bytes            as stem_prefill (ws_bytes >= plan.ws_prefill_bytes).
 * The layer is processed one group of KV heads (with their query heads) at a
 * time, at most 8 groups: the inputs of group g+1 are copied while group g
 * computes, the results of group g are copied back while g+1 computes.  The
 * work is ordered after the work already on `stream`, and `stream` completes
 * only once the results are in host memory; the call itself only enqueues.
 * Results equal stem_prefill's bit for bit.  Host-side errors as stem_prefill;
 * STEM_ERR_INVALID_ARG also for a NULL host pointer. */
STEM_API stem_status_t stem_prefill_host(const stem_qkv_t* qkv, const stem_params_t* params,
                                const void* q_host, const void* k_host, const void* v_host,
                                void* out_dev, float* lse_dev, void* out_host, float* lse_host,
                                void* ws, size_t ws_bytes, stem_stream_t stream);

/* stem_prefill without a caller workspace, for callers that cannot allocate
 * device memory (code running where cudaMalloc is not allowed or not wanted:
 * host callbacks, allocator hooks, plugins whose host owns every device
 * buffer, fixed memory pools).  The pages have no counterpart: this is a
 * deployment convenience of this library.
 *   Uses a built-in 32 MiB device array as the workspace; a problem whose
 *   plan.ws_prefill_bytes exceeds 32 MiB returns STEM_ERR_WORKSPACE_TOO_SMALL
 *   before anything is enqueued.  Allocates and frees nothing.
 *   Every GPU that loads the library keeps the 32 MiB until the process exits.
 *   All calls on a device share that array and it keeps the last call's
 *   contents: calls that may overlap on the GPU race; serialise them.
 *   The first call on each device looks up the array's address (with that
 *   device current); make it before any stream capture.  The address is kept
 *   for the life of the process and does not survive cudaDeviceReset.
 *   `stream` must belong to the current device: STEM_ERR_INVALID_ARG if not.
 *   Device-side errors go to the built-in workspace's status word: read them
 *   with stem_noalloc_read_device_status.
 * Arguments, outputs and host-side errors are those of stem_prefill. */
STEM_API stem_status_t stem_prefill_noalloc(const stem_qkv_t* qkv, const stem_params_t* params,
                                            void* out, float* lse,
                                            int32_t* row_ptr_out, int32_t* col_idx_out,
                                            stem_stream_t stream);

/* The device status word of stem_prefill_noalloc's built-in workspace on the
 * current device (no counterpart in the pages): synchronises `stream` (which
 * must belong to the current device) and copies the word into *out, STEM_OK
 * or the device-side error of the last call (STEM_ERR_TIMEOUT,
 * STEM_ERR_BAD_BLOCKLIST).  Each stem_prefill_noalloc call clears it first.
 * Returns STEM_ERR_INVALID_ARG for a NULL `out` or a stream of another device,
 * STEM_ERR_CUDA if the copy fails. */
STEM_API stem_status_t stem_noalloc_read_device_status(stem_stream_t stream, stem_status_t* out);

/* Self-test of the device-side failure detection (no counterpart in the
 * pages).  Launches one kernel that waits, through the same bounded wait the
 * pipelines use, on a barrier nothing arrives on; after the 2 s bound it
 * records STEM_ERR_TIMEOUT in the status word of `ws` (>= 256 bytes) and
 * returns.  Read the result with stem_read_device_status(); the context stays
 * usable.  Nothing faults, traps or hangs. */
STEM_API stem_status_t stem_selftest_wait_timeout(void* ws, stem_stream_t stream);

/* Synchronise `stream` and read the device status word of `ws` into *out.
 * Returns STEM_ERR_CUDA if the copy fails. */
STEM_API stem_status_t stem_read_device_status(const void* ws, stem_stream_t stream, stem_status_t* out);

/* Static string for a status code; never NULL. */
STEM_API const char* stem_status_string(stem_status_t status);

/* Library version, MAJOR*10000 + MINOR*100 + PATCH. */
STEM_API int32_t stem_version(void);

#ifdef __cplusplus
}
#endif

#endif /* STEM_H */
