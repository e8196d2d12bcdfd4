/*
 * dsaidx.h — C ABI of the B200 (sm_100a) DSA lightning-indexer library.
 *
 * What the library computes (sources are the pages this project restates):
 *
 *   DSA indexer score.  H_I indexer query heads q_{t,j} (dimension d) share one
 *   indexer key k_s per token; each head carries a weight w_{t,j}:
 *       I_{t,s} = sum_j  w_{t,j} * ReLU(q_{t,j} . k_s)
 *   Every query scans its whole causal prefix and keeps a token-level top-k
 *   ("PaperTrace 2.2.2 MISA, LISA and ResMiSA", opening definition of the DSA
 *   score and section 2.2 "kernel boundary"; "The new bottleneck of sparse
 *   attention", section "level three: DeepSeek DSA").
 *
 *   MISA (head routing).  Pool keys into M = ceil(L/B) blocks, score each head
 *   by E_{t,j} = (1/M) sum_b |w_{t,j} ReLU(q_{t,j} . k~_b)|, keep the top-h
 *   heads, score every legal token with those heads only, take the top-k.
 *   MISA-dagger keeps k' candidates from that pass and reranks them with all
 *   H_I heads ("MISA: Mixture of Indexer Sparse Attention", method steps 1-6).
 *
 *   HISA (block -> token hierarchy).  Mean-pool keys into blocks of b tokens,
 *   score the representatives with the same indexer query, keep the top-r
 *   blocks and rerank only their tokens with the full formula
 *   ("PaperTrace 2.2.2", section 2.1 "HISA"; "The new bottleneck of sparse
 *   attention", section "route one: HISA").
 *
 * Conventions shared by every call
 *   - All tensor pointers are DEVICE pointers, row-major, densely packed:
 *       q      [batch, n_q, heads, dim]   dtype q_dtype
 *       q_scale[batch, n_q]  fp32         required iff q_dtype == DSA_E4M3
 *       k      [batch, n_k, dim]          dtype k_dtype
 *       k_scale[batch, n_k]  fp32         required iff k_dtype == DSA_E4M3
 *       w      [batch, n_q, heads] fp32
 *       out_idx   [batch, n_q, topk] int32
 *       out_score [batch, n_q, topk] fp32
 *     bf16 is passed as raw 16-bit words, e4m3 as raw bytes (OCP FP8 E4M3).
 *     The dequantised operand is scale * code; the scale of a key multiplies
 *     its whole row, the scale of a query multiplies all heads of that query.
 *   - Causality.  Query i of sequence b sits at position pos = q_pos0[b] + i
 *     (q_pos0 == NULL: pos0 = n_k - n_q).  Its legal keys are
 *     0 <= s <= pos and s < k_len[b] (k_len == NULL: n_k).
 *   - Output contract.  Each query row receives its top-k set: the
 *     min(topk, |legal|) legal keys that are best by (score descending, index
 *     ascending) — the lower index wins a tie — followed by padding (index -1,
 *     score -inf).  The entries come in an unspecified order unless
 *     DSA_FLAG_SORTED is set, which orders them by (score descending, index
 *     ascending), or DSA_FLAG_BY_POSITION, which orders them by index.  Sparse attention consumes the set, so order is optional
 *     ("PaperTrace 2.2.2", section 2.2: indices returned by the top-k are
 *     unordered or score-ordered).  -0.0 is written as +0.0.  The reported
 *     score is the one the final selection used: the full I for dsa_index,
 *     misa_dagger_index and hisa_index (route_h == 0); the routed-head score
 *     for misa_index and the stacked hisa_index.
 *   - Memory.  The caller owns every buffer (inputs, outputs, workspace) and
 *     the stream.  The library allocates no device memory, keeps no global
 *     state between calls and never synchronises the stream unless
 *     DSA_FLAG_CHECK is set.  Calls are asynchronous on `stream` (a
 *     cudaStream_t passed as void*; NULL = the legacy default stream).  Two
 *     calls in flight at once need two distinct workspaces.
 *   - Alignment.  q, k and the workspace start on 16-byte boundaries (the scan
 *     reads q, k and buffers inside the workspace with TMA copies); every other
 *     array is aligned to its element size.  A misaligned q, k or workspace
 *     returns DSA_ERR_INVALID before any launch.
 *   - Errors.  Every call returns DSA_OK (0) or a negative status; nothing is
 *     thrown across the ABI.  Argument errors are detected on the host before
 *     any launch.  A bounded device wait that expires (DSA_ERR_TIMEOUT) or a
 *     non-finite scale (DSA_ERR_NONFINITE, only checked under DSA_FLAG_CHECK)
 *     is recorded in a status word inside the workspace; with DSA_FLAG_CHECK the
 *     call synchronises the stream and returns it, otherwise
 *     dsa_read_status() returns it after the caller synchronises.
 *   - Supported shapes: dim == 128; heads a power of two in [8, 128];
 *     topk in [1, 8192]; n_k <= 2^24.  Anything else returns
 *     DSA_ERR_UNSUPPORTED.
 */
#ifndef DSAIDX_H
#define DSAIDX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  DSA_OK = 0,
  DSA_ERR_INVALID = -1,      /* null pointer, negative size, inconsistent shape */
  DSA_ERR_UNSUPPORTED = -2,  /* dtype / dim / heads / topk outside the supported set */
  DSA_ERR_WORKSPACE = -3,    /* workspace NULL or smaller than dsa_workspace_size() */
  DSA_ERR_CUDA = -4,         /* a CUDA runtime call or launch failed */
  DSA_ERR_NONFINITE = -5,    /* a scale is NaN, inf, zero or negative (DSA_FLAG_CHECK) */
  DSA_ERR_TIMEOUT = -6,      /* a bounded device-side wait expired */
  DSA_ERR_INTERNAL = -7      /* a device-side capacity or bounds check failed (a library
                                fault; the outputs of that call are not to be used) */
};

typedef enum { DSA_F32 = 0, DSA_BF16 = 1, DSA_E4M3 = 2 } dsa_dtype;

/* Algorithm ids for dsa_workspace_size(). */
enum {
  DSA_ALGO_DSA = 0,
  DSA_ALGO_MISA = 1,
  DSA_ALGO_MISA_DAGGER = 2,
  DSA_ALGO_HISA = 3,
  DSA_ALGO_LISA = 4,     /* indexer LISA and LISA-dagger (lisa_index) */
  DSA_ALGO_RESMISA = 5   /* ResMiSA (resmisa_index) */
};

/* problem.flags */
#define DSA_FLAG_CHECK 1u  /* validate scales/lengths on device, synchronise, return device status */
#define DSA_FLAG_SORTED 2u /* order each row's top-k by (score desc, index asc) */
/* Order each row's top-k by token position (index ascending), the order in which
 * a sparse attention kernel gathers the selected keys most contiguously
 * ("PaperTrace 2.2.2", section 2.2: re-sorting score-ordered indices by
 * position makes the gather more contiguous).  Not with DSA_FLAG_SORTED. */
#define DSA_FLAG_BY_POSITION 4u
/* DoSA bound pruning ("The new bottleneck of sparse attention", route five:
 * DoSA, exact pruning by upper and lower bounds).  dsa_index / dsa_index_scan
 * first compute, for every query row and every 1024-token key block, an upper
 * and a lower bound of I over the block's keys from the block's per-dimension
 * key range.  The blocks of largest lower bound holding k legal keys (the seed
 * set) give each row a starting threshold that none of its k best keys can be
 * below; the scan raises it as it goes, filters candidates by it, and skips the
 * head sums of a (row, 128-key tile) pair whose block's upper bound lies below
 * it.  The selected set and scores are bit-identical to the call without the
 * flag; only the work differs.  bf16 q and k, heads >= 32; otherwise
 * DSA_ERR_UNSUPPORTED.  Needs the larger workspace dsa_workspace_size reports
 * for the flagged problem.  dsa_read_pruned returns the count of skipped pairs. */
#define DSA_FLAG_DOSA 8u
/* For tests of the timeout path only, never in production: dsa_index /
 * dsa_index_scan run with a wait budget of about 1 ms instead of about 4 s, and
 * the scan's first CTA withholds one stage of keys, so its bounded waits run
 * out.  The call then records DSA_ERR_TIMEOUT, every role of that CTA drains
 * its own copies and MMAs and exits, the select writes padding rows, and the
 * GPU context stays usable for the next call. */
#define DSA_FLAG_TEST_STALL 0x80000000u

typedef struct {
  int32_t batch;          /* sequences */
  int32_t n_q;            /* query rows per sequence */
  int32_t n_k;            /* key rows per sequence */
  int32_t heads;          /* H_I */
  int32_t dim;            /* indexer dimension d */
  int32_t topk;           /* k */
  int32_t q_dtype;        /* dsa_dtype */
  int32_t k_dtype;        /* dsa_dtype; must equal q_dtype except (q BF16, k E4M3) */
  const int32_t* q_pos0;  /* device [batch] or NULL */
  const int32_t* k_len;   /* device [batch] or NULL */
  uint32_t flags;
} dsa_problem;

/* Routing / hierarchy parameters (ignored fields may be zero).
 *   misa_block  B  : tokens per pooled key of the MISA router (e.g. 1024)
 *   misa_h      h  : routed heads kept per query (e.g. 8); a power of two in
 *                    [8, heads]
 *   k_prime     k' : MISA-dagger candidate pool (e.g. 8192), topk <= k' <= 8192
 *   hisa_block  b  : tokens per HISA block (e.g. 64)
 *   hisa_r      r  : HISA blocks kept per query (e.g. 128), r * b <= 8192
 * Block sizes must be powers of two in [16, 4096], and the router sees at
 * most 224 full blocks: n_k / B <= 224 (B = 1024 covers 229,376 tokens).
 * The routed entry points take bf16 q and k only (q_dtype == k_dtype ==
 * DSA_BF16; anything else returns DSA_ERR_UNSUPPORTED) and batch <= 65535.
 * Their workspace holds the pooled keys, the routed query rows and the
 * candidate logs of one chunk of query rows; long prefills run in several
 * row chunks so that the logs stay within 8 GiB. */
typedef struct {
  int32_t misa_block;
  int32_t misa_h;
  int32_t k_prime;
  int32_t hisa_block;
  int32_t hisa_r;
  int32_t lisa_pool;   /* M: LISA-dagger pool, topk <= M <= 8192 (0: plain indexer LISA) */
  int32_t res_block;   /* ResMiSA router block B: a power of two in [16, 4096] */
  int32_t res_r;       /* ResMiSA residual heads r, 0 <= r <= min(heads, 124) */
} dsa_route_params;

/* Bytes of device workspace that `algo` needs for problem `p` (route params
 * may be NULL for DSA_ALGO_DSA).  Writes *bytes; returns a status. */
int dsa_workspace_size(const dsa_problem* p, int32_t algo, const dsa_route_params* rp,
                       size_t* bytes);

/* Query rows per sequence that a routed entry point (algo MISA, MISA_DAGGER or
 * HISA) processes per row chunk for problem p: its scan and select launches
 * repeat once per chunk of *rows rows.  Host only; returns a status. */
int dsa_route_chunk_rows(const dsa_problem* p, int32_t algo, const dsa_route_params* rp,
                         int32_t* rows);

/* DSA lightning-indexer top-k: score -> causal mask -> token top-k. */
int dsa_index(const dsa_problem* p, const void* q, const float* q_scale, const void* k,
              const float* k_scale, const float* w, int32_t* out_idx, float* out_score,
              void* workspace, size_t workspace_bytes, void* stream);

/* dsa_index without a caller-provided workspace, for callers that cannot
 * allocate device memory when they call (a serving loop whose memory plan is
 * fixed after start-up, or a host framework whose own allocator owns all
 * device memory and forbids side allocations).  The pages describe no such
 * call; it exists for those callers only.  Scratch is a fixed 64 MiB array in
 * device memory inside the library (held on every GPU that loads the library,
 * until the process exits); problems whose dsa_workspace_size() exceeds
 * 64 MiB are rejected with DSA_ERR_WORKSPACE.  Nothing is allocated or freed.
 * The first call on a device looks up that device's scratch address (a
 * one-time set-up per device; make that first call before any stream
 * capture).  Every call on a device shares the one scratch array, so calls
 * whose executions overlap on the GPU (different streams, no ordering between
 * them) race and corrupt each other's results; order them on one stream or
 * with events.  The scratch address is looked up once per device and kept, so
 * the library must not be used on a device again after cudaDeviceReset there.
 * A device-side status (a bounded wait that expired, or a bad scale or length
 * under DSA_FLAG_CHECK) is recorded in that scratch, which the caller cannot
 * read with dsa_read_status: pass DSA_FLAG_CHECK to have the call synchronise
 * the stream and return the device status itself (without it an expired wait
 * shows only as padded output rows).  Other arguments and results are as for
 * dsa_index. */
int dsa_index_noalloc(const dsa_problem* p, const void* q, const float* q_scale, const void* k,
                      const float* k_scale, const float* w, int32_t* out_idx, float* out_score,
                      void* stream);

/* The two stages of dsa_index, for callers that schedule (or time) them
 * separately: dsa_index is exactly dsa_index_scan followed by
 * dsa_index_select on the same workspace and stream.  The scan stage scores
 * every legal (query, key) pair and leaves per-row candidate logs in the
 * workspace; the select stage takes each row's exact top-k from them and
 * writes the outputs. */
int dsa_index_scan(const dsa_problem* p, const void* q, const float* q_scale, const void* k,
                   const float* k_scale, const float* w, void* workspace, size_t workspace_bytes,
                   void* stream);
int dsa_index_select(const dsa_problem* p, int32_t* out_idx, float* out_score, void* workspace,
                     size_t workspace_bytes, void* stream);

/* MISA: block-pooled router picks rp->misa_h heads per query, those heads score
 * every legal token, token top-k.  out_heads [batch,n_q,h] int32 (ascending head
 * order) and out_E [batch,n_q,heads] fp32 (the router importance E) are optional
 * (NULL skips them).  Router: full blocks of the legal prefix plus the boundary
 * block (the mean of its legal tokens); heads ranked by
 * S_{t,j} = sum_b |w_{t,j}| ReLU(q_{t,j} . k~_b) = M_t E_{t,j}, ties to the
 * lower head index. */
int misa_index(const dsa_problem* p, const dsa_route_params* rp, const void* q,
               const void* k, const float* w, int32_t* out_idx, float* out_score,
               int32_t* out_heads, float* out_E, void* workspace, size_t workspace_bytes,
               void* stream);

/* MISA-dagger: the MISA pass keeps rp->k_prime candidates, which are reranked
 * by the full H_I-head score; final token top-k.  out_heads as for misa_index;
 * out_pool [batch,n_q,k_prime] int32 (optional) receives the first-pass pool
 * (unordered, padded with -1). */
int misa_dagger_index(const dsa_problem* p, const dsa_route_params* rp, const void* q,
                      const void* k, const float* w, int32_t* out_idx, float* out_score,
                      int32_t* out_heads, int32_t* out_pool, void* workspace,
                      size_t workspace_bytes, void* stream);

/* HISA: score block representatives (blocks of rp->hisa_block tokens), keep
 * rp->hisa_r blocks, rerank their legal tokens, token top-k.  With
 * rp->misa_h > 0 the MISA router (rp->misa_block) first picks misa_h heads and
 * both HISA stages use only those heads (the stacked variant).  out_blocks
 * [batch,n_q,r] int32 (optional) receives the kept block ids (unordered,
 * padded with -1); out_heads [batch,n_q,h] (optional, stacked only). */
int hisa_index(const dsa_problem* p, const dsa_route_params* rp, const void* q,
               const void* k, const float* w, int32_t* out_idx, float* out_score,
               int32_t* out_blocks, int32_t* out_heads, void* workspace,
               size_t workspace_bytes, void* stream);

/* Indexer LISA ("PaperTrace 2.2.2", section 3.1: the shared key lets the linear
 * part of every head merge exactly, since ReLU(x) = x + ReLU(-x)): the fused
 * query g_t = sum_j w_{t,j} q_{t,j} scores every legal token by the linear term
 * l_{t,s} = g_t . k_s alone, and the top-k by l is returned with l as its score.
 * With rp->lisa_pool = M > 0 (LISA-dagger) the top-M by l form a pool that is
 * reranked by the full score I over every head: top-k of I, scores I;
 * out_pool [batch, n_q, M] int32 (optional) receives the pool (unordered,
 * -1 padded).  The pool is the exact top-min(M, |legal|) by l (ties to the lower
 * index), one fixed size within the page's range for it.  g is accumulated in
 * fp32 over the heads in ascending order and enters the tensor core as two bf16
 * parts (hi + lo, about 16 significant bits).  bf16 q and k only. */
int lisa_index(const dsa_problem* p, const dsa_route_params* rp, const void* q, const void* k,
               const float* w, int32_t* out_idx, float* out_score, int32_t* out_pool,
               void* workspace, size_t workspace_bytes, void* stream);

/* ResMiSA ("PaperTrace 2.2.2", section 3.2, MISA-2): the linear term l of every
 * head plus r routed residual heads,
 *   I^_{t,s} = l_{t,s} + sum_{j in A_t} w_{t,j} ReLU(-q_{t,j} . k_s).
 * Router: the legal prefix is cut into blocks of rp->res_block tokens (the last
 * holds only legal tokens); with the per-dimension key range [kmin, kmax] of
 * block b, U-_{t,b,j} = sum_c max(q_c,0)(-kmin_c) + max(-q_c,0) kmax_c bounds
 * -q_{t,j} . k over the block; S_{t,j} = |w_{t,j}| max_b ReLU(U-); A_t = the r
 * heads of largest S (ties to the lower head), ascending in out_heads
 * [batch, n_q, r] (optional); out_S [batch, n_q, heads] fp32 (optional).  The
 * reported score is I^ (r = heads gives the DSA score, r = 0 the LISA score).
 * bf16 q and k only. */
int resmisa_index(const dsa_problem* p, const dsa_route_params* rp, const void* q, const void* k,
                  const float* w, int32_t* out_idx, float* out_score, int32_t* out_heads,
                  float* out_S, void* workspace, size_t workspace_bytes, void* stream);

/* Sparse MLA on a fixed set of selected positions ("PaperTrace 2.2.2", section
 * 2.2: the indexer's top-k positions feed Sparse MLA, which reads the latent
 * KV at those positions; section 2.3, acceptance step two: with the set fixed,
 * check logits, row maximum, softmax denominator and output against a naive
 * gather attention).  Token t (sequence t / tokens_per_seq) with absorbed
 * query heads q_{t,h} attends to the cached rows kv_s of its selected
 * positions s = idx[t, i] (entries < 0 or >= n_k are empty):
 *     x_s = scale * q_{t,h} . kv_s,   o_{t,h} = sum_s softmax(x)_s kv_s[0:dim_v],
 *     lse_{t,h} = log sum_s exp(x_s)      (natural log; -inf for an empty set)
 * The value is the latent part of the row (its first dim_v dimensions); the
 * trailing dim_qk - dim_v (rope) dimensions join the logits only.
 *   q   [batch * tokens_per_seq, heads, dim_qk] bf16
 *   kv  [batch, n_k, dim_qk] bf16
 *   idx [batch * tokens_per_seq, topk] int32 (any order; DSA_FLAG_BY_POSITION
 *       output gathers most contiguously)
 *   out [batch * tokens_per_seq, heads, dim_v] bf16; out_lse [.., heads] fp32 or NULL
 * Supported: dim_qk == 576, dim_v == 512 (MLA latent 512 + rope 64), heads <= 128.
 * The softmax weights enter the value product in bf16 (fp32 accumulation).
 * workspace: >= 256 bytes (status word; DSA_FLAG_CHECK synchronises and
 * returns it). */
typedef struct {
  int32_t batch;
  int32_t tokens_per_seq;
  int32_t n_k;
  int32_t heads;
  int32_t dim_qk;
  int32_t dim_v;
  int32_t topk;
  float scale;
  uint32_t flags;
} dsa_mla_problem;

int dsa_sparse_mla(const dsa_mla_problem* p, const void* q, const void* kv, const int32_t* idx,
                   void* out, float* out_lse, void* workspace, size_t workspace_bytes,
                   void* stream);

/* Indexer backward with score recompute ("PaperTrace 2.2.2", section 2.3 "why
 * training gradients need recomputation"): for the loss L = sum_t sum_{s in S_t}
 * g_{t,s} I_{t,s}, with z = q_{t,j} . k_s recomputed over each row's selected
 * positions and m = 1[z > 0] (ReLU's derivative 0 at 0):
 *   dq_{t,j} = sum_s g_{t,s} w_{t,j} m k_s        dq [batch, n_q, heads, dim] fp32, written
 *   dk_s    += sum_t sum_j g_{t,s} w_{t,j} m q_{t,j}  dk [batch, n_k, dim] fp32, ADDED TO
 *   dw_{t,j} = sum_s g_{t,s} ReLU(z)              dw [batch, n_q, heads] fp32, written
 * sel / grad [batch, n_q, p->topk]: selected positions (-1 empty) and the
 * upstream gradient on I at each.  q, k bf16 (dim 128), w fp32; heads == 64.
 * The products g w m enter the dq / dk tensor-core products in bf16 (fp32
 * accumulation); dw is exact up to fp32 sums.  dk receives one vector reduction
 * per (row, selected position), so its summation order is not fixed.
 * workspace >= 256 bytes (status word). */
int dsa_indexer_backward(const dsa_problem* p, const void* q, const void* k, const float* w,
                         const int32_t* sel, const float* grad, float* dq, float* dk, float* dw,
                         void* workspace, size_t workspace_bytes, void* stream);

/* dsa_index with the query rows and results in host memory ("PaperTrace 2.2.2
 * MISA, LISA and ResMiSA", section 2.3: the indexer runs once per layer on the
 * whole prefix, its inputs arriving from the host in serving): q_host [batch,
 * n_q, heads, dim], w_host [batch, n_q, heads] (and q_scale_host [batch, n_q]
 * for e4m3 q) in page-locked host memory, k / k_scale on the device as for
 * dsa_index, idx_host / score_host [batch, n_q, topk] in page-locked host
 * memory.  The rows stream in chunks of chunk_rows through two device slots in
 * `staging`: host->device copies on one library-owned stream, the scan and
 * select on `stream`, device->host copies on another, so the copies of one
 * chunk overlap the scan of the next.  The results equal dsa_index's (same
 * order rules and flags); work on `stream` after the call starts after every
 * result has reached the host.  staging: caller-owned device memory of at
 * least dsa_host_staging_size() bytes, 16-byte aligned; its first 256 bytes
 * hold the call's device status (the first error of any chunk), read with
 * dsa_read_status(staging) or returned under DSA_FLAG_CHECK.  Pageable host
 * memory also works but serialises the copies.  The two copy streams are
 * created on the first call on a device and kept for the process: do not call
 * it on a device again after a cudaDeviceReset there. */
int dsa_host_staging_size(const dsa_problem* p, int32_t chunk_rows, size_t* bytes);
int dsa_index_host(const dsa_problem* p, const void* q_host, const float* q_scale_host,
                   const void* k, const float* k_scale, const float* w_host,
                   int32_t* idx_host, float* score_host, int32_t chunk_rows, void* staging,
                   size_t staging_bytes, void* stream);

/* Operand preparation for the FP8 path: per-row scale a = amax/448 (amax == 0
 * gives a = 1), code = round-to-nearest-even, saturating e4m3 of x/a, both
 * divisions in IEEE fp32 ("PaperTrace 2.2.2", section 2.3 "from formula to
 * FP8 cache": k^ = round(k/a), FP8 data plus a scale).
 *   x [rows, cols] (x_dtype F32 or BF16), out [rows, cols] uint8, out_scale [rows]. */
int dsa_quantize_e4m3(const void* x, int32_t x_dtype, int64_t rows, int32_t cols,
                      uint8_t* out, float* out_scale, void* stream);

/* Device status word recorded in `workspace` by the last call that used it
 * (DSA_OK, DSA_ERR_TIMEOUT or DSA_ERR_NONFINITE).  Synchronises `stream`. */
int dsa_read_status(const void* workspace, void* stream);

/* The DoSA block bounds themselves ("The new bottleneck of sparse attention",
 * route five), as dsa_index computes them under DSA_FLAG_DOSA:
 * ub and lb [batch * n_q, ceil(n_k / 1024)] fp32 (caller-owned device memory;
 * lb may be NULL), for row t and block a (keys [1024 a, min(1024 (a + 1), n_k))
 * of its sequence), with slack = 2^-12 sum_j |w_j| ||q_j||_1 max_c max(|kmin_c|, |kmax_c|):
 *   UB = sum_j (w_j > 0 ? w_j ReLU(hi_j) : w_j ReLU(lo_j)) + slack,
 *   LB = sum_j (w_j > 0 ? w_j ReLU(lo_j) : w_j ReLU(hi_j)) - slack,
 * hi_j / lo_j the largest / smallest q_{t,j} . k over the block's
 * per-dimension key range [kmin, kmax]; -inf (both) for blocks past the row's
 * legal keys.  UB bounds every key's score in the block from above and LB from
 * below.  p->flags must include DSA_FLAG_DOSA (else DSA_ERR_INVALID);
 * workspace as dsa_workspace_size reports for that problem. */
int dsa_dosa_bounds(const dsa_problem* p, const void* q, const void* k, const float* w,
                    float* ub, float* lb, void* workspace, size_t workspace_bytes, void* stream);

/* DoSA pruning count recorded in `workspace` by the last dsa_index /
 * dsa_index_scan call with DSA_FLAG_DOSA: (query row, 128-key tile) pairs whose
 * head sums were skipped (0 without the flag).  Synchronises `stream`; the
 * count is written to *pruned.  DSA_ERR_INVALID for a null argument. */
int dsa_read_pruned(const void* workspace, void* stream, unsigned long long* pruned);

/* Human-readable text for a status code (static storage, never NULL). */
const char* dsa_status_string(int32_t status);

#ifdef __cplusplus
}
#endif

#endif /* DSAIDX_H */
